// Paged top-k decode: split-KV attention over gathered cache rows, then an LSE combine.
//
// Split kernel, one CTA per (split, kv head, sequence): the CTA takes a contiguous chunk of
// the canonical (ascending) token list of its (sequence, kv head), looks each token's page up
// in block_table, and streams the 256-byte K and V rows of those tokens through a 3-stage
// cp.async ring in shared memory (XOR-swizzled 16-byte chunks).  The G query heads of the kv
// head form the rows of a warp-level bf16 MMA (m16n8k16, fp32 accumulate): decode is bound by
// HBM bandwidth on the gathered rows, and this keeps the arithmetic to a few instructions per
// token.  Each warp keeps its own online-softmax state over a quarter of every 64-token tile;
// the four states are merged at the end and written as a normalised partial output plus its
// natural-log LSE.
//
// Combine kernel, one CTA per (sequence, q head): lse = log sum_s e^{lse_s};
// out = sum_s e^{lse_s - lse} o_s (the split-KV merge named by num_splits in the
// flash-attention-npu flash_attn_with_kvcache docstring; split-KV for decode load balance is
// listed in the Flash-Sparse-Attention README).  A split with no token has lse_s = -inf and
// weight 0; a row with no token at all outputs 0 and lse = -inf.
#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kDecThreads = 128;
constexpr int kTileTok = 64;  // tokens per pipeline stage; each warp owns 16 of them
constexpr int kDecStages = 3;
constexpr float kLn2d = 0.6931471805599453f;

template <int D>
struct DecCfg {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kChunks = D / 8;  // 16-byte chunks per row
    static constexpr int kTileBytes = kTileTok * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;  // K then V
    static constexpr int kOffStages = 0;
    static constexpr int kOffQ = kDecStages * kStageBytes;          // 16 rows x D bf16
    static constexpr int kOffRed = kOffQ + 16 * kRowBytes;          // float O[16][D]
    static constexpr int kOffStats = kOffRed + 16 * D * 4;          // m[4][16], l[4][16]
    static constexpr int kOffRows = kOffStats + 2 * 4 * 16 * 4;     // int rowoff[chunk]
};

// Byte offset of 16-byte chunk c of row r in a tile whose rows are D*2 bytes: the chunk index
// is XOR-ed with (r & 7) so eight consecutive rows read by ldmatrix hit distinct banks.
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)(r * DecCfg<D>::kRowBytes + ((c ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecSplitParams p)
{
    using C = DecCfg<D>;
    extern __shared__ __align__(128) uint8_t dsm[];
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = p.cnt[b * p.Hkv + hk];
    const int chunk = (n + p.S - 1) / p.S;
    const int begin = min(n, split * chunk);
    const int ntok = min(n, begin + chunk) - begin;
    int *rowoff = reinterpret_cast<int *>(dsm + C::kOffRows);
    float *red = reinterpret_cast<float *>(dsm + C::kOffRed);
    float *st_m = reinterpret_cast<float *>(dsm + C::kOffStats);
    float *st_l = st_m + 4 * 16;
    const uint32_t sbase = smem_u32(dsm);

    // Query rows of this kv head (rows >= G are zero) and the reduction buffer.
    {
        __nv_bfloat16 *sq = reinterpret_cast<__nv_bfloat16 *>(dsm + C::kOffQ);
        for (int e = threadIdx.x; e < 16 * D; e += kDecThreads) {
            const int rr = e / D, c = e % D;
            sq[e] = rr < p.G ? p.q[((int64_t)b * p.Hq + hk * p.G + rr) * D + c] : __float2bfloat16_rn(0.f);
            red[e] = 0.f;
        }
    }
    // Physical row of every token of the chunk (-1: the page is outside the pool).
    {
        const int32_t *toks = p.tok_c + ((int64_t)b * p.Hkv + hk) * p.topk + begin;
        bool bad = false;
        for (int e = threadIdx.x; e < ntok; e += kDecThreads) {
            const int pos = toks[e];
            const int pg = p.bt[(int64_t)b * p.max_pages + pos / p.page];
            if (pg < 0 || pg >= p.num_pages) {
                rowoff[e] = -1;
                bad = true;
            } else {
                rowoff[e] = (pg * p.page + pos % p.page) * p.Hkv + hk;
            }
        }
        if (bad && p.status) atomicOr(p.status, SFA_DEV_BAD_PAGE);
    }
    __syncthreads();

    // A fragments of Q for every k-step of 16.
    uint32_t aq[D / 16][4];
    {
        const int mi = lane >> 3;
        const int rr = (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t addr = sbase + C::kOffQ + rr * C::kRowBytes + (ks * 2 + (mi >> 1)) * 16;
            ldmatrix_x4(addr, aq[ks][0], aq[ks][1], aq[ks][2], aq[ks][3]);
        }
    }

    const int ntiles = (ntok + kTileTok - 1) / kTileTok;
    auto load_tile = [&](int stage, int tix) {
        const uint32_t kdst = sbase + C::kOffStages + stage * C::kStageBytes;
        const uint32_t vdst = kdst + C::kTileBytes;
        const int c = threadIdx.x % C::kChunks;
        for (int rr = threadIdx.x / C::kChunks; rr < kTileTok; rr += kDecThreads / C::kChunks) {
            const int e = tix * kTileTok + rr;
            const int ro = e < ntok ? rowoff[e] : -1;
            const int64_t off = ro >= 0 ? (int64_t)ro * D + c * 8 : 0;
            const uint32_t nbytes = ro >= 0 ? 16u : 0u;
            cp_async16(kdst + swz<D>(rr, c), p.kc + off, nbytes);
            cp_async16(vdst + swz<D>(rr, c), p.vc + off, nbytes);
        }
    };

    float o[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY};  // running max (base-2 scaled) of rows lane/4, lane/4+8
    float l_r[2] = {0.f, 0.f};              // this thread's share of the running sums

#pragma unroll
    for (int s = 0; s < kDecStages - 1; ++s) {
        if (s < ntiles) load_tile(s, s);
        cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
        cp_async_wait<kDecStages - 2>();
        __syncthreads();
        {
            const int nxt = it + kDecStages - 1;
            if (nxt < ntiles) load_tile(nxt % kDecStages, nxt);
            cp_async_commit();
        }
        const int stage = it % kDecStages;
        const uint32_t kt = sbase + C::kOffStages + stage * C::kStageBytes;
        const uint32_t vt = kt + C::kTileBytes;
        const int r0 = warp * 16;  // this warp's 16 tokens of the tile

        // S = Q K^T for tokens r0..r0+7 (s0) and r0+8..r0+15 (s1).
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int mi = lane >> 3;
            const int rr = r0 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t k0, k1, k2, k3;
                ldmatrix_x4(kt + swz<D>(rr, ks * 2 + (mi & 1)), k0, k1, k2, k3);
                mma_bf16_16816(s0, aq[ks], k0, k1);
                mma_bf16_16816(s1, aq[ks], k2, k3);
            }
        }
        // Mask tokens past the chunk end or on a bad page; online softmax per q row.
        float sv[2][4];  // [row half][token slot]: slots = s0 cols, s1 cols
        {
            const int tbase = it * kTileTok + r0 + 2 * (lane & 3);
            const int toks4[4] = {tbase, tbase + 1, tbase + 8, tbase + 9};
            bool valid[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) valid[u] = toks4[u] < ntok && rowoff[toks4[u]] >= 0;
            sv[0][0] = valid[0] ? s0[0] : -INFINITY;
            sv[0][1] = valid[1] ? s0[1] : -INFINITY;
            sv[0][2] = valid[2] ? s1[0] : -INFINITY;
            sv[0][3] = valid[3] ? s1[1] : -INFINITY;
            sv[1][0] = valid[0] ? s0[2] : -INFINITY;
            sv[1][1] = valid[1] ? s0[3] : -INFINITY;
            sv[1][2] = valid[2] ? s1[2] : -INFINITY;
            sv[1][3] = valid[3] ? s1[3] : -INFINITY;
        }
        float pr[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float mx = fmaxf(fmaxf(sv[h][0], sv[h][1]), fmaxf(sv[h][2], sv[h][3]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_r[h], mx * p.scale_log2);
            // O and l are still 0 while m_r is -inf, so any finite factor works there.
            const float factor = m_r[h] == -INFINITY ? 0.f : ex2(m_r[h] - m_new);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            m_r[h] = m_new;
            float sum = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                pr[h][u] = ex2(fmaf(sv[h][u], p.scale_log2, -m_use));
                sum += pr[h][u];
            }
            l_r[h] = l_r[h] * factor + sum;
            if (factor != 1.f) {
#pragma unroll
                for (int nt = 0; nt < D / 8; ++nt) {
                    o[nt][2 * h] *= factor;
                    o[nt][2 * h + 1] *= factor;
                }
            }
        }
        // O += P V for this warp's 16 tokens.
        uint32_t ap[4];
        ap[0] = pack_bf16x2(pr[0][0], pr[0][1]);
        ap[1] = pack_bf16x2(pr[1][0], pr[1][1]);
        ap[2] = pack_bf16x2(pr[0][2], pr[0][3]);
        ap[3] = pack_bf16x2(pr[1][2], pr[1][3]);
        {
            const int mi = lane >> 3;
            const int rr = r0 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
            for (int c2 = 0; c2 < D / 16; ++c2) {
                uint32_t v0, v1, v2, v3;
                ldmatrix_x4_trans(vt + swz<D>(rr, c2 * 2 + (mi >> 1)), v0, v1, v2, v3);
                mma_bf16_16816(o[2 * c2], ap, v0, v1);
                mma_bf16_16816(o[2 * c2 + 1], ap, v2, v3);
            }
        }
    }
    cp_async_wait<0>();

    // Merge the four warps' states.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float l = l_r[h];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        l_r[h] = l;
        if ((lane & 3) == 0) {
            st_m[warp * 16 + (lane >> 2) + 8 * h] = m_r[h];
            st_l[warp * 16 + (lane >> 2) + 8 * h] = l;
        }
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = (lane >> 2) + 8 * h;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, st_m[w * 16 + row]);
        const float f = M == -INFINITY ? 0.f : ex2(m_r[h] - M);
        if (row < p.G) {
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                const int col = nt * 8 + 2 * (lane & 3);
                atomicAdd(&red[row * D + col], o[nt][2 * h] * f);
                atomicAdd(&red[row * D + col + 1], o[nt][2 * h + 1] * f);
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.G * D; e += kDecThreads) {
        const int row = e / D, c = e % D;
        float M = -INFINITY, L = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, st_m[w * 16 + row]);
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float mw = st_m[w * 16 + row];
                if (mw != -INFINITY) L += st_l[w * 16 + row] * ex2(mw - M);
            }
        }
        const int h = hk * p.G + row;
        const int64_t slot = ((int64_t)b * p.Hq + h) * p.S + split;
        p.po[slot * D + c] = L > 0.f ? red[e] / L : 0.f;
        if (c == 0) p.plse[slot] = L > 0.f ? (M + log2f(L)) * kLn2d : -INFINITY;
    }
}

template <int D>
__global__ void decode_combine_kernel(const DecCombineParams p)
{
    const int row = blockIdx.x;  // b * Hq + h
    const float *ls = p.plse + (int64_t)row * p.S;
    float M = -INFINITY;
    for (int s = 0; s < p.S; ++s) M = fmaxf(M, ls[s]);
    float Z = 0.f;
    if (M != -INFINITY)
        for (int s = 0; s < p.S; ++s) Z += __expf(ls[s] - M);
    const float lse = M == -INFINITY ? -INFINITY : M + __logf(Z);
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        float acc = 0.f;
        if (M != -INFINITY)
            for (int s = 0; s < p.S; ++s) {
                const float w = ls[s] == -INFINITY ? 0.f : __expf(ls[s] - lse);
                acc += w * p.po[((int64_t)row * p.S + s) * D + c];
            }
        p.out[(int64_t)row * D + c] = __float2bfloat16_rn(acc);
    }
    if (threadIdx.x == 0) p.lse[row] = lse;
}

template <int D>
size_t dec_smem_bytes(int S, int topk)
{
    const int chunk = (topk + S - 1) / S;
    return DecCfg<D>::kOffRows + (size_t)chunk * 4;
}

template <int D>
cudaError_t launch_split_t(const DecGeom &g, const DecSplitParams &p, cudaStream_t st)
{
    const size_t smem = dec_smem_bytes<D>(g.S, g.topk);
    static int configured = 0;
    if ((int)smem > configured) {
        cudaError_t e =
            cudaFuncSetAttribute(decode_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = (int)smem;
    }
    dim3 grid(g.S, g.Hkv, g.B);
    decode_split_kernel<D><<<grid, kDecThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

int decode_split_blocks_per_sm(int d)
{
    // Shared memory decides: three 64-token stages of K and V rows per CTA.
    const size_t per = d == 64 ? dec_smem_bytes<64>(8, 2048) : dec_smem_bytes<128>(8, 2048);
    const size_t sm = 228 * 1024;
    int n = (int)(sm / (per + 1024));
    return n < 1 ? 1 : n;
}

cudaError_t launch_decode_split(const DecGeom &g, const DecSplitParams &p, cudaStream_t st)
{
    return g.d == 64 ? launch_split_t<64>(g, p, st) : launch_split_t<128>(g, p, st);
}

cudaError_t launch_decode_combine(const DecGeom &g, const DecCombineParams &p, cudaStream_t st)
{
    if (g.d == 64) decode_combine_kernel<64><<<g.B * g.Hq, 64, 0, st>>>(p);
    else decode_combine_kernel<128><<<g.B * g.Hq, 128, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sfa
