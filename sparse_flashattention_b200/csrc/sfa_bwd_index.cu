// Prefill backward, the small kernels around the two attention kernels.
//
//   delta  D[h][t] = rowsum(dO o O) of every (token, q head) row: the term the softmax Jacobian
//          subtracts ("Sparse FlashAttention" on Ascend, FlashAttentionScoreGrad case study: dS =
//          P o (dP - rowsum(dO o O))).
//   index  inverts the canonical selections: for each (sequence, kv head, key block) row a bitmap
//          over the sequence's tokens that selected the block, and the row's token count.
//   plan   one CTA: exclusive scans of the counts give each row's offset in the token-list array;
//          rows are cut into pieces of at most kBwdPieceChunks chunks of Tq tokens; a row longer
//          than one piece gets one partial slot per piece.
//   fill   one warp per row: the bitmap, compacted, is the row's ascending token list; a block of a
//          sequence that no token selected gets dK = dV = 0 here (no other kernel touches it).
#include "sfa_device.cuh"

namespace sfa {

namespace {

__global__ void __launch_bounds__(256) bwd_delta_kernel(BwdParams p, int D)
{
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)p.total_q * p.Hq;
    const int per = D / 32;  // elements per lane: 4 (d = 128) or 2 (d = 64)
    for (int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); row < rows; row += (int64_t)gridDim.x * 8) {
        const __nv_bfloat16 *o = p.out + row * D + lane * per;
        const __nv_bfloat16 *g = p.dout + row * D + lane * per;
        float acc = 0.f;
        for (int e = 0; e < per; e += 2) {
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(o + e));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(g + e));
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            const int64_t t = row / p.Hq;
            const int h = (int)(row - t * p.Hq);
            p.delta[(int64_t)h * p.total_q + t] = acc;
        }
    }
}

__device__ __forceinline__ int owner_seq(const int32_t *cu, int batch, int64_t t)
{
    int lo = 0, hi = batch - 1;  // the b with cu[b] <= t < cu[b + 1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(&cu[mid]) <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(256) bwd_index_kernel(BwdParams p)
{
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.total_q * p.Hkv) return;
    const int64_t t = idx / p.Hkv;
    const int hk = (int)(idx - t * p.Hkv);
    const int b = owner_seq(p.cu_q, p.batch, t);
    const int i = (int)(t - __ldg(&p.cu_q[b]));
    if (i >= p.max_sq) return;  // a sequence longer than max_seqlen_q: flagged by the prep kernel
    const int n = p.cnt[idx];
    const int32_t *list = p.sel_c + idx * p.topk;
    const int64_t row0 = ((int64_t)b * p.Hkv + hk) * p.nblk_max;
    for (int e = 0; e < n; ++e) {
        const int64_t row = row0 + list[e];
        atomicOr(&p.bits[row * p.words + (i >> 5)], 1u << (i & 31));
        atomicAdd(&p.rowcnt[row], 1);
    }
}

// Exclusive scan of one value per thread over a 1024-thread block; returns the block total.
__device__ int scan1024(int v, int *scratch, int &excl)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = scratch[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        scratch[lane] = w;
    }
    __syncthreads();
    excl = (warp > 0 ? scratch[warp - 1] : 0) + x - v;
    const int total = scratch[31];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(1024) bwd_plan_kernel(BwdParams p)
{
    __shared__ int scratch[32];
    const int per_piece = kBwdPieceChunks * p.Tq;
    int64_t tok_base = 0, piece_base = 0, slot_base = 0;
    bool overflow = false;
    for (int base = 0; base < p.R; base += 1024) {
        const int r = base + threadIdx.x;
        const int c = r < p.R ? p.rowcnt[r] : 0;
        const int np = (c + per_piece - 1) / per_piece;
        const int multi = np > 1 ? np : 0;  // partial slots the row needs
        int ec, ep, es;
        const int tc = scan1024(c, scratch, ec);
        const int tp = scan1024(np, scratch, ep);
        const int ts = scan1024(multi, scratch, es);
        if (r < p.R) {
            p.rowoff[r] = (int32_t)(tok_base + ec);
            const int64_t first = piece_base + ep;
            const int slot = multi ? (int)(slot_base + es) : -1;
            if (first + np > p.max_pieces || slot + multi > p.max_slots) {
                overflow = true;  // cannot happen for lists the prep kernel wrote (the bounds are exact maxima)
            } else {
                for (int k = 0; k < np; ++k) {
                    BwdPiece pc;
                    pc.row = r;
                    pc.tok_begin = k * per_piece;
                    pc.ntok = min(per_piece, c - k * per_piece);
                    pc.idx = k;
                    pc.npieces = np;
                    pc.slot = slot;
                    pc.pad[0] = pc.pad[1] = 0;
                    p.pieces[first + k] = pc;
                }
            }
        }
        tok_base += tc;
        piece_base += tp;
        slot_base += ts;
    }
    if (__syncthreads_or(overflow)) {
        if (threadIdx.x == 0) {
            if (p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
            p.ctrl->npieces = 0;
            p.ctrl->counter = 0;
        }
        return;
    }
    if (threadIdx.x == 0) {
        p.ctrl->npieces = (int)piece_base;
        p.ctrl->counter = 0;
    }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_fill_kernel(BwdParams p, int bs)
{
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= p.R) return;
    const int c = p.rowcnt[r];
    const int s = r % p.nblk_max;
    const int bh = r / p.nblk_max;
    const int hk = bh % p.Hkv, b = bh / p.Hkv;
    if (c > 0) {
        const uint32_t *bm = p.bits + (int64_t)r * p.words;
        int32_t *dst = p.toks + p.rowoff[r];
        int total = 0;
        for (int w0 = 0; w0 < p.words && total < c; w0 += 32) {
            const int w = w0 + lane;
            uint32_t bits = w < p.words ? bm[w] : 0u;
            const int n = __popc(bits);
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int pos = total + incl - n;
            while (bits) {
                const int bit = __ffs(bits) - 1;
                bits &= bits - 1;
                dst[pos++] = w * 32 + bit;
            }
            total += __shfl_sync(0xffffffffu, incl, 31);
        }
        return;
    }
    const int k0 = __ldg(&p.cu_k[b]), sk = __ldg(&p.cu_k[b + 1]) - k0;
    const int j0 = s * bs, j1 = min(sk, j0 + bs);
    if (j0 >= j1) return;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    constexpr int kVec = D / 8;  // 16-byte pieces per key row
    for (int e = lane; e < (j1 - j0) * kVec; e += 32) {
        const int j = j0 + e / kVec, v = e % kVec;
        const int64_t off = ((int64_t)(k0 + j) * p.Hkv + hk) * D;
        reinterpret_cast<uint4 *>(p.dk + off)[v] = z;
        reinterpret_cast<uint4 *>(p.dv + off)[v] = z;
    }
}

}  // namespace

cudaError_t launch_bwd_delta(const BwdGeom &g, const BwdParams &p, cudaStream_t st)
{
    const int64_t rows = (int64_t)p.total_q * p.Hq;
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, 148 * 32);
    bwd_delta_kernel<<<(unsigned)std::max<int64_t>(blocks, 1), 256, 0, st>>>(p, g.f.d);
    return cudaGetLastError();
}

cudaError_t launch_bwd_index(const BwdGeom &g, const BwdParams &p, cudaStream_t st)
{
    const int64_t n = (int64_t)p.total_q * p.Hkv;
    bwd_index_kernel<<<(unsigned)std::max<int64_t>((n + 255) / 256, 1), 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_bwd_plan(const BwdGeom &g, const BwdParams &p, cudaStream_t st)
{
    (void)g;
    bwd_plan_kernel<<<1, 1024, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_bwd_fill(const BwdGeom &g, const BwdParams &p, cudaStream_t st)
{
    const unsigned blocks = (unsigned)std::max((p.R + 7) / 8, 1);
    if (g.f.d == 64) bwd_fill_kernel<64><<<blocks, 256, 0, st>>>(p, g.f.bs);
    else bwd_fill_kernel<128><<<blocks, 256, 0, st>>>(p, g.f.bs);
    return cudaGetLastError();
}

}  // namespace sfa
