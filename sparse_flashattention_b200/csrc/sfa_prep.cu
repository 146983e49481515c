// Index preparation: turn the caller's top-k selections into canonical sets.
//
// Prefill (one CTA per query tile): for every (token, kv head) of the tile keep the block ids
// that are -1-free, inside the sequence, and hold at least one key the mask keeps; sort them
// ascending without duplicates (a selection is a set); count them; and OR them into a bitmap
// whose ascending scan is the tile's union of blocks — the list the attention kernel walks.
// INVALID = -1 marks an unused slot (Ascend SFA article, ConstInfo listing); the mask is the
// bottom-right aligned causal mask plus window of the flash-attention-npu docstrings.
//
// Decode (one CTA per (sequence, kv head)): a bitmap over the positions [0, L) turns the
// selected token positions into an ascending duplicate-free list in O(L/32) work.
#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kPrepThreads = 128;

// Exclusive scan of one int per thread over a 128- or 256-thread block; returns the total.
template <int NT>
__device__ int block_exclusive_scan(int v, int *scratch, int &excl)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NT / 32 ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NT / 32) scratch[lane] = w;  // inclusive per-warp totals
    }
    __syncthreads();
    const int before = warp > 0 ? scratch[warp - 1] : 0;
    excl = before + x - v;
    const int total = scratch[NT / 32 - 1];
    __syncthreads();
    return total;
}

// Bitmap words [0, words) -> ascending ids written to dst; returns the count.  All threads.
template <int NT>
__device__ int compact_bitmap(const uint32_t *bm, int words, int32_t *dst, int *scratch)
{
    const int per = (words + NT - 1) / NT;
    const int w0 = min(words, (int)threadIdx.x * per), w1 = min(words, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(bm[w]);
    int pos;
    const int total = block_exclusive_scan<NT>(c, scratch, pos);
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = bm[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            dst[pos++] = w * 32 + b;
        }
    }
    return total;
}

__global__ void __launch_bounds__(kPrepThreads) fwd_prep_kernel(FwdPrepParams p)
{
    extern __shared__ uint32_t prep_smem[];
    __shared__ int scan_scratch[32];
    const int tile = blockIdx.x;
    const int hk = tile % p.Hkv;
    const int rest = tile / p.Hkv;
    const int b = rest % p.batch;
    const int qt = p.nqt - 1 - rest / p.batch;

    const int q0 = p.cu_q[b], sq = p.cu_q[b + 1] - q0;
    const int k0 = p.cu_k[b], sk = p.cu_k[b + 1] - k0;
    const int tok0 = qt * p.Tq;
    const int ntok = min(p.Tq, sq - tok0);
    if (ntok <= 0) {
        if (threadIdx.x == 0) p.ucnt[tile] = 0;
        return;
    }
    (void)k0;
    int nblk = (sk + p.bs - 1) / p.bs;
    if (sq > p.max_sq || nblk > p.nblk_max) {  // lengths beyond the caller's max_seqlen bounds
        if (threadIdx.x == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
        nblk = min(nblk, p.nblk_max);
    }
    const int words = (nblk + 31) / 32;
    uint32_t *bm = prep_smem;
    int *lists = reinterpret_cast<int *>(prep_smem + words);  // [topk][kPrepThreads]
    for (int w = threadIdx.x; w < words; w += kPrepThreads) bm[w] = 0;
    __syncthreads();

    const int tt = threadIdx.x;
    if (tt < ntok) {
        const int i = tok0 + tt;  // local query index
        const int64_t t = (int64_t)q0 + i;
        const int delta = sk - sq;
        int lo = 0, hi = sk - 1;
        if (p.wl >= 0) lo = max(lo, i + delta - p.wl);
        if (p.causal) hi = min(hi, i + delta);
        if (p.wr >= 0) hi = min(hi, i + delta + p.wr);
        const int32_t *row = p.sel + (t * p.Hkv + hk) * p.topk;
        int n = 0;
        bool bad = false;
        for (int e = 0; e < p.topk; ++e) {
            const int s = row[e];
            if (s == -1) continue;
            if (s < 0 || s >= nblk) {
                bad = true;
                continue;
            }
            const int bl = s * p.bs, bh = min(bl + p.bs, sk) - 1;
            if (max(bl, lo) > min(bh, hi)) continue;  // no key of this block survives the mask
            // Insert into the ascending list, skipping duplicates.
            int pos = n;
            while (pos > 0 && lists[(pos - 1) * kPrepThreads + tt] > s) --pos;
            if (pos > 0 && lists[(pos - 1) * kPrepThreads + tt] == s) continue;
            for (int m = n; m > pos; --m) lists[m * kPrepThreads + tt] = lists[(m - 1) * kPrepThreads + tt];
            lists[pos * kPrepThreads + tt] = s;
            ++n;
        }
        int32_t *dst = p.sel_c + (t * p.Hkv + hk) * p.topk;
        for (int e = 0; e < p.topk; ++e) {
            const int s = e < n ? lists[e * kPrepThreads + tt] : -1;
            dst[e] = s;
            if (e < n) atomicOr(&bm[s >> 5], 1u << (s & 31));
        }
        p.cnt[t * p.Hkv + hk] = n;
        if (bad && p.status) atomicOr(p.status, SFA_DEV_BAD_INDEX);
    }
    __syncthreads();
    const int total = compact_bitmap<kPrepThreads>(bm, words, p.uni + (int64_t)tile * p.umax, scan_scratch);
    if (threadIdx.x == 0) p.ucnt[tile] = total;
}

constexpr int kDecPrepThreads = 512;

__global__ void __launch_bounds__(kDecPrepThreads) decode_prep_kernel(DecPrepParams p)
{
    extern __shared__ uint32_t dprep_smem[];
    __shared__ int scan_scratch[32];
    const int b = blockIdx.x / p.Hkv, hk = blockIdx.x % p.Hkv;
    int L = p.seqlens[b];
    bool bad_len = false;
    if (L > p.max_len) {  // more tokens than the block table can address
        L = p.max_len;
        bad_len = true;
    }
    if (L < 0) L = 0;
    const int words = (L + 31) / 32;
    for (int w = threadIdx.x; w < words; w += kDecPrepThreads) dprep_smem[w] = 0;
    __syncthreads();
    const int32_t *row = p.sel + ((int64_t)b * p.Hkv + hk) * p.topk;
    bool bad = false;
    for (int e = threadIdx.x; e < p.topk; e += kDecPrepThreads) {
        const int j = row[e];
        if (j == -1) continue;
        if (j < 0 || j >= L) {
            bad = true;
            continue;
        }
        if (p.wl >= 0 && j < L - 1 - p.wl) continue;  // left of the window
        atomicOr(&dprep_smem[j >> 5], 1u << (j & 31));
    }
    if (bad && p.status) atomicOr(p.status, SFA_DEV_BAD_INDEX);
    if (bad_len && threadIdx.x == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
    __syncthreads();
    int32_t *dst = p.tok_c + ((int64_t)b * p.Hkv + hk) * p.topk;
    const int n = compact_bitmap<kDecPrepThreads>(dprep_smem, words, dst, scan_scratch);
    for (int e = n + threadIdx.x; e < p.topk; e += kDecPrepThreads) dst[e] = -1;
    if (threadIdx.x == 0) p.cnt[b * p.Hkv + hk] = n;
}

}  // namespace

cudaError_t launch_fwd_prep(const FwdGeom &g, const FwdPrepParams &p, cudaStream_t st)
{
    const size_t words = (size_t)(g.nblk_max + 31) / 32;
    const size_t smem = words * 4 + (size_t)g.topk * kPrepThreads * 4;
    static int configured_bytes = 0;
    if ((int)smem > 48 * 1024 && (int)smem > configured_bytes) {
        cudaError_t e = cudaFuncSetAttribute(fwd_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured_bytes = (int)smem;
    }
    fwd_prep_kernel<<<g.tiles, kPrepThreads, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_decode_prep(const DecGeom &g, const DecPrepParams &p, cudaStream_t st)
{
    const size_t smem = (size_t)((p.max_len + 31) / 32) * 4;
    static int configured_bytes = 0;
    if ((int)smem > 48 * 1024 && (int)smem > configured_bytes) {
        cudaError_t e =
            cudaFuncSetAttribute(decode_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured_bytes = (int)smem;
    }
    decode_prep_kernel<<<g.B * g.Hkv, kDecPrepThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sfa
