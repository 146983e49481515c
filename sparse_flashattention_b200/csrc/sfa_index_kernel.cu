// Index producer for the paged top-k decode: a Lightning-Indexer-style scan ("Sparse FlashAttention" on
// Ascend, ggplus blog post, section "那个叫Lightning Indexer的家伙": the current query is scored against
// every key with FP8-quantized dot products and the top-k token positions crop K and V for the sparse
// attention; one O(L) pass over the keys).
//
// One CTA of 1024 threads per (sequence, kv head):
//   1. the group's G query rows rounded to FP8 E4M3 and summed per dimension (exact in fp32);
//   2. every cache position's key row (through the block table) rounded to E4M3 and dotted with that
//      sum in fp64, D/8 lanes per row, 8 elements each.  Every product and partial sum is exact (the
//      format's values have 4 significant bits and span 2^-9 .. 448), so the score does not depend on
//      the summation order and equals the definition bit for bit.  The score becomes an
//      order-preserving 64-bit key in the workspace, and its top 12 bits go into a histogram;
//   3. the k-th largest key T by radix refinement: per 12-bit digit (12, 12, 12, 12, 12, 4 bits) the
//      boundary digit from the suffix counts, then a histogram of the next digit over the keys that
//      share the prefix;
//   4. one ordered pass: each thread takes a contiguous range of positions, a block scan places its
//      picks (keys above T, then the first keys equal to T in position order), so the list comes out
//      ascending; the forced most recent positions follow, then -1 padding.
// No waits: the kernel has no pipeline, only block barriers.
#include <cuda_fp16.h>

#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kIdxThreads = 1024;
constexpr int kIdxBins = 4096;  // 12-bit digits
constexpr int kIdxBtMax = 4096; // block-table entries of a sequence kept in shared memory

// x rounded to FP8 E4M3 (round to nearest even, saturated at +-448) and back to float.  Both halves of
// the pair carry x, so the result does not depend on which half a conversion fills.
__device__ __forceinline__ float e4m3_round_trip(float x)
{
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(h) : "f"(x));
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
    return __half2float(__ushort_as_half((unsigned short)(r & 0xffffu)));
}

// Two values at once: (lo, hi) rounded to E4M3 as above, returned as floats (one conversion each way
// for the pair; the E4M3 values are exact in f16 and in f32).
__device__ __forceinline__ float2 e4m3_round_trip2(float lo, float hi)
{
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
    return __half22float2(*reinterpret_cast<const __half2 *>(&r));
}

// Order-preserving key of a finite score (larger score, larger key); -0 and +0 tie.  Keys of finite
// values are never 0, which marks "no candidate".
__device__ __forceinline__ unsigned long long order_key(double s)
{
    if (s == 0.0) s = 0.0;
    const unsigned long long b = (unsigned long long)__double_as_longlong(s);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Inclusive prefix sum of one value per thread over the 1024 threads; *total gets the block sum.
__device__ int block_incl_scan(int v, int *scratch, int *total)
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
    const int r = (warp > 0 ? scratch[warp - 1] : 0) + x;
    *total = scratch[31];
    __syncthreads();
    return r;
}

template <int D>
__global__ void __launch_bounds__(kIdxThreads, 1) index_topk_kernel(IndexParams p)
{
    __shared__ double qs[D];
    __shared__ unsigned int hist[kIdxBins];
    __shared__ int bt_s[kIdxBtMax];
    __shared__ int scratch[32];
    __shared__ int s_digit, s_above;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x / p.Hkv, hk = blockIdx.x % p.Hkv;
    int64_t L = p.seqlens[b];
    if (L < 0) L = 0;
    if (L > p.max_len) {  // longer than the block table holds
        if (tid == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
        L = p.max_len;
    }
    const int64_t nl = min((int64_t)min(p.n_local, p.topk), L);
    const int64_t Lc = L - nl;  // positions that compete on score
    unsigned long long *keys = p.keys + (int64_t)blockIdx.x * p.max_len;
    int32_t *out = p.sel + (int64_t)blockIdx.x * p.topk;

    // 1. the group's summed E4M3 query (exact in fp64), and the sequence's block-table row when it
    // fits in shared memory
    for (int c = tid; c < D; c += kIdxThreads) {
        double a = 0.0;
        for (int g = 0; g < p.G; ++g)
            a += (double)e4m3_round_trip(__bfloat162float(p.q[((int64_t)b * p.Hq + hk * p.G + g) * D + c]));
        qs[c] = a;
    }
    const int32_t *bt_g = p.bt + (int64_t)b * p.max_pages;
    const bool bt_smem = p.max_pages <= kIdxBtMax;
    if (bt_smem)
        for (int i = tid; i < p.max_pages; i += kIdxThreads) bt_s[i] = __ldg(&bt_g[i]);
    for (int i = tid; i < kIdxBins; i += kIdxThreads) hist[i] = 0u;
    __syncthreads();

    // 2. scores -> keys, and the histogram of their top digit.  A lane group of D/8 lanes scores a row;
    // each group takes kRowsPerGroup rows at a time, their loads issued before any arithmetic.
    // score = sum over the row of e4m3(k) * qsum in fp64: every product and partial sum is exact (see
    // above), so the order of the sum does not matter.
    constexpr int kLanesPerRow = D / 8;
    constexpr int kRowsPerWarp = 32 / kLanesPerRow;
    constexpr int kRowsPerGroup = 4;
    constexpr int64_t kStep = (int64_t)(kIdxThreads / 32) * kRowsPerWarp * kRowsPerGroup;
    const int sub = lane / kLanesPerRow, part = lane % kLanesPerRow;
    double qv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] = qs[part * 8 + e];
    bool bad_page = false;
    for (int64_t j0 = (int64_t)warp * kRowsPerWarp * kRowsPerGroup; j0 < L; j0 += kStep) {
        uint4 raw[kRowsPerGroup];
        bool okp[kRowsPerGroup];
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) {
            const int64_t j = j0 + u * kRowsPerWarp + sub;
            const bool in = j < L;
            const int pi = in ? (int)(j / p.page) : 0;
            const int pg = in ? (bt_smem ? bt_s[pi] : __ldg(&bt_g[pi])) : -1;
            okp[u] = in && pg >= 0 && pg < p.num_pages;
            raw[u] = okp[u] ? __ldg(reinterpret_cast<const uint4 *>(
                                  p.kc + (((int64_t)pg * p.page + (j - (int64_t)pi * p.page)) * p.Hkv + hk) * D + part * 8))
                            : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) {
            const int64_t j = j0 + u * kRowsPerWarp + sub;
            const __nv_bfloat162 *v = reinterpret_cast<const __nv_bfloat162 *>(&raw[u]);
            double acc = 0.0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(v[e]);
                const float2 k8 = e4m3_round_trip2(x.x, x.y);
                acc = fma((double)k8.x, qv[2 * e], acc);
                acc = fma((double)k8.y, qv[2 * e + 1], acc);
            }
#pragma unroll
            for (int o = kLanesPerRow / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (part == 0 && j < L) {
                const unsigned long long key = (okp[u] && j < Lc) ? order_key(acc) : 0ull;
                keys[j] = key;
                if (key) atomicAdd(&hist[key >> 52], 1u);
                bad_page |= !okp[u];
            }
        }
    }
    if (__syncthreads_or(bad_page) && tid == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_PAGE);

    // 3. the k-th largest key T; `remaining` = how many keys equal to T the result takes
    int cand = 0;
    for (int i = tid * 4; i < tid * 4 + 4; ++i) cand += (int)hist[i];
    int total;
    block_incl_scan(cand, scratch, &total);
    int remaining = (int)min((int64_t)(p.topk - nl), (int64_t)total);
    const int need = remaining;
    unsigned long long prefix = 0ull, pmask = 0ull;
    int shift = 52, width = 12;
    while (remaining > 0) {
        // boundary digit: the largest t with (count of digits >= t) >= remaining
        int mine = 0;
        for (int i = tid * 4; i < tid * 4 + 4; ++i) mine += (int)hist[i];
        int tot;
        const int incl = block_incl_scan(mine, scratch, &tot);
        int run = tot - incl;  // digits owned by higher threads
        for (int i = tid * 4 + 3; i >= tid * 4; --i) {
            const int c = (int)hist[i];
            if (c > 0 && run < remaining && run + c >= remaining) {
                s_digit = i;
                s_above = run;
            }
            run += c;
        }
        __syncthreads();
        remaining -= s_above;
        prefix |= (unsigned long long)s_digit << shift;
        pmask |= (unsigned long long)((1 << width) - 1) << shift;
        if (shift == 0) break;
        width = shift >= 12 ? 12 : shift;
        shift -= width;
        __syncthreads();
        for (int i = tid; i < kIdxBins; i += kIdxThreads) hist[i] = 0u;
        __syncthreads();
        for (int64_t j = tid; j < Lc; j += kIdxThreads) {
            const unsigned long long key = keys[j];
            if (key != 0ull && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & ((1u << width) - 1u)], 1u);
        }
        __syncthreads();
    }
    const unsigned long long T = prefix;

    // 4. ordered picks: keys above T, and the first `remaining` keys equal to T by position
    const int64_t per = (Lc + kIdxThreads - 1) / kIdxThreads;
    const int64_t j_begin = min(Lc, (int64_t)tid * per), j_end = min(Lc, j_begin + per);
    int gt = 0, eq = 0;
    if (need > 0)
        for (int64_t j = j_begin; j < j_end; ++j) {
            const unsigned long long key = keys[j];
            gt += key > T;
            eq += key == T;
        }
    int eq_tot;
    const int eq_before = block_incl_scan(eq, scratch, &eq_tot) - eq;
    const int eq_take = max(0, min(eq, remaining - eq_before));
    int cnt_tot;
    const int out_before = block_incl_scan(gt + eq_take, scratch, &cnt_tot) - (gt + eq_take);
    if (need > 0) {
        int w = out_before, taken = 0;
        for (int64_t j = j_begin; j < j_end; ++j) {
            const unsigned long long key = keys[j];
            if (key > T || (key == T && taken < eq_take)) {
                if (key == T) ++taken;
                if (w < p.topk) out[w] = (int32_t)j;
                ++w;
            }
        }
    }
    __syncthreads();
    if (tid == 0) {  // the forced most recent positions (valid pages only), then padding
        int w = cnt_tot;
        for (int64_t j = Lc; j < L && w < p.topk; ++j) {
            const int pg = __ldg(&p.bt[(int64_t)b * p.max_pages + j / p.page]);
            if (pg >= 0 && pg < p.num_pages) out[w++] = (int32_t)j;
        }
        for (; w < p.topk; ++w) out[w] = -1;
    }
}

}  // namespace

cudaError_t launch_index_topk(const IndexParams &p, cudaStream_t st)
{
    const unsigned grid = (unsigned)(p.B * p.Hkv);
    if (grid == 0) return cudaSuccess;
    if (p.d == 64) index_topk_kernel<64><<<grid, kIdxThreads, 0, st>>>(p);
    else index_topk_kernel<128><<<grid, kIdxThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sfa
