// Index producer for the paged top-k decode: a Lightning-Indexer-style scan ("Sparse FlashAttention" on
// Ascend, ggplus blog post, section "那个叫Lightning Indexer的家伙": the current query is scored against
// every key with FP8-quantized dot products and the top-k token positions crop K and V for the sparse
// attention; one O(L) pass over the keys).
//
// Two kernels.  Scoring, one CTA of 256 threads per (sequence, kv head, run of kIdxChunk positions), so
// every SM streams keys whatever the number of sequences, each thread keeping several iterations of
// its key rows in flight through a cp.async ring in shared memory:
//   1. the group's G query rows rounded to FP8 E4M3 and summed per dimension in fp64;
//   2. every cache position's key row (through the block table) rounded to E4M3 and dotted with that
//      sum in fp64, D/8 lanes per row, 8 elements each.  The format's values are multiples of 2^-9
//      below 2^9, so a product is a multiple of 2^-18 below G 2^18 and a row's sum, below G 2^25,
//      needs at most 43 + log2(G) <= 53 bits for G <= 1024: every product and partial sum is exact,
//      the score does not depend on the summation order and equals the definition bit for bit.  The
//      key values enter scaled by 2^-1016 (the decode below); the scaled products, multiples of
//      2^-1034, still sit on the fp64 grid (subnormal spacing 2^-1074), so they too are exact, and a
//      power-of-two scale keeps the order and the ties of the scores.  The scaled score becomes an
//      order-preserving 64-bit key in the workspace.
// Selection, one CTA of 1024 threads per (sequence, kv head):
//   3. the k-th largest key T by radix refinement: per 12-bit digit (12, 12, 12, 12, 12, 4 bits) a
//      histogram of the digit over the keys that share the prefix so far, then the boundary digit from
//      the suffix counts (every pass over the keys keeps four loads per thread in flight);
//   4. one ordered pass: each thread takes a contiguous range of positions, a block scan places its
//      picks (keys above T, then the first keys equal to T in position order), so the list comes out
//      ascending; the forced most recent positions follow, then -1 padding.
// No spin-waits: block barriers, and a thread waiting on the hardware for its own cp.async groups.
#include <cuda_fp16.h>

#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kIdxThreads = 1024;     // selection CTA
constexpr int kIdxScoreThreads = 256; // scoring CTA
constexpr int kIdxChunk = 4096;       // positions a scoring CTA takes
constexpr int kIdxBins = 4096;        // 12-bit digits
constexpr int kRowsPerGroup = 4;      // key rows a scoring lane group takes per iteration
constexpr int kIdxStages = 4;         // depth of a scoring thread's copy ring
constexpr size_t kIdxScoreSmem = sizeof(uint4) * kIdxStages * kRowsPerGroup * kIdxScoreThreads;  // 64 KB

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

// Two values at once: (lo, hi) rounded to E4M3 as above (one conversion for the pair), each returned
// as its value times 2^-1016 in fp64 with no further conversion.  The code's exponent field E and
// mantissa field M placed in the low bits of the fp64 exponent and the top of its fraction read as
// (1 + M/8) 2^(E-1023) for E >= 1 and as the fp64 subnormal (M/8) 2^-1022 for E = 0: the E4M3 values
// (1 + M/8) 2^(E-7) and (M/8) 2^-6, both times 2^-1016, exactly.  (The NaN code, which satfinite
// makes only from a NaN, reads as 480.)
__device__ __forceinline__ void e4m3_round_trip2_scaled(float lo, float hi, double &dlo, double &dhi)
{
    uint16_t h16;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h16) : "f"(hi), "f"(lo));
    const uint32_t h = h16;
    dlo = __hiloint2double((int)(((h & 0x7fu) << 17) | ((h & 0x80u) << 24)), 0);
    dhi = __hiloint2double((int)(((h & 0x7f00u) << 9) | ((h & 0x8000u) << 16)), 0);
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

// The sequence's length after the checks both kernels make (clamped to the block table; the scoring
// kernel's first CTA of the sequence reports a longer one).
__device__ __forceinline__ int64_t index_len(const IndexParams &p, int b)
{
    int64_t L = p.seqlens[b];
    if (L < 0) L = 0;
    return L > p.max_len ? p.max_len : L;
}

template <int D>
__global__ void __launch_bounds__(kIdxScoreThreads, 3) index_score_kernel(IndexParams p)
{
    extern __shared__ __align__(16) uint4 stage[];  // [kIdxStages][kRowsPerGroup][kIdxScoreThreads]
    __shared__ double qs[D];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nchunk = (int)((p.max_len + kIdxChunk - 1) / kIdxChunk);
    const int unit = blockIdx.x / nchunk, chunk = blockIdx.x - unit * nchunk;
    const int b = unit / p.Hkv, hk = unit % p.Hkv;
    if (chunk == 0 && tid == 0 && p.status && p.seqlens[b] > p.max_len) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
    const int64_t L = index_len(p, b);
    const int64_t c0 = (int64_t)chunk * kIdxChunk;
    if (c0 >= L) return;
    const int64_t c1 = min(L, c0 + kIdxChunk);
    const int64_t nl = min((int64_t)min(p.n_local, p.topk), L);
    const int64_t Lc = L - nl;  // positions that compete on score
    unsigned long long *keys = p.keys + (int64_t)unit * p.max_len;

    // the group's summed E4M3 query (exact in fp64)
    for (int c = tid; c < D; c += kIdxScoreThreads) {
        double a = 0.0;
        for (int g = 0; g < p.G; ++g)
            a += (double)e4m3_round_trip(__bfloat162float(p.q[((int64_t)b * p.Hq + hk * p.G + g) * D + c]));
        qs[c] = a;
    }
    __syncthreads();

    // scores -> keys.  A lane group of D/8 lanes scores a row, 16 bytes a lane; each group takes
    // kRowsPerGroup rows per iteration.  Every thread runs its own copy pipeline: the iteration's rows
    // go to the thread's slots of a kIdxStages-deep ring in shared memory by cp.async, issued
    // kIdxStages - 1 iterations ahead, so about three iterations of key bytes are in flight per thread
    // while it scores the oldest (a thread reads only the slots it filled: no block barrier).
    // score * 2^-1016 = sum over the row of (e4m3(k) * 2^-1016) * qsum in fp64, exact in any order
    // (step 2 above).
    constexpr int kLanesPerRow = D / 8;
    constexpr int kRowsPerWarp = 32 / kLanesPerRow;
    constexpr int64_t kStep = (int64_t)(kIdxScoreThreads / 32) * kRowsPerWarp * kRowsPerGroup;
    static_assert(kIdxStages * kRowsPerGroup <= 32, "row-valid bits of the ring in one word");
    const int sub = lane / kLanesPerRow, part = lane % kLanesPerRow;
    double qv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[e] = qs[part * 8 + e];
    const int32_t *bt_g = p.bt + (int64_t)b * p.max_pages;
    const int64_t j_first = c0 + (int64_t)warp * kRowsPerWarp * kRowsPerGroup;
    const int n_it = j_first < c1 ? (int)((c1 - j_first + kStep - 1) / kStep) : 0;
    bool bad_page = false;
    uint32_t okm = 0;  // bit slot * kRowsPerGroup + u: row u of the iteration held in that slot is readable

    // A warp's rows of one iteration are the kGroupRows consecutive positions from a multiple of
    // kGroupRows; when the page size is a multiple of that, they sit in one page: one block-table
    // lookup serves them all and the rows are constant offsets from the first.
    constexpr int kGroupRows = kRowsPerWarp * kRowsPerGroup;
    const bool one_page = p.page % kGroupRows == 0;
    const int64_t row_elems = (int64_t)p.Hkv * D;  // elements from one cache row to the next
    auto issue = [&](int it) {
        const int slot = it % kIdxStages;
        const int64_t j0 = j_first + (int64_t)it * kStep;
        uint32_t m = 0;
        if (one_page) {
            // j0 < c1 <= 2^20: 32-bit division (a 64-bit one is a long software routine)
            const unsigned pi = (unsigned)j0 / (unsigned)p.page;
            const int pg = __ldg(&bt_g[pi]);
            const bool okg = pg >= 0 && pg < p.num_pages;
            const __nv_bfloat16 *base =
                p.kc + ((int64_t)pg * p.page + ((int)j0 - (int)pi * p.page)) * row_elems + hk * D + part * 8;
#pragma unroll
            for (int u = 0; u < kRowsPerGroup; ++u) {
                const int du = u * kRowsPerWarp + sub;
                const bool in = j0 + du < c1;
                const bool ok = in && okg;
                cp_async16(smem_u32(&stage[(slot * kRowsPerGroup + u) * kIdxScoreThreads + tid]),
                           ok ? base + du * row_elems : p.kc, ok ? 16u : 0u);
                m |= (uint32_t)ok << u;
                bad_page |= in && !ok;
            }
        } else {
#pragma unroll
            for (int u = 0; u < kRowsPerGroup; ++u) {
                const int64_t j = j0 + u * kRowsPerWarp + sub;
                const bool in = j < c1;
                const unsigned pi = in ? (unsigned)j / (unsigned)p.page : 0u;
                const int pg = in ? __ldg(&bt_g[pi]) : -1;
                const bool ok = in && pg >= 0 && pg < p.num_pages;
                const int row = (int)j - (int)pi * p.page;
                const __nv_bfloat16 *src = ok ? p.kc + ((int64_t)pg * p.page + row) * row_elems + hk * D + part * 8 : p.kc;
                cp_async16(smem_u32(&stage[(slot * kRowsPerGroup + u) * kIdxScoreThreads + tid]), src, ok ? 16u : 0u);
                m |= (uint32_t)ok << u;
                bad_page |= in && !ok;
            }
        }
        const int sh = slot * kRowsPerGroup;
        okm = (okm & ~(((1u << kRowsPerGroup) - 1u) << sh)) | (m << sh);
    };

#pragma unroll
    for (int s = 0; s < kIdxStages - 1; ++s) {
        if (s < n_it) issue(s);
        cp_async_commit();
    }
    for (int it = 0; it < n_it; ++it) {
        cp_async_wait<kIdxStages - 2>();  // this iteration's group has landed
        const int slot = it % kIdxStages;
        uint4 raw[kRowsPerGroup];
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) raw[u] = stage[(slot * kRowsPerGroup + u) * kIdxScoreThreads + tid];
        const uint32_t m = okm >> (slot * kRowsPerGroup);
        if (it + kIdxStages - 1 < n_it) issue(it + kIdxStages - 1);  // refills the slot read last iteration
        cp_async_commit();
        const int64_t j0 = j_first + (int64_t)it * kStep;
#pragma unroll
        for (int u = 0; u < kRowsPerGroup; ++u) {
            const int64_t j = j0 + u * kRowsPerWarp + sub;
            const __nv_bfloat162 *v = reinterpret_cast<const __nv_bfloat162 *>(&raw[u]);
            double acc = 0.0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(v[e]);
                double k0, k1;
                e4m3_round_trip2_scaled(x.x, x.y, k0, k1);
                acc = fma(k0, qv[2 * e], acc);
                acc = fma(k1, qv[2 * e + 1], acc);
            }
#pragma unroll
            for (int o = kLanesPerRow / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (part == 0 && j < c1) keys[j] = (((m >> u) & 1u) && j < Lc) ? order_key(acc) : 0ull;
        }
    }
    if (__syncthreads_or(bad_page) && tid == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_PAGE);
}

template <int D>
__global__ void __launch_bounds__(kIdxThreads, 1) index_select_kernel(IndexParams p)
{
    __shared__ unsigned int hist[kIdxBins];
    __shared__ int scratch[32];
    __shared__ int s_digit, s_above;
    const int tid = threadIdx.x;
    const int b = blockIdx.x / p.Hkv;
    const int64_t L = index_len(p, b);
    const int64_t nl = min((int64_t)min(p.n_local, p.topk), L);
    const int64_t Lc = L - nl;
    const unsigned long long *keys = p.keys + (int64_t)blockIdx.x * p.max_len;
    int32_t *out = p.sel + (int64_t)blockIdx.x * p.topk;

    // histogram of a digit over the keys with the prefix so far (four keys per thread in flight)
    auto digit_hist = [&](unsigned long long prefix, unsigned long long pmask, int shift, int width) {
        for (int i = tid; i < kIdxBins; i += kIdxThreads) hist[i] = 0u;
        __syncthreads();
        for (int64_t j0 = tid; j0 < Lc; j0 += 4 * kIdxThreads) {
            unsigned long long kk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) kk[u] = j0 + u * kIdxThreads < Lc ? keys[j0 + u * kIdxThreads] : 0ull;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (kk[u] != 0ull && (kk[u] & pmask) == prefix)
                    atomicAdd(&hist[(kk[u] >> shift) & ((1u << width) - 1u)], 1u);
        }
        __syncthreads();
    };

    // 3. the k-th largest key T; `remaining` = how many keys equal to T the result takes
    digit_hist(0ull, 0ull, 52, 12);
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
        digit_hist(prefix, pmask, shift, width);
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
    const unsigned units = (unsigned)(p.B * p.Hkv);
    if (units == 0) return cudaSuccess;
    const unsigned nchunk = (unsigned)((p.max_len + kIdxChunk - 1) / kIdxChunk);
    if (nchunk == 0) return cudaSuccess;
    if (p.d == 64) {
        const cudaError_t e = ensure_smem_for(index_score_kernel<64>, kIdxScoreSmem);
        if (e != cudaSuccess) return e;
        index_score_kernel<64><<<units * nchunk, kIdxScoreThreads, kIdxScoreSmem, st>>>(p);
        index_select_kernel<64><<<units, kIdxThreads, 0, st>>>(p);
    } else {
        const cudaError_t e = ensure_smem_for(index_score_kernel<128>, kIdxScoreSmem);
        if (e != cudaSuccess) return e;
        index_score_kernel<128><<<units * nchunk, kIdxScoreThreads, kIdxScoreSmem, st>>>(p);
        index_select_kernel<128><<<units, kIdxThreads, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace sfa
