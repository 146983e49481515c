// Paged top-k decode: split-KV attention over gathered cache rows, then an LSE combine.
//
// Split kernel: the splits of one (sequence, kv head) run six to a CTA.  For selections of up to
// 2048 positions the CTA first deduplicates its (sequence, kv head)'s selection itself: a bitmap
// over the positions [0, L) in the (not yet used) pipeline rings, scanned into an ascending list
// in shared memory — the same canonical list the prep kernel writes for longer selections.
// Then every warp is an independent worker for one split: it
// takes a contiguous chunk of the canonical (ascending) token list of its (sequence, kv head),
// looks each token's physical row up through block_table, and streams the 256-byte K and V
// rows of 16 tokens at a time through its own 2-stage cp.async ring in shared memory
// (16-byte chunks XOR-swizzled so ldmatrix reads are bank-conflict free).  The G query heads of
// the kv head are the rows of a warp-level bf16 MMA (m16n8k16, fp32 accumulate): decode is
// bound by HBM bandwidth on the gathered rows, and this keeps the arithmetic to a few
// instructions per token.  The warp keeps its own online softmax (running max rescaled only
// when it grows by more than 2^8) and writes a normalised partial output plus its natural-log
// LSE; no shared state with other warps, so a CTA is just six workers sharing an SM.
//
// Combine kernel, one CTA per (sequence, q head): lse = log sum_s e^{lse_s};
// out = sum_s e^{lse_s - lse} o_s (the split-KV merge named by num_splits in the
// flash-attention-npu flash_attn_with_kvcache docstring; split-KV for decode load balance is
// listed in the Flash-Sparse-Attention README).  A split with no token has lse_s = -inf and
// weight 0; a row with no token at all outputs 0 and lse = -inf.
#include <cuda_fp16.h>

#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kDecWarps = 6;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kStageTok = 16;     // tokens per pipeline stage (one m16n8k16 K extent)
constexpr int kDecStages = 2;     // per-warp ring depth: one stage in flight while the other is consumed
constexpr int kFusedMaxTopk = 2048;  // the in-kernel dedupe keeps a (sequence, kv head)'s list in shared memory
// Without the in-kernel dedupe a warp stages its canonical positions from global memory this many
// at a time, in its own slice of the list buffer.
constexpr int kNfWin = (kFusedMaxTopk / kDecWarps) / kStageTok * kStageTok;
constexpr float kLn2d = 0.6931471805599453f;
constexpr float kRescaleLog2d = 8.0f;

template <int D>
struct DecCfg {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kChunks = D / 8;  // 16-byte chunks per row
    static constexpr int kTileBytes = kStageTok * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;  // K then V
    static constexpr int kWarpRing = kDecStages * kStageBytes;
    static constexpr int kOffRows = kDecWarps * kWarpRing;
    static constexpr int kBtMax = 1536;                   // block-table entries kept in shared memory
    static constexpr int kOffBt = kOffRows;               // the sequence's block-table row
    static constexpr int kOffList = kOffBt + kBtMax * 4;  // positions, then physical row offsets
    static constexpr int kBytes = kOffList + kFusedMaxTopk * 4;
    static constexpr int kBitmapWords = kOffRows / 4;  // the dedupe bitmap borrows the rings
};

// Byte offset of 16-byte chunk c of row r in a tile whose rows are D*2 bytes: the chunk index
// is XOR-ed with (r & 7) so eight consecutive rows read by ldmatrix hit distinct banks.
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)(r * DecCfg<D>::kRowBytes + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t ld_q2(const __nv_bfloat16 *p)
{
    return __ldg(reinterpret_cast<const uint32_t *>(p));
}

// Exclusive scan over the CTA's kDecThreads threads; returns the total (all threads call it).
__device__ __forceinline__ int cta_exclusive_scan(int v, int *scratch, int &excl)
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
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
        const int t = scratch[w];
        if (w < warp) before += t;
        total += t;
    }
    __syncthreads();
    excl = before + x - v;
    return total;
}

// Ascending, duplicate-free positions of one (sequence, kv head)'s selection, each in [0, L) and
// (window_left >= 0) >= L-1-window_left, into list[]; returns their number.  A bitmap over a
// range of positions at a time lives in `bm` (the pipeline rings, not in use yet).  Ids that are
// neither -1 nor in [0, L) set *bad.  All threads of the CTA call it.
template <int D>
__device__ int dedupe_positions(const int32_t *sel, int topk, int L, int wl, uint32_t *bm, int *list,
                                int *scratch, bool &bad)
{
    using C = DecCfg<D>;
    const bool vec = (topk & 3) == 0 && (reinterpret_cast<uintptr_t>(sel) & 15) == 0;
    const int lo_pos = wl >= 0 ? max(0, L - 1 - wl) : 0;
    // This thread's ids, read from global memory once for both passes (-1 past the end).
    constexpr int kIdRegs = 4 * ((kFusedMaxTopk / 4 + kDecThreads - 1) / kDecThreads);
    int ids[kIdRegs];
    if (vec) {
#pragma unroll
        for (int k = 0; k < kIdRegs / 4; ++k) {
            const int e = (threadIdx.x + k * kDecThreads) * 4;
            const int4 v = e < topk ? __ldg(reinterpret_cast<const int4 *>(sel + e)) : make_int4(-1, -1, -1, -1);
            ids[4 * k] = v.x;
            ids[4 * k + 1] = v.y;
            ids[4 * k + 2] = v.z;
            ids[4 * k + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < kIdRegs; ++k) {
            const int e = threadIdx.x + k * kDecThreads;
            ids[k] = e < topk ? __ldg(&sel[e]) : -1;
        }
    }
    int n = 0;
    // Positions [c0, c1) at a time.  Thread t owns the `per` consecutive bitmap words
    // [t*per, (t+1)*per); word w is stored at (w % per) * kDecThreads + w / per, so when every
    // thread walks its own words in order, the 32 lanes of a warp read 32 consecutive addresses.
    // Beside the bitmap: wpref, the number of kept positions before each word.  A kept position j
    // then goes straight to list[wpref[word] + (set bits below j in its word)] — duplicates write
    // the same value to the same slot.
    constexpr int kPer = C::kBitmapWords / 2 / kDecThreads;  // words per thread and range
    constexpr int kRange = kPer * kDecThreads * 32;
    int *wpref = reinterpret_cast<int *>(bm + kPer * kDecThreads);
    for (int c0 = 0; c0 < L; c0 += kRange) {
        const int c1 = min(L, c0 + kRange);
        const int nw = (c1 - c0 + 31) >> 5;
        // words per thread, rounded up to a power of two so the slot arithmetic is shifts and masks
        int per_shift = 0;
        while ((kDecThreads << per_shift) < nw) ++per_shift;
        const int per = 1 << per_shift;
        for (int w = threadIdx.x; w < per * kDecThreads; w += kDecThreads) bm[w] = 0u;
        __syncthreads();
        // slot of word w of this range, or -1 when position j is not kept here
        auto slot = [&](int j) -> int {
            if (j < lo_pos || j < c0 || j >= c1) return -1;
            const int w = (j - c0) >> 5;
            return (w & (per - 1)) * kDecThreads + (w >> per_shift);
        };
        auto for_each_id = [&](auto &&f) {
#pragma unroll
            for (int k = 0; k < kIdRegs; ++k) f(ids[k]);
        };
        for_each_id([&](int j) {
            if (j == -1) return;
            if (j < 0 || j >= L) {
                bad = true;
                return;
            }
            const int sl = slot(j);
            if (sl >= 0) atomicOr(&bm[sl], 1u << ((j - c0) & 31));
        });
        __syncthreads();
        int cnt = 0;
        for (int k = 0; k < per; ++k) cnt += __popc(bm[k * kDecThreads + threadIdx.x]);
        int pos;
        const int total = cta_exclusive_scan(cnt, scratch, pos);
        pos += n;
        for (int k = 0; k < per; ++k) {
            wpref[k * kDecThreads + threadIdx.x] = pos;
            pos += __popc(bm[k * kDecThreads + threadIdx.x]);
        }
        __syncthreads();
        for_each_id([&](int j) {
            if (j < 0 || j >= L) return;
            const int sl = slot(j);
            if (sl >= 0) list[wpref[sl] + __popc(bm[sl] & ((1u << ((j - c0) & 31)) - 1u))] = j;
        });
        n += total;
        __syncthreads();  // the list is complete and the bitmap read out before the next range
    }
    return n;
}

// FP8 caches (F8): a warp's ring keeps the same size, split into one bf16 K/V tile pair (the layout
// the MMA code reads, at the start of the ring) and two landing stages of E4M3 rows (D bytes each,
// unswizzled) behind it; each stage is converted into the bf16 tiles before its products.  E4M3
// values are exact in bf16, so the products see the cached values themselves; the per (sequence, kv
// head) descales multiply the score scale (k) and the normalised output (v).
template <int D>
struct DecF8 {
    static constexpr int kRowBytes = D;                        // E4M3 row
    static constexpr int kChunks = D / 16;                     // 16-byte chunks per row
    static constexpr int kTileBytes = kStageTok * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;         // K then V
    static constexpr int kOffLanding = DecCfg<D>::kStageBytes;  // behind the bf16 tile pair
    static_assert(kOffLanding + kDecStages * kStageBytes == DecCfg<D>::kWarpRing, "ring size");
};

// 16 E4M3 values (one 16-byte chunk, lowest byte first) to 16 bf16 values (two 16-byte chunks).
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4 in, uint4 &lo, uint4 &hi)
{
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t r[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint16_t pair = (uint16_t)(w[i] >> (16 * hh));
            uint32_t h2;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
            r[2 * i + hh] = pack_bf16x2(f.x, f.y);
        }
    }
    lo = make_uint4(r[0], r[1], r[2], r[3]);
    hi = make_uint4(r[4], r[5], r[6], r[7]);
}

template <int D, bool F8>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecSplitParams p)
{
    using C = DecCfg<D>;
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ int scan_scratch[kDecWarps];
    __shared__ int s_n;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cps = (p.S + kDecWarps - 1) / kDecWarps;  // CTAs per (sequence, kv head)
    const int bh = blockIdx.x / cps;                     // b * Hkv + hk
    const int split = (blockIdx.x - bh * cps) * kDecWarps + warp;
    const int hk = bh % p.Hkv, b = bh / p.Hkv;
    const float k_ds = F8 && p.kd ? __ldg(&p.kd[bh]) : 1.f, v_ds = F8 && p.vd ? __ldg(&p.vd[bh]) : 1.f;
    const float scale_log2 = p.scale_log2 * k_ds;  // the k descale scales every score of this (b, kv head)
    // The sequence's block-table row into shared memory when it fits (read while the selection is
    // deduplicated), so a token's physical row is found without a dependent global load.
    int *bt_s = reinterpret_cast<int *>(dsm + C::kOffBt);
    const int32_t *bt_g = p.bt + (int64_t)b * p.max_pages;
    const bool bt_smem = p.max_pages <= C::kBtMax;
    if (bt_smem)
        for (int i = threadIdx.x; i < p.max_pages; i += kDecThreads) bt_s[i] = __ldg(&bt_g[i]);
    const int32_t *toks;
    int n;
    if (p.fused) {
        int L = p.seqlens[b];
        if (L > p.max_pages * p.page) {  // more tokens than the block table can address
            if (threadIdx.x == 0 && split == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
            L = p.max_pages * p.page;
        }
        L = max(L, 0);
        int *list = reinterpret_cast<int *>(dsm + C::kOffList);
        bool bad = false;
        const int nn = dedupe_positions<D>(p.sel + (int64_t)bh * p.topk, p.topk, L, p.wl,
                                           reinterpret_cast<uint32_t *>(dsm), list, scan_scratch, bad);
        if (bad && split == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_INDEX);
        if (threadIdx.x == 0) s_n = nn;
        __syncthreads();
        n = s_n;
        toks = list;
    } else {
        n = p.cnt[bh];
        toks = p.tok_c + (int64_t)bh * p.topk;
        __syncthreads();  // the block-table row is in shared memory
    }
    const bool active = split < p.S;  // a CTA's last warps may have no split
    const int chunk = (n + p.S - 1) / p.S;
    const int begin = min(n, split * chunk);
    const int ntok = active ? min(n, begin + chunk) - begin : 0;
    toks += begin;
    const uint32_t ring = smem_u32(dsm) + warp * C::kWarpRing;
    // Physical row offsets of the warp's tokens: in place over its part of the deduplicated list
    // (one pass), or, from the prep kernel's list, kNfWin at a time in the warp's slice of the buffer.
    int *list_s = reinterpret_cast<int *>(dsm + C::kOffList);
    int *rowoff = p.fused ? list_s + begin : list_s + warp * kNfWin;
    const int wcap = p.fused ? max(ntok, 1) : kNfWin;

    // A fragments of the G query rows (rows >= G are zero), straight from global memory.
    uint32_t aq[D / 16][4];
    {
        const int r = lane >> 2, cq = 2 * (lane & 3);
        const __nv_bfloat16 *qb = p.q + ((int64_t)b * p.Hq + hk * p.G) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            aq[ks][0] = r < p.G ? ld_q2(qb + r * D + ks * 16 + cq) : 0u;
            aq[ks][1] = r + 8 < p.G ? ld_q2(qb + (r + 8) * D + ks * 16 + cq) : 0u;
            aq[ks][2] = r < p.G ? ld_q2(qb + r * D + ks * 16 + 8 + cq) : 0u;
            aq[ks][3] = r + 8 < p.G ? ld_q2(qb + (r + 8) * D + ks * 16 + 8 + cq) : 0u;
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY};  // running max (scaled, base 2) of rows lane/4, lane/4+8
    float l_r[2] = {0.f, 0.f};              // this thread's share of the running sums
    bool bad_page = false;

    for (int w0 = 0; w0 < ntok; w0 += wcap) {
        const int wn = min(wcap, ntok - w0);
        __syncwarp();
        for (int e = lane; e < wn; e += 32) {
            const int pos = toks[w0 + e];  // (fused: the same shared-memory slot the offset goes to)
            const int pi = p.page_shift >= 0 ? pos >> p.page_shift : pos / p.page;  // page of the position
            const int pg = bt_smem ? bt_s[pi] : __ldg(&bt_g[pi]);
            if (pg < 0 || pg >= p.num_pages) {
                rowoff[e] = -1;
                bad_page = true;
            } else {
                rowoff[e] = (pg * p.page + (pos - pi * p.page)) * p.Hkv + hk;
            }
        }
        __syncwarp();
        const int nst = (wn + kStageTok - 1) / kStageTok;
        auto load_stage = [&](int stage, int s) {
            if constexpr (F8) {
                using F = DecF8<D>;
                const uint32_t kdst = ring + F::kOffLanding + stage * F::kStageBytes;
                const uint32_t vdst = kdst + F::kTileBytes;
                const uint8_t *kc8 = reinterpret_cast<const uint8_t *>(p.kc);
                const uint8_t *vc8 = reinterpret_cast<const uint8_t *>(p.vc);
                const int c = lane % F::kChunks;
#pragma unroll
                for (int tt = lane / F::kChunks; tt < kStageTok; tt += 32 / F::kChunks) {
                    const int e = s * kStageTok + tt;
                    const int ro = e < wn ? rowoff[e] : -1;
                    const int64_t off = ro >= 0 ? (int64_t)ro * D + c * 16 : 0;
                    const uint32_t nbytes = ro >= 0 ? 16u : 0u;
                    cp_async16(kdst + tt * D + c * 16, kc8 + off, nbytes);
                    cp_async16(vdst + tt * D + c * 16, vc8 + off, nbytes);
                }
            } else {
                const uint32_t kdst = ring + stage * C::kStageBytes;
                const uint32_t vdst = kdst + C::kTileBytes;
                const int c = lane % C::kChunks;
#pragma unroll
                for (int tt = lane / C::kChunks; tt < kStageTok; tt += 32 / C::kChunks) {
                    const int e = s * kStageTok + tt;
                    const int ro = e < wn ? rowoff[e] : -1;
                    const int64_t off = ro >= 0 ? (int64_t)ro * D + c * 8 : 0;
                    const uint32_t nbytes = ro >= 0 ? 16u : 0u;
                    cp_async16(kdst + swz<D>(tt, c), p.kc + off, nbytes);
                    cp_async16(vdst + swz<D>(tt, c), p.vc + off, nbytes);
                }
            }
        };
#pragma unroll
        for (int s = 0; s < kDecStages - 1; ++s) {
            if (s < nst) load_stage(s, s);
            cp_async_commit();
        }
        for (int it = 0; it < nst; ++it) {
            cp_async_wait<kDecStages - 2>();
            __syncwarp();
            {
                const int nxt = it + kDecStages - 1;
                if (nxt < nst) load_stage(nxt % kDecStages, nxt);
                cp_async_commit();
            }
            uint32_t kt = ring + (it % kDecStages) * C::kStageBytes;
            if constexpr (F8) {
                // this stage's E4M3 rows into the bf16 tile pair (swizzled as the MMA code reads it)
                using F = DecF8<D>;
                const uint8_t *land = dsm + (ring - smem_u32(dsm)) + F::kOffLanding + (it % kDecStages) * F::kStageBytes;
                uint8_t *tiles = dsm + (ring - smem_u32(dsm));
#pragma unroll
                for (int e = lane; e < 2 * kStageTok * F::kChunks; e += 32) {
                    const int kv = e / (kStageTok * F::kChunks), rem = e - kv * (kStageTok * F::kChunks);
                    const int tt = rem / F::kChunks, c = rem - tt * F::kChunks;
                    const uint4 in = *reinterpret_cast<const uint4 *>(land + kv * F::kTileBytes + tt * D + c * 16);
                    uint4 lo, hi;
                    e4m3x16_to_bf16(in, lo, hi);
                    uint8_t *tile = tiles + kv * C::kTileBytes;
                    *reinterpret_cast<uint4 *>(tile + swz<D>(tt, 2 * c)) = lo;
                    *reinterpret_cast<uint4 *>(tile + swz<D>(tt, 2 * c + 1)) = hi;
                }
                __syncwarp();
                kt = ring;
            }
            const uint32_t vt = kt + C::kTileBytes;
            const int mi = lane >> 3;

            // S = Q K^T for the stage's tokens 0..7 (s0) and 8..15 (s1).
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const int rr = (mi >> 1) * 8 + (lane & 7);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t k0, k1, k2, k3;
                    ldmatrix_x4(kt + swz<D>(rr, ks * 2 + (mi & 1)), k0, k1, k2, k3);
                    mma_bf16_16816(s0, aq[ks], k0, k1);
                    mma_bf16_16816(s1, aq[ks], k2, k3);
                }
            }
            // Tokens past the window or on a bad page are masked.
            const int tb = it * kStageTok + 2 * (lane & 3);
            bool valid[4];
            {
                const int t4[4] = {tb, tb + 1, tb + 8, tb + 9};
#pragma unroll
                for (int u = 0; u < 4; ++u) valid[u] = t4[u] < wn && rowoff[t4[u]] >= 0;
            }
            float sv[2][4] = {{valid[0] ? s0[0] : -INFINITY, valid[1] ? s0[1] : -INFINITY,
                               valid[2] ? s1[0] : -INFINITY, valid[3] ? s1[1] : -INFINITY},
                              {valid[0] ? s0[2] : -INFINITY, valid[1] ? s0[3] : -INFINITY,
                               valid[2] ? s1[2] : -INFINITY, valid[3] ? s1[3] : -INFINITY}};
            float pr[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mx = fmaxf(fmaxf(sv[h][0], sv[h][1]), fmaxf(sv[h][2], sv[h][3]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_blk = mx * scale_log2;
                if (m_blk > m_r[h] + kRescaleLog2d) {  // uniform across the 4 lanes of a row
                    const float f = m_r[h] == -INFINITY ? 0.f : ex2(m_r[h] - m_blk);
                    m_r[h] = m_blk;
                    l_r[h] *= f;
#pragma unroll
                    for (int nt = 0; nt < D / 8; ++nt) {
                        o[nt][2 * h] *= f;
                        o[nt][2 * h + 1] *= f;
                    }
                }
                const float m_use = m_r[h] == -INFINITY ? 0.f : m_r[h];
                float sum = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    pr[h][u] = ex2(fmaf(sv[h][u], scale_log2, -m_use));
                    sum += pr[h][u];
                }
                l_r[h] += sum;
            }
            // O += P V for the stage's 16 tokens.
            uint32_t ap[4];
            ap[0] = pack_bf16x2(pr[0][0], pr[0][1]);
            ap[1] = pack_bf16x2(pr[1][0], pr[1][1]);
            ap[2] = pack_bf16x2(pr[0][2], pr[0][3]);
            ap[3] = pack_bf16x2(pr[1][2], pr[1][3]);
            {
                const int rr = (mi & 1) * 8 + (lane & 7);
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
    }
    if (bad_page && p.status) atomicOr(p.status, SFA_DEV_BAD_PAGE);

    // Normalised partial output and LSE of this split: into global memory for the combine kernel,
    // or, when the CTA holds every split of its (sequence, kv head), into this warp's own ring
    // (its copies have all landed) for the combine below.
    const bool cta_combine = cps == 1;
    float *po_s = reinterpret_cast<float *>(dsm + warp * C::kWarpRing);  // [16][D] then lse[16]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float l = l_r[h];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int row = (lane >> 2) + 8 * h;
        if (active && row < p.G) {
            const int hq = hk * p.G + row;
            const int64_t slot = ((int64_t)b * p.Hq + hq) * p.S + split;
            const float inv = l > 0.f ? v_ds / l : 0.f;  // the v descale scales the output
            float *dst = (cta_combine ? po_s + row * D : p.po + slot * D) + 2 * (lane & 3);
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt)
                *reinterpret_cast<float2 *>(dst + nt * 8) = make_float2(o[nt][2 * h] * inv, o[nt][2 * h + 1] * inv);
            const float ls = l > 0.f ? (m_r[h] + log2f(l)) * kLn2d : -INFINITY;
            if ((lane & 3) == 0) {
                if (cta_combine) po_s[16 * D + row] = ls;
                else p.plse[slot] = ls;
            }
        }
    }
    if (!cta_combine) return;
    // In-CTA LSE combine of the S <= 6 splits: lse = log sum_s e^{lse_s}; out = sum_s e^{lse_s - lse} o_s.
    __syncthreads();
    const int nsp = min(p.S, kDecWarps);
    for (int e = threadIdx.x; e < p.G * D; e += kDecThreads) {
        const int row = e / D, c = e - row * D;
        float ls[kDecWarps];
        float M = -INFINITY;
#pragma unroll
        for (int sp = 0; sp < kDecWarps; ++sp) {
            ls[sp] = sp < nsp ? reinterpret_cast<const float *>(dsm + sp * C::kWarpRing)[16 * D + row] : -INFINITY;
            M = fmaxf(M, ls[sp]);
        }
        float acc = 0.f, lse = -INFINITY;
        if (M != -INFINITY) {
            float Z = 0.f;
#pragma unroll
            for (int sp = 0; sp < kDecWarps; ++sp) Z += ls[sp] == -INFINITY ? 0.f : __expf(ls[sp] - M);
            lse = M + __logf(Z);
#pragma unroll
            for (int sp = 0; sp < kDecWarps; ++sp)
                if (ls[sp] != -INFINITY)
                    acc += __expf(ls[sp] - lse) *
                           reinterpret_cast<const float *>(dsm + sp * C::kWarpRing)[row * D + c];
        }
        const int64_t orow = (int64_t)b * p.Hq + hk * p.G + row;
        p.out_direct[orow * D + c] = __float2bfloat16_rn(acc);
        if (c == 0) p.lse_direct[orow] = lse;
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

template <int D, bool F8>
cudaError_t launch_split_t(const DecGeom &g, const DecSplitParams &p, cudaStream_t st)
{
    const size_t smem = DecCfg<D>::kBytes;
    const cudaError_t e = ensure_smem_for(decode_split_kernel<D, F8>, smem);
    if (e != cudaSuccess) return e;
    const int cps = (g.S + kDecWarps - 1) / kDecWarps;
    decode_split_kernel<D, F8><<<g.B * g.Hkv * cps, kDecThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

int decode_split_blocks_per_sm(int d)
{
    const size_t per = d == 64 ? DecCfg<64>::kBytes : DecCfg<128>::kBytes;
    int n = (int)((228 * 1024) / (per + 1024));
    return n < 1 ? 1 : n;
}

int decode_split_warps_per_block()
{
    return kDecWarps;
}

int decode_fused_max_topk()
{
    return kFusedMaxTopk;
}

cudaError_t launch_decode_split(const DecGeom &g, const DecSplitParams &p, cudaStream_t st)
{
    if (p.fp8) return g.d == 64 ? launch_split_t<64, true>(g, p, st) : launch_split_t<128, true>(g, p, st);
    return g.d == 64 ? launch_split_t<64, false>(g, p, st) : launch_split_t<128, false>(g, p, st);
}

cudaError_t launch_decode_combine(const DecGeom &g, const DecCombineParams &p, cudaStream_t st)
{
    if (g.d == 64) decode_combine_kernel<64><<<g.B * g.Hq, 64, 0, st>>>(p);
    else decode_combine_kernel<128><<<g.B * g.Hq, 128, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sfa
