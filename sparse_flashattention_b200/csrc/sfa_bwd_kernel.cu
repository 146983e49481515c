// Prefill backward attention kernels (sm_100a): gradients of the selected attention.
//
// The chain rule through the softmax (the FlashAttentionScoreGrad case study of the Ascend
// "Sparse FlashAttention" article): recompute P = exp(S - lse) from the forward's LSE, dP = dO V^T,
// dS = P o (dP - D) with D = rowsum(dO o O), then dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO —
// all restricted, like the forward, to the keys a row selected and its mask keeps.
//
// bwd_dq_kernel (query-major, one CTA per SM, persistent): the forward's tiles (Tq tokens x G heads
//   = 128 rows of one kv head) walk the ascending union of their rows' blocks.  Per block the MMA
//   thread issues S = Q K^T and dP = dO V^T into double-buffered TMEM, eight softmax warps (two per
//   row, 32 keys each) turn them into dS (bf16, written over the block's S columns), and dQ += dS K accumulates in TMEM
//   (A operand from TMEM, K read MN-major).  TMEM: 2 x S, 2 x dP, dQ = 384 of 512 columns.
//
// bwd_dkdv_kernel (block-major, one CTA per SM, persistent): a piece is up to kBwdPieceChunks
//   chunks of one (sequence, kv head, key block) row's token list.  K and V of the block stay in
//   shared memory; each chunk's Q and dO rows (Tq tokens x G heads) are gathered by two warps with
//   coalesced 16-byte cp.async copies into 128-byte-swizzled tiles (a TMA gather4 copy per four
//   rows measured several times slower: the copy engine, not the bytes, was the limit).  Per chunk: S = Q K^T and dP = dO V^T (TMEM,
//   double-buffered); eight softmax warps (two per row) write P and dS (bf16) into shared memory,
//   each row's token and (lse, D) read one chunk ahead from arrays the fill kernel wrote; then
//   dV^T += dO^T P and dK^T += Q^T dS, with the gathered tiles read MN-major as the A operand
//   (M = d = 128) and P / dS MN-major as B.  The accumulators live in TMEM across the piece; the
//   epilogue writes bf16 dK / dV, or, for a row cut into several pieces, writes an fp32 partial and
//   counts the piece done; the piece that completes the count sums the row's partials in piece
//   order, so the sums do not depend on timing and no piece waits for another.
//
// Every wait is bounded (sfa_device.cuh); on a timeout the CTA records SFA_DEV_TIMEOUT, lets its
// copies and MMAs land, frees TMEM and exits.
#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// =========================================================================================
// dQ
// =========================================================================================
// warp 0 producer, 1 MMA, 2..9 softmax / epilogue (two warps per TMEM lane quadrant, one per half
// of a block's keys and of dQ's columns), 10 tile fetch
constexpr int kDqThreads = 352;
constexpr int kDqFetchWarp = 10;
// K and V rings: K is held until its block's dQ product, V only until dP, so K gets the deeper ring
// (a K load is issued when the dQ product of the block kDqKStages back is done).
constexpr int kDqKStages = 5;
constexpr int kDqVStages = 3;

template <int D, int BS>
struct DqCfg {
    static constexpr int kTileBytes = 128 * D * 2;  // the tile's Q (or dO)
    static constexpr int kKVBytes = BS * D * 2;     // one K (or V) block
    static constexpr int kOffDO = kTileBytes;
    static constexpr int kOffK = 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kDqKStages * kKVBytes;
    static constexpr int kOffMeta = kOffV + kDqVStages * kKVBytes;
    static constexpr int kTmemCols = 512;
    static constexpr int kColDP = 2 * BS;
    static constexpr int kColDQ = 4 * BS;
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false);
    static constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, D, true);
    static_assert(kColDQ + D <= kTmemCols, "TMEM columns");
    static_assert(BS == 32 || BS == 64, "two softmax warps per row, BS / 2 keys each");
    static_assert(D == 64 || D == 128, "head dimension");
};

struct DqTile {
    int done, nU, hk, q0, sq, k0, sk, tok0, ntok;
};

struct DqMeta {
    uint64_t q_full, q_empty;
    uint64_t k_full[kDqKStages], k_empty[kDqKStages];
    uint64_t v_full[kDqVStages], v_empty[kDqVStages];
    uint64_t s_full[2], p_full[2], dq_done[2];
    uint64_t o_free;
    uint64_t meta_full[2], meta_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    DqTile info[2];
};

template <int D, int BS>
__host__ __device__ constexpr size_t dq_union_offset()
{
    return DqCfg<D, BS>::kOffMeta + ((sizeof(DqMeta) + 15) & ~size_t(15));
}

template <int D, int BS>
__global__ void __launch_bounds__(kDqThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
                  const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv, const BwdParams p)
{
    using C = DqCfg<D, BS>;
    extern __shared__ uint8_t dq_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dq_smem_raw) + 1023) & ~uintptr_t(1023));
    DqMeta *meta = reinterpret_cast<DqMeta *>(smem + C::kOffMeta);
    const int U = p.umax;
    int *s_union = reinterpret_cast<int *>(smem + dq_union_offset<D, BS>());  // [2][U]
    uint8_t *sQ = smem, *sDO = smem + C::kOffDO, *sK = smem + C::kOffK, *sV = smem + C::kOffV;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned full = 0xffffffffu;

    if (threadIdx.x == 0) {
        mbar_init(&meta->q_full, 1);
        mbar_init(&meta->q_empty, 1);
        for (int s = 0; s < kDqKStages; ++s) {
            mbar_init(&meta->k_full[s], 1);
            mbar_init(&meta->k_empty[s], 1);
        }
        for (int s = 0; s < kDqVStages; ++s) {
            mbar_init(&meta->v_full[s], 1);
            mbar_init(&meta->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&meta->s_full[s], 1);
            mbar_init(&meta->p_full[s], 256);
            mbar_init(&meta->dq_done[s], 1);
            mbar_init(&meta->meta_full[s], 32);
            mbar_init(&meta->meta_empty[s], 10);  // producer, MMA thread, 8 softmax warps
        }
        mbar_init(&meta->o_free, 256);
        mbar_init(&meta->drain, 1);
        meta->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&meta->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = meta->tmem_base;
    volatile int *abort_flag = &meta->abort_flag;
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmdo);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
    }

    if (warp == kDqFetchWarp) {
        // ------------------------------------------------------------------ tile fetch
        int k = 0;
        bool ok = true;
        while (ok) {
            const int m = k & 1;
            if (k >= 2) ok = mbar_wait(&meta->meta_empty[m], ((k >> 1) - 1) & 1, abort_flag, p.status);
            ok = __all_sync(full, ok);
            if (!ok) break;
            DqTile &ti = meta->info[m];
            int *uni = s_union + m * U;
            int tile, hk, b, qt, q0, sq;
            while (true) {  // next tile that holds query rows
                tile = 0;
                if (lane == 0) tile = atomicAdd(p.tile_counter, 1);
                tile = __shfl_sync(full, tile, 0);
                if (tile >= p.tiles) break;
                hk = tile % p.Hkv;
                const int rest = tile / p.Hkv;
                b = rest % p.batch;
                qt = p.nqt - 1 - rest / p.batch;
                q0 = p.cu_q[b];
                sq = p.cu_q[b + 1] - q0;
                if (qt * p.Tq < sq) break;
            }
            if (tile >= p.tiles) {
                if (lane == 0) ti.done = 1;
                mbar_arrive(&meta->meta_full[m]);
                break;
            }
            const int nU = p.ucnt[tile];
            for (int i = lane; i < nU; i += 32) uni[i] = p.uni[(int64_t)tile * U + i];
            if (lane == 0) {
                ti.done = 0;
                ti.nU = nU;
                ti.hk = hk;
                ti.q0 = q0;
                ti.sq = sq;
                ti.k0 = p.cu_k[b];
                ti.sk = p.cu_k[b + 1] - ti.k0;
                ti.tok0 = qt * p.Tq;
                ti.ntok = min(p.Tq, sq - ti.tok0);
            }
            mbar_arrive(&meta->meta_full[m]);
            ++k;
        }
    } else if (warp == 0) {
        // ------------------------------------------------------------------ producer
        int k_st = 0, k_ph = 0, nk = 0, v_st = 0, v_ph = 0, nv = 0, q_phases = 0;
        if (lane == 0) {
            int k = 0;
            bool ok = true;
            while (ok) {
                const int m = k & 1;
                ok = mbar_wait(&meta->meta_full[m], (k >> 1) & 1, abort_flag, p.status);
                if (!ok) break;
                const DqTile &ti = meta->info[m];
                if (ti.done) break;
                const int *uni = s_union + m * U;
                const int n = ti.nU, hk = ti.hk, k0 = ti.k0;
                if (k >= 1) ok = mbar_wait(&meta->q_empty, (k - 1) & 1, abort_flag, p.status);
                if (!ok) break;
                mbar_arrive_expect_tx(&meta->q_full, n > 0 ? 2u * D * (uint32_t)(p.G * p.Tq) * 2u : 0u);
                if (n > 0)
                    for (int c = 0; c < D / 64; ++c) {
                        tma_load_3d(&tmq, &meta->q_full, sQ + c * (128 * 128), c * 64, hk * p.G, ti.q0 + ti.tok0);
                        tma_load_3d(&tmdo, &meta->q_full, sDO + c * (128 * 128), c * 64, hk * p.G, ti.q0 + ti.tok0);
                    }
                q_phases = k + 1;
                for (int u = 0; ok && u < n; ++u) {
                    const int row = k0 + uni[u] * BS;
                    if (nk >= kDqKStages && !mbar_wait(&meta->k_empty[k_st], k_ph ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&meta->k_full[k_st], (uint32_t)C::kKVBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(&tmk, &meta->k_full[k_st], sK + k_st * C::kKVBytes + c * (BS * 128), c * 64, hk, row);
                    ++nk;
                    if (++k_st == kDqKStages) {
                        k_st = 0;
                        k_ph ^= 1;
                    }
                    if (nv >= kDqVStages && !mbar_wait(&meta->v_empty[v_st], v_ph ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&meta->v_full[v_st], (uint32_t)C::kKVBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(&tmv, &meta->v_full[v_st], sV + v_st * C::kKVBytes + c * (BS * 128), c * 64, hk, row);
                    ++nv;
                    if (++v_st == kDqVStages) {
                        v_st = 0;
                        v_ph ^= 1;
                    }
                }
                if (!ok) break;
                mbar_arrive(&meta->meta_empty[m]);
                ++k;
            }
            if (*abort_flag) {  // let every copy this CTA started land
                if (q_phases > 0) mbar_drain(&meta->q_full, (q_phases - 1) & 1);
                for (int st = 0; st < kDqKStages; ++st) {
                    const int c = nk > st ? (nk - st + kDqKStages - 1) / kDqKStages : 0;
                    if (c > 0) mbar_drain(&meta->k_full[st], (c - 1) & 1);
                }
                for (int st = 0; st < kDqVStages; ++st) {
                    const int c = nv > st ? (nv - st + kDqVStages - 1) / kDqVStages : 0;
                    if (c > 0) mbar_drain(&meta->v_full[st], (c - 1) & 1);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint64_t dQd = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dDOd = sdesc_sw128(smem_u32(sDO), 16, 1024);
            const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dV0 = sdesc_sw128(smem_u32(sV), 16, 1024);
            const uint64_t dKmn0 = sdesc_sw128(smem_u32(sK), BS * 128, 1024);  // K as the MN-major B of dS K
            int k = 0, jg0 = 0;
            int sk_st = 0, sk_ph = 0, sv_st = 0, sv_ph = 0, qk_st = 0;  // K/V stages of the next S/dP, K stage of the next dQ
            bool ok = true;
            while (ok) {
                const int m = k & 1;
                ok = mbar_wait(&meta->meta_full[m], (k >> 1) & 1, abort_flag, p.status);
                if (!ok) break;
                const DqTile &ti = meta->info[m];
                if (ti.done) break;
                const int n = ti.nU;
                ok = mbar_wait(&meta->q_full, k & 1, abort_flag, p.status);
                if (!ok) break;
                if (n == 0) umma_commit(&meta->q_empty);
                // S/dP of block u once its K and V have landed and dQ u-2 was issued (S u overwrites
                // the buffer whose dS that MMA reads); dQ u once dS u is written.  The tile's first
                // dQ MMA overwrites the accumulator: it waits until the previous epilogue read it.
                bool ofree = (k == 0);
                int ns = 0, np = 0, spins = 0;
                uint64_t idle_since = 0;
                while (ok && np < n) {
                    bool progressed = false;
                    if (ns < n && ns <= np + 1) {
                        const int jg = jg0 + ns;
                        if (mbar_test(smem_u32(&meta->k_full[sk_st]), sk_ph) &&
                            mbar_test(smem_u32(&meta->v_full[sv_st]), sv_ph)) {
                            tc_fence_after();
                            const uint32_t tS = tmem + (jg & 1) * BS, tDP = tmem + C::kColDP + (jg & 1) * BS;
                            const uint32_t ko = (uint32_t)sk_st * C::kKVBytes, vo = (uint32_t)sv_st * C::kKVBytes;
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint64_t ao = (uint64_t)(((ks >> 2) * (128 * 128) + (ks & 3) * 32) >> 4);
                                const uint64_t bo = (uint64_t)((ko + (ks >> 2) * (BS * 128) + (ks & 3) * 32) >> 4);
                                umma_bf16(tS, dQd + ao, dK0 + bo, C::kIdescS, ks > 0 ? 1u : 0u);
                            }
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint64_t ao = (uint64_t)(((ks >> 2) * (128 * 128) + (ks & 3) * 32) >> 4);
                                const uint64_t bo = (uint64_t)((vo + (ks >> 2) * (BS * 128) + (ks & 3) * 32) >> 4);
                                umma_bf16(tDP, dDOd + ao, dV0 + bo, C::kIdescS, ks > 0 ? 1u : 0u);
                            }
                            umma_commit(&meta->s_full[jg & 1]);
                            umma_commit(&meta->v_empty[sv_st]);  // V is done once dP is
                            ++ns;
                            if (++sk_st == kDqKStages) {
                                sk_st = 0;
                                sk_ph ^= 1;
                            }
                            if (++sv_st == kDqVStages) {
                                sv_st = 0;
                                sv_ph ^= 1;
                            }
                            if (ns == n) umma_commit(&meta->q_empty);
                            progressed = true;
                        }
                    }
                    if (np < ns) {
                        const int ig = jg0 + np, st = qk_st;
                        if (mbar_test(smem_u32(&meta->p_full[ig & 1]), (ig >> 1) & 1) &&
                            (ofree || mbar_test(smem_u32(&meta->o_free), (k - 1) & 1))) {
                            ofree = true;
                            tc_fence_after();
#pragma unroll
                            for (int ks = 0; ks < BS / 16; ++ks)  // dS (bf16) sits in the first BS/2 columns
                                umma_bf16_tmem_a(tmem + C::kColDQ, tmem + (ig & 1) * BS + ks * 8,
                                                 dKmn0 + (uint64_t)((st * C::kKVBytes + ks * 16 * 128) >> 4), C::kIdescDQ,
                                                 (np > 0 || ks > 0) ? 1u : 0u);
                            umma_commit(&meta->dq_done[ig & 1]);
                            umma_commit(&meta->k_empty[st]);
                            ++np;
                            if (++qk_st == kDqKStages) qk_st = 0;
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        spins = 0;
                    } else if (*abort_flag) {
                        ok = false;
                    } else if (spins++ == 0) {
                        idle_since = global_timer_ns();
                    } else if ((spins & 63) == 0 && global_timer_ns() - idle_since > kWaitLimitNs) {
                        *abort_flag = 1;
                        if (p.status) atomicOr(p.status, SFA_DEV_TIMEOUT);
                        ok = false;
                    }
                }
                if (!ok) break;
                mbar_arrive(&meta->meta_empty[m]);
                jg0 += n;
                ++k;
            }
            if (!ok) {
                umma_commit(&meta->drain);
                mbar_drain(&meta->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;
        const int hs = (warp - 2) >> 2;  // which half of the keys (and of dQ's columns) this warp takes
        const int r = quad * 32 + lane;
        const int tok = r / p.G, g = r - tok * p.G;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        int k = 0, jg0 = 0;
        bool ok = true;
        while (ok) {
            const int m = k & 1;
            ok = warp_all_ok(mbar_wait(&meta->meta_full[m], (k >> 1) & 1, abort_flag, p.status));
            if (!ok) break;
            const DqTile &ti = meta->info[m];
            if (ti.done) break;
            const int n = ti.nU, ntok = ti.ntok, hk = ti.hk;
            const int *uni = s_union + m * U;
            const bool row_valid = tok < ntok;
            const int i = ti.tok0 + tok;
            const int64_t t = (int64_t)ti.q0 + i;
            const int h = hk * p.G + g;
            const int delta_k = ti.sk - ti.sq;
            int lo = 0, hi = ti.sk - 1;
            if (p.wl >= 0) lo = max(lo, i + delta_k - p.wl);
            if (p.causal) hi = min(hi, i + delta_k);
            if (p.wr >= 0) hi = min(hi, i + delta_k + p.wr);
            const int32_t *gl = p.sel_c + (row_valid ? (t * p.Hkv + hk) * p.topk : 0);
            const int mycnt = row_valid ? p.cnt[t * p.Hkv + hk] : 0;
            int nxt = mycnt > 0 ? gl[0] : -1, ptr = 0;
            const float lse2 = row_valid ? p.lse[(int64_t)h * p.total_q + t] * kLog2e : 0.f;
            const float dlt = row_valid ? p.delta[(int64_t)h * p.total_q + t] : 0.f;
            for (int j = 0; j < n; ++j) {
                const int jg = jg0 + j;
                const int s = uni[j];
                const bool selected = nxt == s;
                if (selected) {
                    ++ptr;
                    nxt = ptr < mycnt ? gl[ptr] : -1;
                }
                ok = warp_all_ok(mbar_wait(&meta->s_full[jg & 1], (jg >> 1) & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                const uint32_t tS = lane_base + (jg & 1) * BS, tDP = lane_base + C::kColDP + (jg & 1) * BS;
                constexpr int KH = BS / 2;  // keys of this warp's half of the block
                if (!__any_sync(full, selected)) {  // dS = 0 for all 32 rows: dQ unchanged
                    uint32_t zero[KH / 2];
#pragma unroll
                    for (int e = 0; e < KH / 2; ++e) zero[e] = 0u;
                    tmem_st_cols<KH / 2>(tS + hs * (KH / 2), zero);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&meta->p_full[jg & 1]);
                    continue;
                }
                // Branch-free masking (the rows of a warp differ in what they keep): a row that did not
                // select the block gets exponent -inf, a key outside the row's window too; 2^-inf = 0.
                const int kb = s * BS;
                const float sl = selected ? p.scale_log2 : 0.f, bias = selected ? -lse2 : -INFINITY;
                {  // this warp's KH keys; dS of keys [KH hs, KH hs + KH) -> columns [KH/2 hs, KH/2 hs + KH/2)
                    uint32_t sr[KH], dr[KH], packed[KH / 2];
                    tmem_ld_cols<KH>(tS + hs * KH, sr);
                    tmem_ld_cols<KH>(tDP + hs * KH, dr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < KH / 2; ++e) {
                        const int c0 = kb + hs * KH + 2 * e;
                        float y0 = fmaf(__uint_as_float(sr[2 * e]), sl, bias);
                        float y1 = fmaf(__uint_as_float(sr[2 * e + 1]), sl, bias);
                        y0 = ((c0 >= lo) & (c0 <= hi)) ? y0 : -INFINITY;
                        y1 = ((c0 + 1 >= lo) & (c0 + 1 <= hi)) ? y1 : -INFINITY;
                        const float p0 = ex2(y0), p1 = ex2(y1);
                        packed[e] = pack_bf16x2(p0 * (__uint_as_float(dr[2 * e]) - dlt),
                                                p1 * (__uint_as_float(dr[2 * e + 1]) - dlt));
                    }
                    tmem_st_cols<KH / 2>(tS + hs * (KH / 2), packed);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&meta->p_full[jg & 1]);
            }
            if (!ok) break;
            // ------------------------------------------------------------ epilogue: dq = scale * dS K
            if (n > 0) {
                const int lg = jg0 + n - 1;
                ok = warp_all_ok(mbar_wait(&meta->dq_done[lg & 1], (lg >> 1) & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
            }
            __nv_bfloat16 *qrow = p.dq + (t * p.Hq + h) * D;
#pragma unroll 1
            for (int c = hs * (D / 64); c < (hs + 1) * (D / 64); ++c) {  // this warp's half of the columns
                uint32_t o[32];
                if (n > 0) {
                    tmem_ld32(lane_base + C::kColDQ + c * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0u;
                }
                if (row_valid) {
                    uint32_t wv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * p.scale, __uint_as_float(o[2 * e + 1]) * p.scale);
                    uint4 *dst = reinterpret_cast<uint4 *>(qrow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&meta->o_free);
            __syncwarp();
            if (lane == 0) mbar_arrive(&meta->meta_empty[m]);
            jg0 += n;
            ++k;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {  // the last CTA out leaves the tile counters cleared
        __threadfence();
        if (atomicAdd(&p.tile_counter[1], 1) == (int)gridDim.x - 1) {
            p.tile_counter[0] = 0;
            p.tile_counter[1] = 0;
        }
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// =========================================================================================
// dK, dV
// =========================================================================================
// warp 0 control + gather, 1 MMA, 2..9 softmax / epilogue (two warps per TMEM lane quadrant, one
// per half of the block's keys), 10 gather
constexpr int kKvThreads = 352;
constexpr int kKvGatherWarp2 = 10;
constexpr int kGatherLanes = 64;  // warps 0 and 10: each copies 64 of a chunk's 128 rows

// The transposed products dV^T += dO^T P and dK^T += Q^T dS take d as the MMA's M dimension (128
// rows of TMEM).  With d = 64 the A descriptor's second 64-row half reads the first one again: the
// products run at M = 128 and TMEM lanes 64..127 hold a copy that the epilogue ignores.  Their N
// dimension (keys) is 64: a block of 32 keys keeps 64-key rows in its P and dS tiles, keys 32..63
// written as zero, so the same 128-byte-swizzled layout serves both block sizes.
template <int D, int BS>
struct KvCfg {
    static_assert(D == 64 || D == 128, "head dimension");
    static_assert(BS == 32 || BS == 64, "two softmax warps per row, BS / 2 keys each");
    static constexpr int kNT = 64;                  // N of the transposed products
    static constexpr int kTileBytes = 128 * D * 2;  // 128 gathered rows of Q (or dO)
    static constexpr int kKVBytes = BS * D * 2;
    static constexpr int kPBytes = 128 * kNT * 2;   // P (or dS): 128 rows x 64 keys, bf16
    static constexpr int kOffQ = 0;                 // [2] stages
    static constexpr int kOffDO = 2 * kTileBytes;   // [2]
    static constexpr int kOffK = 4 * kTileBytes;
    static constexpr int kOffV = kOffK + kKVBytes;
    static constexpr int kOffP = kOffV + kKVBytes;  // [2]
    static constexpr int kOffDS = kOffP + 2 * kPBytes;
    static constexpr int kOffMeta = kOffDS + 2 * kPBytes;
    static constexpr int kTmemCols = 512;
    static constexpr int kColDP = 2 * BS;
    static constexpr int kColDV = 4 * BS;
    static constexpr int kColDK = kColDV + kNT;
    static constexpr uint32_t kALbo = D == 128 ? 128 * 128 : 0;  // M-halves of the transposed A operand
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false);
    static constexpr uint32_t kIdescT = idesc_bf16_f32_ab(128, kNT, true, true);
    static_assert(kColDK + kNT <= kTmemCols, "TMEM columns");
};

struct PieceInfo {
    int done, ntok, tok_begin, idx, npieces, slot, hk, s, q0, sq, k0, sk, rowoff, pad[3];
};

struct KvMeta {
    uint64_t meta_full[2], meta_empty[2];
    uint64_t kv_full, kv_empty;
    uint64_t qd_full[2], qd_empty[2];
    uint64_t s_full[2], p_full[2], p_free[2];
    uint64_t acc_full, acc_free, epi_bar, drain;
    uint32_t tmem_base;
    int abort_flag;
    int last_flag;  // the epilogue's piece finished its row last
    PieceInfo info[2];
};

template <int D, int BS>
__global__ void __launch_bounds__(kKvThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv, const BwdParams p)
{
    using C = KvCfg<D, BS>;
    extern __shared__ uint8_t kv_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(kv_smem_raw) + 1023) & ~uintptr_t(1023));
    KvMeta *meta = reinterpret_cast<KvMeta *>(smem + C::kOffMeta);
    uint8_t *sQ = smem + C::kOffQ, *sDO = smem + C::kOffDO, *sK = smem + C::kOffK, *sV = smem + C::kOffV;
    uint8_t *sP = smem + C::kOffP, *sDS = smem + C::kOffDS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&meta->meta_full[s], 1);
            mbar_init(&meta->meta_empty[s], 11);  // warp 0, MMA thread, 8 softmax warps, warp 10
            mbar_init(&meta->qd_full[s], kGatherLanes);  // one cp.async arrival per gathering lane
            mbar_init(&meta->qd_empty[s], 1);
            mbar_init(&meta->s_full[s], 1);
            mbar_init(&meta->p_full[s], 256);
            mbar_init(&meta->p_free[s], 1);
        }
        mbar_init(&meta->kv_full, 1);
        mbar_init(&meta->kv_empty, 1);
        mbar_init(&meta->acc_full, 1);
        mbar_init(&meta->acc_free, 256);
        mbar_init(&meta->epi_bar, 256);
        mbar_init(&meta->drain, 1);
        meta->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&meta->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = meta->tmem_base;
    volatile int *abort_flag = &meta->abort_flag;
    const int npieces_total = p.ctrl->npieces;

    if (warp == 0 || warp == kKvGatherWarp2) {
        // ------------------------------------------------------------------ loads
        // Warp 0 lane 0 takes the next piece, publishes it and TMA-loads the block's K and V; warps 0
        // and 10 gather each chunk's Q and dO rows (row r = token * G + head) with 16-byte cp.async
        // copies into the 128-byte-swizzled tiles, eight lanes per 128-byte row segment (coalesced);
        // rows past the chunk's tokens are zero-filled (they meet P = dS = 0).  Each lane's copies
        // arrive on the stage's barrier when they land.
        const int half = warp == 0 ? 0 : 1;
        if (warp == 0 && lane == 0) {
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
        }
        int kp = 0, cg = 0, kv_issued = 0;
        bool ok = true;
        while (ok) {
            const int m = kp & 1;
            PieceInfo &pi = meta->info[m];
            if (warp == 0) {
                if (kp >= 2) ok = warp_all_ok(mbar_wait(&meta->meta_empty[m], ((kp >> 1) - 1) & 1, abort_flag, p.status));
                if (!ok) break;
                int piece = 0;
                if (lane == 0) piece = atomicAdd(&p.ctrl->counter, 1);
                piece = __shfl_sync(0xffffffffu, piece, 0);
                if (piece >= npieces_total) {
                    if (lane == 0) {
                        pi.done = 1;
                        mbar_arrive(&meta->meta_full[m]);
                    }
                    break;
                }
                if (lane == 0) {
                    const BwdPiece pc = p.pieces[piece];
                    const int s = pc.row % p.nblk_max, bh = pc.row / p.nblk_max;
                    const int hk = bh % p.Hkv, b = bh / p.Hkv;
                    const int q0 = __ldg(&p.cu_q[b]), k0 = __ldg(&p.cu_k[b]);
                    pi.done = 0;
                    pi.ntok = pc.ntok;
                    pi.tok_begin = pc.tok_begin;
                    pi.idx = pc.idx;
                    pi.npieces = pc.npieces;
                    pi.slot = pc.slot;
                    pi.hk = hk;
                    pi.s = s;
                    pi.q0 = q0;
                    pi.sq = __ldg(&p.cu_q[b + 1]) - q0;
                    pi.k0 = k0;
                    pi.sk = __ldg(&p.cu_k[b + 1]) - k0;
                    pi.rowoff = p.rowoff[pc.row];
                    mbar_arrive(&meta->meta_full[m]);
                    // K and V of the block, once the previous piece's MMAs are done with them.
                    if (kp >= 1) ok = mbar_wait(&meta->kv_empty, (kp - 1) & 1, abort_flag, p.status);
                    if (ok) {
                        mbar_arrive_expect_tx(&meta->kv_full, 2u * (uint32_t)C::kKVBytes);
                        for (int c = 0; c < D / 64; ++c) {
                            tma_load_3d(&tmk, &meta->kv_full, sK + c * (BS * 128), c * 64, hk, k0 + s * BS);
                            tma_load_3d(&tmv, &meta->kv_full, sV + c * (BS * 128), c * 64, hk, k0 + s * BS);
                        }
                        ++kv_issued;
                    }
                }
                ok = warp_all_ok(ok);
                if (!ok) break;
            } else {
                ok = warp_all_ok(mbar_wait(&meta->meta_full[m], (kp >> 1) & 1, abort_flag, p.status));
                if (!ok) break;
                if (pi.done) break;
            }
            __syncwarp();
            const int ntok = pi.ntok, q0 = pi.q0, hk = pi.hk;
            const int32_t *toks = p.toks + pi.rowoff + pi.tok_begin;
            const int nch = (ntok + p.Tq - 1) / p.Tq;
            // Lane l resolves rows half*64 + l and half*64 + 32 + l of each chunk (one token lookup and
            // one division each); the copies then run along whole rows, D/8 lanes per row, each row's
            // global row index broadcast from the lane that resolved it.
            constexpr int kChunks = D / 8;              // 16-byte pieces per row
            constexpr int kRowsPerIter = 32 / kChunks;  // rows one copy instruction covers
            const int cl = lane % kChunks, chalf = cl >> 3, k8 = cl & 7;
            for (int c = 0; c < nch; ++c) {
                const int st = cg & 1;
                if (cg >= 2) ok = warp_all_ok(mbar_wait(&meta->qd_empty[st], ((cg >> 1) - 1) & 1, abort_flag, p.status));
                if (!ok) break;
                const int ntc = min(p.Tq, ntok - c * p.Tq), rows = ntc * p.G;
                const uint32_t qbase = smem_u32(sQ + st * C::kTileBytes), dbase = smem_u32(sDO + st * C::kTileBytes);
                long long grow2[2];  // global (token, head) rows of this lane's two rows, -1 past the chunk
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int rr = half * 64 + 32 * h2 + lane;
                    const int tt = rr / p.G, gg = rr - tt * p.G;
                    grow2[h2] = rr < rows ? ((long long)(q0 + toks[c * p.Tq + tt]) * p.Hq + hk * p.G + gg) : -1ll;
                }
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
                    for (int i = 0; i < 32 / kRowsPerIter; ++i) {
                        const int rl = i * kRowsPerIter + lane / kChunks;  // row within this half of 32
                        const int rr = half * 64 + 32 * h2 + rl;
                        const long long g = __shfl_sync(0xffffffffu, grow2[h2], rl);
                        const bool live = g >= 0;
                        const int64_t off = live ? (int64_t)g * D + cl * 8 : 0;
                        const uint32_t so = (uint32_t)(chalf * (128 * 128) + rr * 128 + ((k8 ^ (rr & 7)) << 4));
                        cp_async16(qbase + so, p.q + off, live ? 16u : 0u);
                        cp_async16(dbase + so, p.dout + off, live ? 16u : 0u);
                    }
                }
                cp_async_mbar_arrive(&meta->qd_full[st]);
                ++cg;
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&meta->meta_empty[m]);
            ++kp;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // this lane's copies have all landed
        if (*abort_flag && warp == 0 && lane == 0 && kv_issued > 0)
            mbar_drain(&meta->kv_full, (uint32_t)((kv_issued - 1) & 1));
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint64_t dQ[2], dDO[2], dQt[2], dDOt[2], dP[2], dDS[2];
            for (int b = 0; b < 2; ++b) {
                dQ[b] = sdesc_sw128(smem_u32(sQ + b * C::kTileBytes), 16, 1024);
                dDO[b] = sdesc_sw128(smem_u32(sDO + b * C::kTileBytes), 16, 1024);
                dQt[b] = sdesc_sw128(smem_u32(sQ + b * C::kTileBytes), C::kALbo, 1024);   // M = d, MN-major
                dDOt[b] = sdesc_sw128(smem_u32(sDO + b * C::kTileBytes), C::kALbo, 1024);
                dP[b] = sdesc_sw128(smem_u32(sP + b * C::kPBytes), C::kPBytes, 1024);     // N = keys, MN-major
                dDS[b] = sdesc_sw128(smem_u32(sDS + b * C::kPBytes), C::kPBytes, 1024);
            }
            const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dV = sdesc_sw128(smem_u32(sV), 16, 1024);
            int kp = 0, cg0 = 0;
            bool ok = true;
            while (ok) {
                const int m = kp & 1;
                ok = mbar_wait(&meta->meta_full[m], (kp >> 1) & 1, abort_flag, p.status);
                if (!ok) break;
                const PieceInfo &pi = meta->info[m];
                if (pi.done) break;
                const int nch = (pi.ntok + p.Tq - 1) / p.Tq;
                ok = mbar_wait(&meta->kv_full, kp & 1, abort_flag, p.status);
                if (!ok) break;
                // S/dP of chunk c once its rows have landed and the dK/dV products of chunk c-2 were
                // issued (their softmax has read that TMEM buffer); dK/dV of chunk c once P and dS
                // are written.  The piece's first dK/dV product overwrites the accumulators, so it
                // waits until the previous piece's epilogue has read them.
                bool accfree = (kp == 0);
                int ns = 0, np = 0, spins = 0;
                uint64_t idle_since = 0;
                while (ok && np < nch) {
                    bool progressed = false;
                    if (ns < nch && ns <= np + 1) {
                        const int cg = cg0 + ns, b = cg & 1;
                        if (mbar_test(smem_u32(&meta->qd_full[b]), (cg >> 1) & 1)) {
                            fence_proxy_async_smem();  // the rows came through cp.async (generic proxy)
                            tc_fence_after();
                            const uint32_t tS = tmem + b * BS, tDP = tmem + C::kColDP + b * BS;
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint64_t ao = (uint64_t)(((ks >> 2) * (128 * 128) + (ks & 3) * 32) >> 4);
                                const uint64_t bo = (uint64_t)(((ks >> 2) * (BS * 128) + (ks & 3) * 32) >> 4);
                                umma_bf16(tS, dQ[b] + ao, dK + bo, C::kIdescS, ks > 0 ? 1u : 0u);
                            }
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint64_t ao = (uint64_t)(((ks >> 2) * (128 * 128) + (ks & 3) * 32) >> 4);
                                const uint64_t bo = (uint64_t)(((ks >> 2) * (BS * 128) + (ks & 3) * 32) >> 4);
                                umma_bf16(tDP, dDO[b] + ao, dV + bo, C::kIdescS, ks > 0 ? 1u : 0u);
                            }
                            umma_commit(&meta->s_full[b]);
                            ++ns;
                            progressed = true;
                        }
                    }
                    if (np < ns) {
                        const int cg = cg0 + np, b = cg & 1;
                        if (mbar_test(smem_u32(&meta->p_full[b]), (cg >> 1) & 1) &&
                            (accfree || mbar_test(smem_u32(&meta->acc_free), (kp - 1) & 1))) {
                            accfree = true;
                            tc_fence_after();
#pragma unroll
                            for (int ks = 0; ks < 128 / 16; ++ks) {  // K dimension: the chunk's 128 rows
                                const uint64_t o = (uint64_t)((ks * 16 * 128) >> 4);
                                umma_bf16(tmem + C::kColDV, dDOt[b] + o, dP[b] + o, C::kIdescT, (np > 0 || ks > 0) ? 1u : 0u);
                            }
#pragma unroll
                            for (int ks = 0; ks < 128 / 16; ++ks) {
                                const uint64_t o = (uint64_t)((ks * 16 * 128) >> 4);
                                umma_bf16(tmem + C::kColDK, dQt[b] + o, dDS[b] + o, C::kIdescT, (np > 0 || ks > 0) ? 1u : 0u);
                            }
                            umma_commit(&meta->qd_empty[b]);
                            umma_commit(&meta->p_free[b]);
                            ++np;
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        spins = 0;
                    } else if (*abort_flag) {
                        ok = false;
                    } else if (spins++ == 0) {
                        idle_since = global_timer_ns();
                    } else if ((spins & 63) == 0 && global_timer_ns() - idle_since > kWaitLimitNs) {
                        *abort_flag = 1;
                        if (p.status) atomicOr(p.status, SFA_DEV_TIMEOUT);
                        ok = false;
                    }
                }
                if (!ok) break;
                umma_commit(&meta->acc_full);
                umma_commit(&meta->kv_empty);
                mbar_arrive(&meta->meta_empty[m]);
                cg0 += nch;
                ++kp;
            }
            if (!ok) {
                umma_commit(&meta->drain);
                mbar_drain(&meta->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;
        const int hs = (warp - 2) >> 2;  // which half of the block's keys this warp takes
        const int r = quad * 32 + lane;  // a chunk row in the softmax, a d index in the epilogue
        const int tl = r / p.G, g = r - tl * p.G;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        int kp = 0, cg0 = 0, epi_uses = 0;
        bool ok = true;
        while (ok) {
            const int m = kp & 1;
            ok = warp_all_ok(mbar_wait(&meta->meta_full[m], (kp >> 1) & 1, abort_flag, p.status));
            if (!ok) break;
            const PieceInfo pi = meta->info[m];
            if (pi.done) break;
            const int nch = (pi.ntok + p.Tq - 1) / p.Tq;
            const int kb = pi.s * BS, delta_k = pi.sk - pi.sq;
            const int32_t *toks = p.toks + pi.rowoff + pi.tok_begin;
            const int64_t hrow = (int64_t)(pi.hk * p.G + g) * p.total_q + pi.q0;
            // The row's token two chunks ahead and its lse and D one chunk ahead of use, so neither
            // the token lookup nor the two loads that depend on it wait on the critical path.
            auto tok_of = [&](int c) { return (c < nch && tl < min(p.Tq, pi.ntok - c * p.Tq)) ? toks[c * p.Tq + tl] : -1; };
            int i1 = tok_of(0), i2 = tok_of(1);
            float lse1 = i1 >= 0 ? p.lse[hrow + i1] : 0.f, dlt1 = i1 >= 0 ? p.delta[hrow + i1] : 0.f;
            for (int c = 0; c < nch; ++c) {
                const int cg = cg0 + c, b = cg & 1;
                const int i = i1;
                const float lse2 = lse1 * kLog2e, dlt = dlt1;
                i1 = i2;
                i2 = tok_of(c + 2);
                lse1 = i1 >= 0 ? p.lse[hrow + i1] : 0.f;
                dlt1 = i1 >= 0 ? p.delta[hrow + i1] : 0.f;
                int lo = 0, hi = pi.sk - 1;
                if (p.wl >= 0) lo = max(lo, i + delta_k - p.wl);
                if (p.causal) hi = min(hi, i + delta_k);
                if (p.wr >= 0) hi = min(hi, i + delta_k + p.wr);
                if (i < 0) hi = -1;  // a row past the chunk's tokens keeps nothing
                ok = warp_all_ok(mbar_wait(&meta->s_full[b], (cg >> 1) & 1, abort_flag, p.status));
                if (ok && cg >= 2) ok = warp_all_ok(mbar_wait(&meta->p_free[b], ((cg >> 1) - 1) & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                const uint32_t tS = lane_base + b * BS, tDP = lane_base + C::kColDP + b * BS;
                uint8_t *prow = sP + b * C::kPBytes + r * 128;
                uint8_t *dsrow = sDS + b * C::kPBytes + r * 128;
                constexpr int KH = BS / 2;  // keys of this warp's half of the block
                {
                    uint32_t sr[KH], dr[KH], pk[KH / 2], dk[KH / 2];
                    tmem_ld_cols<KH>(tS + hs * KH, sr);
                    tmem_ld_cols<KH>(tDP + hs * KH, dr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < KH / 2; ++e) {  // branch-free masking: exponent -inf outside the row's keys
                        const int c0 = kb + hs * KH + 2 * e;
                        float y0 = fmaf(__uint_as_float(sr[2 * e]), p.scale_log2, -lse2);
                        float y1 = fmaf(__uint_as_float(sr[2 * e + 1]), p.scale_log2, -lse2);
                        y0 = ((c0 >= lo) & (c0 <= hi)) ? y0 : -INFINITY;
                        y1 = ((c0 + 1 >= lo) & (c0 + 1 <= hi)) ? y1 : -INFINITY;
                        const float p0 = ex2(y0), p1 = ex2(y1);
                        pk[e] = pack_bf16x2(p0, p1);
                        dk[e] = pack_bf16x2(p0 * (__uint_as_float(dr[2 * e]) - dlt), p1 * (__uint_as_float(dr[2 * e + 1]) - dlt));
                    }
                    // 16-byte pieces (8 keys) of the row, 128-byte swizzle: piece x at (x ^ (row & 7)) * 16.
#pragma unroll
                    for (int x = 0; x < KH / 8; ++x) {
                        const int piece = hs * (KH / 8) + x, so = ((piece ^ (r & 7)) << 4);
                        *reinterpret_cast<uint4 *>(prow + so) = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
                        *reinterpret_cast<uint4 *>(dsrow + so) = make_uint4(dk[4 * x], dk[4 * x + 1], dk[4 * x + 2], dk[4 * x + 3]);
                    }
                    if constexpr (BS < C::kNT) {  // keys BS..63 of the 64-key row are zero
#pragma unroll
                        for (int x = 0; x < (C::kNT - BS) / 16; ++x) {
                            const int piece = BS / 8 + hs * ((C::kNT - BS) / 16) + x, so = ((piece ^ (r & 7)) << 4);
                            *reinterpret_cast<uint4 *>(prow + so) = make_uint4(0u, 0u, 0u, 0u);
                            *reinterpret_cast<uint4 *>(dsrow + so) = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&meta->p_full[b]);
            }
            if (!ok) break;
            // ------------------------------------------------------------ epilogue (thread = d index r, keys
            // [32 hs, 32 hs + 32))
            ok = warp_all_ok(mbar_wait(&meta->acc_full, kp & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            constexpr int HK = BS / 2;
            float dv[HK], dkk[HK];
            const bool dvalid = r < D;  // with d = 64, lanes 64..127 hold the ignored copy
            {
                uint32_t a[HK], bq[HK];
                tmem_ld_cols<HK>(lane_base + C::kColDV + hs * HK, a);
                tmem_ld_cols<HK>(lane_base + C::kColDK + hs * HK, bq);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < HK; ++e) {
                    dv[e] = __uint_as_float(a[e]);
                    dkk[e] = __uint_as_float(bq[e]) * p.scale;
                }
            }
            tc_fence_before();
            mbar_arrive(&meta->acc_free);  // the accumulators are in registers now
            const int nk = min(BS, pi.sk - kb);
            const int e0 = hs * HK;
            bool last = true;
            if (pi.npieces > 1) {
                // Write this piece's partial; the piece whose count arrival is the row's last sums all of
                // the row's partials in piece order (this one's included, read back) and writes dK / dV.
                constexpr size_t kSlot = (size_t)2 * BS * D;
                float *mine = p.part + (size_t)(pi.slot + pi.idx) * kSlot;
                if (dvalid)
#pragma unroll
                    for (int e = 0; e < HK; ++e) {
                        mine[(e0 + e) * D + r] = dv[e];
                        mine[BS * D + (e0 + e) * D + r] = dkk[e];
                    }
                __threadfence();
                ok = group_sync(&meta->epi_bar, epi_uses, abort_flag, p.status);
                if (!ok) break;
                if (r == 0 && hs == 0) meta->last_flag = atomicAdd(p.flags + pi.slot, 1) == pi.npieces - 1 ? 1 : 0;
                ok = group_sync(&meta->epi_bar, epi_uses, abort_flag, p.status);
                if (!ok) break;
                last = meta->last_flag != 0;
                if (last && dvalid) {
                    __threadfence();
#pragma unroll
                    for (int e = 0; e < HK; ++e) dv[e] = dkk[e] = 0.f;
                    for (int j = 0; j < pi.npieces; ++j) {
                        const float *pj = p.part + (size_t)(pi.slot + j) * kSlot;
#pragma unroll
                        for (int e = 0; e < HK; ++e) {
                            dv[e] += __ldcg(pj + (e0 + e) * D + r);
                            dkk[e] += __ldcg(pj + BS * D + (e0 + e) * D + r);
                        }
                    }
                }
            }
            if (last && dvalid) {
                __nv_bfloat16 *dvo = p.dv + ((int64_t)(pi.k0 + kb + e0) * p.Hkv + pi.hk) * D + r;
                __nv_bfloat16 *dko = p.dk + ((int64_t)(pi.k0 + kb + e0) * p.Hkv + pi.hk) * D + r;
                const int64_t stride = (int64_t)p.Hkv * D;
#pragma unroll
                for (int e = 0; e < HK; ++e)
                    if (e0 + e < nk) {
                        dvo[e * stride] = __float2bfloat16_rn(dv[e]);
                        dko[e * stride] = __float2bfloat16_rn(dkk[e]);
                    }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&meta->meta_empty[m]);
            cg0 += nch;
            ++kp;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

int sm_count()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}


template <int D, int BS>
size_t dq_smem_t(const BwdGeom &g)
{
    return 1024 + dq_union_offset<D, BS>() + (size_t)2 * g.f.umax * 4;
}

template <int D, int BS>
size_t dkdv_smem_t()
{
    return 1024 + KvCfg<D, BS>::kOffMeta + sizeof(KvMeta);
}

template <int D, int BS>
cudaError_t launch_dq_t(const BwdGeom &g, const BwdParams &p, const CUtensorMap &tq, const CUtensorMap &tdo,
                        const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st)
{
    const size_t smem = dq_smem_t<D, BS>(g);
    cudaError_t e = ensure_smem_for(bwd_dq_kernel<D, BS>, smem);
    if (e != cudaSuccess) return e;
    const int grid = std::max(1, std::min(p.tiles, sm_count()));
    bwd_dq_kernel<D, BS><<<grid, kDqThreads, smem, st>>>(tq, tdo, tk, tv, p);
    return cudaGetLastError();
}

template <int D, int BS>
cudaError_t launch_dkdv_t(const BwdParams &p, const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st)
{
    const size_t smem = dkdv_smem_t<D, BS>();
    cudaError_t e = ensure_smem_for(bwd_dkdv_kernel<D, BS>, smem);
    if (e != cudaSuccess) return e;
    bwd_dkdv_kernel<D, BS><<<sm_count(), kKvThreads, smem, st>>>(tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_dq_smem_bytes(const BwdGeom &g)
{
    if (g.f.d == 64) return g.f.bs == 32 ? dq_smem_t<64, 32>(g) : dq_smem_t<64, 64>(g);
    return g.f.bs == 32 ? dq_smem_t<128, 32>(g) : dq_smem_t<128, 64>(g);
}

size_t bwd_dkdv_smem_bytes(const BwdGeom &g)
{
    if (g.f.d == 64) return g.f.bs == 32 ? dkdv_smem_t<64, 32>() : dkdv_smem_t<64, 64>();
    return g.f.bs == 32 ? dkdv_smem_t<128, 32>() : dkdv_smem_t<128, 64>();
}

cudaError_t launch_bwd_dq(const BwdGeom &g, const BwdParams &p, const CUtensorMap &tq, const CUtensorMap &tdo,
                          const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st)
{
    if (g.f.d == 64)
        return g.f.bs == 32 ? launch_dq_t<64, 32>(g, p, tq, tdo, tk, tv, st) : launch_dq_t<64, 64>(g, p, tq, tdo, tk, tv, st);
    return g.f.bs == 32 ? launch_dq_t<128, 32>(g, p, tq, tdo, tk, tv, st) : launch_dq_t<128, 64>(g, p, tq, tdo, tk, tv, st);
}

cudaError_t launch_bwd_dkdv(const BwdGeom &g, const BwdParams &p, const CUtensorMap &tk, const CUtensorMap &tv,
                            cudaStream_t st)
{
    if (g.f.d == 64) return g.f.bs == 32 ? launch_dkdv_t<64, 32>(p, tk, tv, st) : launch_dkdv_t<64, 64>(p, tk, tv, st);
    return g.f.bs == 32 ? launch_dkdv_t<128, 32>(p, tk, tv, st) : launch_dkdv_t<128, 64>(p, tk, tv, st);
}

}  // namespace sfa
