// Prefill attention kernel for top-k sparse FlashAttention on sm_100a.
//
// One CTA computes one query tile: Tq consecutive tokens of one sequence times the G query
// heads that share one kv head (and therefore one block selection), Tq*G <= 128 rows — the
// GQA heads are packed into the M dimension of the tensor-core tile.  The CTA walks the
// ascending union of its rows' selected blocks (built by the prep kernel).  Per block s:
//
//   producer warp   TMA-loads K and V rows [s*bs, s*bs+bs) of the kv head into a 3-stage
//                   shared-memory ring (128-byte swizzle), signalling an mbarrier.
//   MMA warp        one thread issues tcgen05.mma: S = Q K^T into one of two TMEM score
//                   buffers, and O += P V into the TMEM output accumulator.
//   softmax warps   4 warps, one thread per row: read S from TMEM, apply the row's mask
//                   (block not selected by this row, bottom-right causal limit, window,
//                   sequence end), keep the running max and sum in fp32 (base-2 domain),
//                   write P = 2^(s*scale*log2e - m) as bf16 back into TMEM over its own scores,
//                   where the PV MMA reads it as the A operand, and rescale O in TMEM when the
//                   running max grows by more than 2^8.
//
// A CTA needs about 100 KB of shared memory and 256 TMEM columns, so two CTAs share an SM and
// one CTA's softmax overlaps the other's MMAs.
//
// The epilogue divides O by the running sum, writes bf16 out and the natural-log LSE.
// The method is the FlashAttention tiling with online softmax applied to the gathered blocks
// only, as the Ascend "Sparse FlashAttention" article describes the fused SFA operator
// (gather the top-k K/V, then QK^T, softmax and PV tile by tile in one kernel); the
// mask/GQA/LSE semantics are those of the flash-attention-npu FlashAttention v2 docstrings.
//
// Every mbarrier wait is bounded (sfa_device.cuh): on a timeout the CTA records
// SFA_DEV_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and exits.
#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kThreads = 192;  // warp 0 producer, warp 1 MMA, warps 2..5 softmax/epilogue
constexpr int kStages = 2;  // two 32 KB K/V stages keep the CTA near 100 KB: two CTAs per SM
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by more than 2^8
constexpr float kLn2 = 0.6931471805599453f;

template <int D, int BS>
struct Cfg {
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kKVBytes = BS * D * 2;  // one K (or V) block
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffMeta = kOffV + kStages * kKVBytes;
    static constexpr int kTmemCols = (2 * BS + D <= 128) ? 128 : 256;
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false);
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
};

struct Meta {
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];  // K of a block is free once its S MMA is done,
    uint64_t v_full[kStages], v_empty[kStages];  // V once its PV MMA is done
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int tile;  // the tile this CTA works on, broadcast by thread 0
};

__device__ __forceinline__ int warp_all(bool v)
{
    return __all_sync(0xffffffffu, v);
}

// Persistent CTAs (two per SM) take query tiles from a counter in the workspace, heaviest
// tiles first.  Barrier phases run on a per-CTA count of processed blocks (jg), so the
// pipeline state carries over from tile to tile; TMEM is allocated once.
template <int D, int BS>
__global__ void __launch_bounds__(kThreads, 2)
    fwd_attend_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const FwdAttendParams p)
{
    using C = Cfg<D, BS>;
    extern __shared__ uint8_t fwd_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(fwd_smem_raw) + 1023) & ~uintptr_t(1023));
    Meta *meta = reinterpret_cast<Meta *>(smem + C::kOffMeta);
    int *s_union = reinterpret_cast<int *>(smem + C::kOffMeta + sizeof(Meta));
    int *s_lists = s_union + p.umax;             // [Tq][topk]
    int *s_cnt = s_lists + p.Tq * p.topk;        // [Tq]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&meta->q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&meta->k_full[s], 1);
            mbar_init(&meta->k_empty[s], 1);
            mbar_init(&meta->v_full[s], 1);
            mbar_init(&meta->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&meta->s_full[s], 1);
            mbar_init(&meta->p_full[s], 128);
            mbar_init(&meta->pv_done[s], 1);
        }
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
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
    }

    grid_dep_wait();  // everything above ran while the prep kernels were finishing
    int jbase = 0;  // blocks this CTA processed in earlier tiles
    int titer = 0;  // tiles this CTA computed (phase of q_full)
    int last_jg[kStages], last_k[kStages];  // last block whose V (K) load went into each stage
#pragma unroll
    for (int s = 0; s < kStages; ++s) last_jg[s] = last_k[s] = -1;

    while (true) {
        if (threadIdx.x == 0) meta->tile = atomicAdd(p.tile_counter, 1);
        __syncthreads();
        const int tile = meta->tile;
        if (tile >= p.tiles || *abort_flag) break;
        const int hk = tile % p.Hkv;
        const int rest = tile / p.Hkv;
        const int b = rest % p.batch;
        const int qt = p.nqt - 1 - rest / p.batch;
        const int q0 = p.cu_q[b], sq = p.cu_q[b + 1] - q0;
        const int k0 = p.cu_k[b], sk = p.cu_k[b + 1] - k0;
        const int tok0 = qt * p.Tq;
        const int ntok = min(p.Tq, sq - tok0);
        const int nU = ntok > 0 ? p.ucnt[tile] : 0;
        if (ntok > 0 && nU < 0) {
            // The block-major kernel computes this tile's rows; only rows that keep no key at all
            // (no partial will ever arrive for them) are written here: output 0, lse -inf.
            for (int e = threadIdx.x; e < ntok * p.G; e += kThreads) {
                const int tt = e / p.G, gg = e - tt * p.G;
                const int64_t t = (int64_t)q0 + tok0 + tt;
                if (p.cnt[t * p.Hkv + hk] != 0) continue;
                const int h = hk * p.G + gg;
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (t * p.Hq + h) * D);
                for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
                p.lse[(int64_t)h * p.total_q + t] = -INFINITY;
            }
        }
        if (ntok > 0 && nU >= 0) {
            // Tile metadata into shared memory: the union of blocks, and each token's sorted list.
            const int *gu = p.uni + (int64_t)tile * p.umax;
            for (int j = threadIdx.x; j < nU; j += kThreads) s_union[j] = gu[j];
            for (int e = threadIdx.x; e < ntok * p.topk; e += kThreads) {
                const int tt = e / p.topk, slot = e - tt * p.topk;
                s_lists[e] = p.sel_c[((int64_t)(q0 + tok0 + tt) * p.Hkv + hk) * p.topk + slot];
            }
            for (int tt = threadIdx.x; tt < ntok; tt += kThreads)
                s_cnt[tt] = p.cnt[(int64_t)(q0 + tok0 + tt) * p.Hkv + hk];
            __syncthreads();

            if (warp == 0) {
                // -------------------------------------------------------------- producer
                if (lane == 0 && nU > 0) {
                    const uint32_t qbytes = (uint32_t)(D / 64) * 64u * (uint32_t)(p.G * p.Tq) * 2u;
                    mbar_arrive_expect_tx(&meta->q_full, qbytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(&tmq, &meta->q_full, sQ + c * (128 * 128), c * 64, hk * p.G, q0 + tok0);
                    // K of block j+1 goes out as soon as S_{j-1} has freed its stage, ahead of V_j
                    // (which waits for PV_{j-2}): S needs only K, so the loads S waits on are
                    // issued a softmax step earlier than a joint K/V stage would allow.
                    auto load_k = [&](int jg, int j) -> bool {
                        const int st = jg % kStages;
                        if (jg >= kStages &&
                            !mbar_wait(&meta->k_empty[st], ((jg / kStages) - 1) & 1, abort_flag, p.status))
                            return false;
                        const int row = k0 + s_union[j] * BS;
                        mbar_arrive_expect_tx(&meta->k_full[st], (uint32_t)C::kKVBytes);
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_3d(&tmk, &meta->k_full[st], sK + st * C::kKVBytes + c * (BS * 128), c * 64,
                                        hk, row);
                        last_k[st] = jg;
                        return true;
                    };
                    auto load_v = [&](int jg, int j) -> bool {
                        const int st = jg % kStages;
                        if (jg >= kStages &&
                            !mbar_wait(&meta->v_empty[st], ((jg / kStages) - 1) & 1, abort_flag, p.status))
                            return false;
                        const int row = k0 + s_union[j] * BS;
                        mbar_arrive_expect_tx(&meta->v_full[st], (uint32_t)C::kKVBytes);
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_3d(&tmv, &meta->v_full[st], sV + st * C::kKVBytes + c * (BS * 128), c * 64,
                                        hk, row);
                        last_jg[st] = jg;
                        return true;
                    };
                    if (load_k(jbase, 0)) {
                        for (int j = 0; j < nU; ++j) {
                            if (j + 1 < nU && !load_k(jbase + j + 1, j + 1)) break;
                            if (!load_v(jbase + j, j)) break;
                        }
                    }
                }
            } else if (warp == 1) {
                // -------------------------------------------------------------- MMA issuer
                // Issues S_j = Q K_j^T and PV_j = P_j V_j in whatever order their inputs become
                // ready, so PV_j never waits for block j+1's loads.  Order constraints: PV_j after
                // S_j; S_j after PV_{j-2} (its TMEM score buffer holds P_{j-2} until that MMA has
                // read it; tcgen05 MMAs of one thread run in issue order).
                if (lane == 0 && nU > 0) {
                    const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
                    const uint32_t tO = tmem + 2 * BS;
                    bool ok = mbar_wait(&meta->q_full, titer & 1, abort_flag, p.status);
                    int ns = 0, np = 0;
                    uint64_t idle_since = global_timer_ns();
                    while (ok && np < nU) {
                        bool progressed = false;
                        if (ns < nU && ns <= np + 1) {
                            const int jg = jbase + ns, st = jg % kStages;
                            if (mbar_test(smem_u32(&meta->k_full[st]), (jg / kStages) & 1)) {
                                tc_fence_after();
                                const uint32_t tS = tmem + (jg & 1) * BS;
#pragma unroll
                                for (int ks = 0; ks < D / 16; ++ks) {
                                    const uint64_t a =
                                        sdesc_sw128(sQa + (ks >> 2) * (128 * 128) + (ks & 3) * 32, 16, 1024);
                                    const uint64_t bd = sdesc_sw128(
                                        sKa + st * C::kKVBytes + (ks >> 2) * (BS * 128) + (ks & 3) * 32, 16, 1024);
                                    umma_bf16(tS, a, bd, C::kIdescS, ks > 0 ? 1u : 0u);
                                }
                                umma_commit(&meta->s_full[jg & 1]);
                                umma_commit(&meta->k_empty[st]);
                                ++ns;
                                progressed = true;
                            }
                        }
                        if (np < ns) {
                            const int ig = jbase + np, st = ig % kStages;
                            if (mbar_test(smem_u32(&meta->p_full[ig & 1]), (ig >> 1) & 1) &&
                                mbar_test(smem_u32(&meta->v_full[st]), (ig / kStages) & 1)) {
                                tc_fence_after();
#pragma unroll
                                for (int ks = 0; ks < BS / 16; ++ks) {
                                    // P (bf16) sits in the first BS/2 columns of its score buffer.
                                    const uint32_t a = tmem + (ig & 1) * BS + ks * 8;
                                    const uint64_t bd =
                                        sdesc_sw128(sVa + st * C::kKVBytes + ks * 16 * 128, BS * 128, 1024);
                                    umma_bf16_tmem_a(tO, a, bd, C::kIdescPV, (np > 0 || ks > 0) ? 1u : 0u);
                                }
                                umma_commit(&meta->pv_done[ig & 1]);
                                umma_commit(&meta->v_empty[st]);
                                ++np;
                                progressed = true;
                            }
                        }
                        if (progressed) {
                            idle_since = global_timer_ns();
                        } else if (*abort_flag) {
                            ok = false;
                        } else if (global_timer_ns() - idle_since > kWaitLimitNs) {
                            *abort_flag = 1;
                            if (p.status) atomicOr(p.status, SFA_DEV_TIMEOUT);
                            ok = false;
                        }
                    }
                    if (!ok) {  // wind down: wait for the MMAs already issued
                        umma_commit(&meta->drain);
                        mbar_drain(&meta->drain, 0);
                    }
                }
            } else {
                // -------------------------------------------------------------- softmax + epilogue
                const int quad = warp & 3;  // TMEM lane quadrant this warp may access
                const int r = quad * 32 + lane;
                const int tok = r / p.G, g = r % p.G;
                const bool row_valid = (tok < ntok);  // r < Tq*G is implied by tok < ntok <= Tq
                const int i = tok0 + tok;
                const int delta = sk - sq;
                int lo = 0, hi = sk - 1;
                if (p.wl >= 0) lo = max(lo, i + delta - p.wl);
                if (p.causal) hi = min(hi, i + delta);
                if (p.wr >= 0) hi = min(hi, i + delta + p.wr);
                const int *mylist = s_lists + (row_valid ? tok : 0) * p.topk;
                const int mycnt = row_valid ? s_cnt[tok] : 0;
                int ptr = 0;
                float m_run = -INFINITY;  // running max of s*scale*log2e
                float l_run = 0.f;
                const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
                const uint32_t tO = lane_base + 2 * BS;
                bool ok = true;

                for (int j = 0; j < nU; ++j) {
                    const int jg = jbase + j;
                    const int s = s_union[j];
                    const bool selected = ptr < mycnt && mylist[ptr] == s;
                    if (selected) ++ptr;
                    ok = warp_all(mbar_wait(&meta->s_full[jg & 1], (jg >> 1) & 1, abort_flag, p.status));
                    if (!ok) break;
                    tc_fence_after();
                    if (!__any_sync(0xffffffffu, selected)) {
                        // None of this warp's 32 rows selected the block: their P is zero, their running
                        // max and sum do not change, and the scores need not be read.
                        uint32_t zero[BS / 2];
#pragma unroll
                        for (int e = 0; e < BS / 2; ++e) zero[e] = 0u;
                        if constexpr (BS == 64) {
                            tmem_st32(lane_base + (jg & 1) * BS, zero);
                        } else {
                            tmem_st16(lane_base + (jg & 1) * BS, zero);
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(&meta->p_full[jg & 1]);
                        continue;
                    }
                    float x[BS];
                    {
                        uint32_t raw[BS];
                        tmem_ld32(lane_base + (jg & 1) * BS, *reinterpret_cast<uint32_t(*)[32]>(raw));
                        if constexpr (BS == 64)
                            tmem_ld32(lane_base + (jg & 1) * BS + 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32));
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < BS; ++e) x[e] = __uint_as_float(raw[e]);
                    }
                    // Rows that did not select this block contribute nothing (handled arithmetically
                    // below); selected rows are masked element by element only where the block
                    // straddles their causal / window edge.
                    const int kb = s * BS;
                    if (selected && !(kb >= lo && kb + BS - 1 <= hi)) {
#pragma unroll
                        for (int c = 0; c < BS; ++c) {
                            const int key = kb + c;
                            x[c] = (key >= lo && key <= hi) ? x[c] : -INFINITY;
                        }
                    }
                    const float mx = selected ? row_max3<BS>(x) : -INFINITY;
                    const float m_new = mx * p.scale_log2;
                    const bool need = m_new > m_run + kRescaleLog2;
                    // O must be rescaled only for rows whose earlier blocks contributed (m_run
                    // finite); a row's O is exactly 0 until its first kept key.
                    const bool need_o = need && m_run != -INFINITY;
                    float factor = 1.f;
                    if (need) {
                        factor = m_run == -INFINITY ? 0.f : ex2(m_run - m_new);
                        m_run = m_new;
                        l_run *= factor;
                    }
                    if (j > 0 && __any_sync(0xffffffffu, need_o)) {
                        const int pg = jg - 1;
                        ok = warp_all(mbar_wait(&meta->pv_done[pg & 1], (pg >> 1) & 1, abort_flag, p.status));
                        if (!ok) break;
                        tc_fence_after();
                        if (!need_o) factor = 1.f;
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tO + c * 32, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
                            tmem_st32(tO + c * 32, o);
                        }
                        tmem_wait_st();
                    }
                    const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                    uint32_t packed[BS / 2];
                    l_run += scores_to_p<BS>(x, selected ? p.scale_log2 : 0.f, selected ? -m_use : -INFINITY, packed);
                    // P overwrites the first BS/2 columns of its own score buffer (already in
                    // registers).  S_{jg} completing implies PV_{jg-2}, which read the previous P
                    // from this buffer, has completed too.
                    if constexpr (BS == 64) {
                        tmem_st32(lane_base + (jg & 1) * BS, packed);
                    } else {
                        tmem_st16(lane_base + (jg & 1) * BS, packed);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&meta->p_full[jg & 1]);
                }

                // ------------------------------------------------------------ epilogue
                if (ok && nU > 0) {
                    const int lg = jbase + nU - 1;
                    ok = warp_all(mbar_wait(&meta->pv_done[lg & 1], (lg >> 1) & 1, abort_flag, p.status));
                    tc_fence_after();
                }
                if (ok) {
                    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
                    const int64_t t = (int64_t)q0 + i;
                    const int h = hk * p.G + g;
                    __nv_bfloat16 *orow = p.out + (t * p.Hq + h) * D;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        if (nU > 0) {
                            tmem_ld32(tO + c * 32, o);
                            tmem_wait_ld();
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = 0u;
                        }
                        if (row_valid) {
                            uint32_t w[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l,
                                                   __uint_as_float(o[2 * e + 1]) * inv_l);
                            uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                        }
                    }
                    if (row_valid)
                        p.lse[(int64_t)h * p.total_q + t] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
                }
            }
            jbase += nU;
            titer += nU > 0 ? 1 : 0;
        }
        tc_fence_before();
        __syncthreads();  // the tile is done everywhere before the next one reuses its buffers
        tc_fence_after();
    }

    if (*abort_flag && warp == 0 && lane == 0) {  // wind down: let every copy this CTA started land
        if (titer > 0) mbar_drain(&meta->q_full, (titer - 1) & 1);
        for (int st = 0; st < kStages; ++st)
            if (last_jg[st] >= 0) mbar_drain(&meta->v_full[st], (last_jg[st] / kStages) & 1);
        for (int st = 0; st < kStages; ++st)
            if (last_k[st] >= 0) mbar_drain(&meta->k_full[st], (last_k[st] / kStages) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {  // the last CTA out leaves the tile counters cleared for the next call
        __threadfence();
        if (atomicAdd(&p.tile_counter[1], 1) == (int)gridDim.x - 1) {
            p.tile_counter[0] = 0;
            p.tile_counter[1] = 0;
        }
    }
    grid_dep_launch();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D, int BS>
size_t smem_bytes_for(const FwdGeom &g)
{
    using C = Cfg<D, BS>;
    return 1024 + C::kOffMeta + sizeof(Meta) + (size_t)g.umax * 4 + (size_t)g.Tq * g.topk * 4 + (size_t)g.Tq * 4;
}

template <int D, int BS>
cudaError_t launch_t(const FwdGeom &g, const FwdAttendParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                     const CUtensorMap &tv, cudaStream_t st)
{
    const size_t smem = smem_bytes_for<D, BS>(g);
    const cudaError_t e = ensure_smem_for(fwd_attend_kernel<D, BS>, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = g.tiles < 2 * sms ? g.tiles : 2 * sms;
    return launch_kernel(fwd_attend_kernel<D, BS>, dim3(grid), dim3(kThreads), smem, st, true, tq, tk, tv, p);
}

}  // namespace

size_t fwd_attend_smem_bytes(const FwdGeom &g)
{
    if (g.d == 64) return g.bs == 32 ? smem_bytes_for<64, 32>(g) : smem_bytes_for<64, 64>(g);
    return g.bs == 32 ? smem_bytes_for<128, 32>(g) : smem_bytes_for<128, 64>(g);
}

cudaError_t launch_fwd_attend(const FwdGeom &g, const FwdAttendParams &p, const CUtensorMap &tq,
                              const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st)
{
    if (g.d == 64) return g.bs == 32 ? launch_t<64, 32>(g, p, tq, tk, tv, st) : launch_t<64, 64>(g, p, tq, tk, tv, st);
    return g.bs == 32 ? launch_t<128, 32>(g, p, tq, tk, tv, st) : launch_t<128, 64>(g, p, tq, tk, tv, st);
}

}  // namespace sfa
