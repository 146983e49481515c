// Block-major prefill attention for sparse query windows, with the partial merge fused in.
//
// When a window's tokens select their blocks with little overlap (an NSA-style random top-k
// over a long prefix), the union of a query tile's blocks is many times the selected work.
// Here the loop is turned around, as the FSA project page describes for its selected-attention
// kernel (key/value block outer, queries inner): an item is one selected K/V block of one kv
// head plus up to Tq tokens of the window that selected it, Tq*G <= 128 query rows gathered
// into one tensor-core tile.  Per item the CTA computes S = Q K^T (tcgen05, TMEM), the masked
// softmax of that one block (max m, sum l, P = 2^(s*scale*log2e - m) in bf16 back into TMEM),
// O = P V (tcgen05), and writes every row's normalised partial o/l (bf16) with (m, l).
//
// A separate merge kernel (the reduction step of FSA's kernel split) then combines each row's
// partials: lse = log of the sum of l*2^m, out = the weighted mean of the partials.
//
// One persistent CTA per SM walks the item list with a fixed stride.  Warp 0 prefetches the
// next item's record and token list, TMA-loads the K/V block and gathers the item's Q rows with
// 16-byte cp.async copies into a 128-byte-swizzled tile; warp 1 issues the MMAs; two
// groups of four warps alternate over items (softmax and epilogue), so one group's softmax
// overlaps the other group's MMAs.  All waits are bounded.
#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kInvThreadsAttn = 384;  // warp 0 producer, warp 1 MMA, warps 2-5 and 6-9: two softmax groups,
                                      // warps 11 and 10: the first and second half of each item's Q-row gather
constexpr float kLn2i = 0.6931471805599453f;
constexpr int kItemSlots = 8;   // item j lives in slot j % 8; softmax group j % 2 handles it
constexpr int kFetchAhead = 4;  // item records are fetched this many items ahead
constexpr int kLoadStages = 3;  // Q and K/V buffers: item j uses buffer j % 3
constexpr int kInvCuCache = 255;  // sequences whose cu_seqlens entries are kept in shared memory

template <int D, int BS>
struct InvCfg {
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kKVBytes = BS * D * 2;
    static constexpr int kOffQ = 0;                                // Q[kLoadStages]
    static constexpr int kOffK = kLoadStages * kQBytes;            // K[kLoadStages]
    static constexpr int kOffV = kOffK + kLoadStages * kKVBytes;   // V[kLoadStages]
    static constexpr int kOffMeta = kOffV + kLoadStages * kKVBytes;
    static constexpr int kOffStage = kOffMeta + 4608;  // 8 softmax warps x 2 KB epilogue staging
    static constexpr int kStageBytes = 8 * 2048;
    static constexpr int kOffCu = kOffStage + kStageBytes;  // cu_seqlens_q, cu_seqlens_k
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false);
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
    static constexpr int kTmemCols = 512;  // S/P of group w at w*BS, O of group w at 128 + w*D
};


struct InvMeta {
    uint64_t item_full[kItemSlots], item_free[kItemSlots];
    uint64_t q_full[kLoadStages], q_empty[kLoadStages];
    uint64_t kv_full[kLoadStages], kv_empty[kLoadStages];
    uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    InvItem slot[kItemSlots];
};

// Rows [r0, r0 + 64) of an item's Q tile (row r = token * G + head; rows >= `rows` zero-filled) into
// the 128-byte-swizzled K-major tile at qt: chunk k of a row's 64-element half c lands at
// c * 16 KB + r * 128 + ((k ^ (r & 7)) << 4).  Lane l first finds the source rows r0 + l and
// r0 + 32 + l (one division and one shared-memory read each); then the lanes take consecutive
// 16-byte chunks of 32 / (D / 8) consecutive rows, each row's address broadcast from the lane that
// found it, so every copy instruction reads whole rows from global memory (coalesced) and fills
// whole 128-byte shared-memory lines.
template <int D>
__device__ __forceinline__ void gather_q_rows(const FwdAttendParams &p, const InvItem *item, int hk, int rows, int r0,
                                              uint32_t qt, int lane)
{
    constexpr int kChunks = D / 8;               // 16-byte chunks per row
    constexpr int kRowsPerIter = 32 / kChunks;   // rows one warp instruction covers
    const __nv_bfloat16 *src_row[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
        const int r = r0 + 32 * h2 + lane;
        const bool live = r < rows;
        const int tk = live ? r / p.G : 0, gg = live ? r - tk * p.G : 0;
        src_row[h2] = p.q + ((int64_t)(live ? (item->tok[tk] >> 7) : 0) * p.Hq + hk * p.G + gg) * D;
    }
    const int cc = lane % kChunks, c = cc >> 3, k = cc & 7;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
        for (int i = 0; i < 32 / kRowsPerIter; ++i) {
            const int rl = i * kRowsPerIter + lane / kChunks;  // row within this half of 32
            const int r = r0 + 32 * h2 + rl;
            const __nv_bfloat16 *src = reinterpret_cast<const __nv_bfloat16 *>(
                __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(src_row[h2]), rl));
            cp_async16(qt + c * (128 * 128) + r * 128 + ((k ^ (r & 7)) << 4), src + c * 64 + k * 8,
                       r < rows ? 16u : 0u);
        }
    }
}

template <int D, int BS>
__global__ void __launch_bounds__(kInvThreadsAttn, 1)
    fwd_attend_inv_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv, const FwdAttendParams p)
{
    using C = InvCfg<D, BS>;
    extern __shared__ uint8_t inv_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(inv_smem_raw) + 1023) & ~uintptr_t(1023));
    InvMeta *meta = reinterpret_cast<InvMeta *>(smem + C::kOffMeta);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dep_wait();
    // No window went block-major: leave before any barrier or TMEM is set up (uniform exit).
    if (__ldcg(&p.ctrl->item_total) == 0) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kItemSlots; ++s) {
            mbar_init(&meta->item_full[s], 1);
            mbar_init(&meta->item_free[s], 128);
        }
        for (int s = 0; s < kLoadStages; ++s) {
            mbar_init(&meta->q_full[s], 64);  // one cp.async arrival per lane of the two gathering warps
            mbar_init(&meta->q_empty[s], 1);
            mbar_init(&meta->kv_full[s], 1);
            mbar_init(&meta->kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&meta->s_full[s], 1);
            mbar_init(&meta->p_full[s], 128);
            mbar_init(&meta->pv_done[s], 1);
            mbar_init(&meta->o_free[s], 128);
        }
        mbar_init(&meta->drain, 1);
        meta->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&meta->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    // cu_seqlens_q / _k in shared memory (batches of up to kInvCuCache sequences), so an item's sequence
    // bounds cost no dependent global load on the softmax groups' path
    int *s_cu = reinterpret_cast<int *>(smem + C::kOffCu);
    if (p.batch <= kInvCuCache)
        for (int i = threadIdx.x; i <= p.batch; i += blockDim.x) {
            s_cu[i] = __ldg(&p.cu_q[i]);
            s_cu[kInvCuCache + 1 + i] = __ldg(&p.cu_k[i]);
        }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = meta->tmem_base;
    volatile int *abort_flag = &meta->abort_flag;
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer (all 32 lanes)
        // Item j of this CTA is item blockIdx.x + j * gridDim.x.  Its record and token list are
        // one 528-byte bulk copy into slot j % 8, issued four items ahead; past the last item the
        // slot gets an end marker instead.
        const int total = *reinterpret_cast<volatile int *>(&p.ctrl->item_total);
        auto fetch = [&](int j) {  // lane 0 only
            const int sl = j % kItemSlots;
            const long long idx = (long long)blockIdx.x + (long long)j * gridDim.x;
            if (idx < total) {
                mbar_arrive_expect_tx(&meta->item_full[sl], (uint32_t)sizeof(InvItem));
                bulk_load(&meta->slot[sl], &p.items[idx], (uint32_t)sizeof(InvItem), &meta->item_full[sl]);
            } else {
                meta->slot[sl].rec = make_int4(0, 0, 0, -1);
                mbar_arrive(&meta->item_full[sl]);
            }
        };
        if (lane == 0) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            for (int f = 0; f < kFetchAhead; ++f) fetch(f);
        }
        int issued[kLoadStages] = {};
        bool ok = true;
        for (int j = 0; ok; ++j) {
            const int sl = j % kLoadStages;                  // K/V and Q buffers
            const int it = j % kItemSlots;                   // item slot
            const uint32_t ph = ((j / kLoadStages) - 1) & 1; // previous use of this K/V or Q buffer
            ok = warp_all_ok(mbar_wait(&meta->item_full[it], (j / kItemSlots) & 1, abort_flag, p.status));
            if (!ok) break;
            const InvItem *item = &meta->slot[it];
            const int4 rec = item->rec;
            if (rec.w < 0) break;  // item j+1 is past the end too, so both groups get a marker
            const int hk = rec.x % p.Hkv;
            // K/V block
            if (j >= kLoadStages) ok = warp_all_ok(mbar_wait(&meta->kv_empty[sl], ph, abort_flag, p.status));
            if (!ok) break;
            if (lane == 0) {
                const int row = rec.z + rec.y * BS;  // the sequence's first K row comes with the record
                mbar_arrive_expect_tx(&meta->kv_full[sl], 2u * (uint32_t)C::kKVBytes);
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_3d(&tmk, &meta->kv_full[sl], sK + sl * C::kKVBytes + c * (BS * 128), c * 64, hk, row);
                    tma_load_3d(&tmv, &meta->kv_full[sl], sV + sl * C::kKVBytes + c * (BS * 128), c * 64, hk, row);
                }
                issued[sl]++;
            }
            // (the item's Q rows are gathered by warps 11 and 10)
            // Item j+4 goes into the slot item j-4 used, once its softmax group is done with it.
            if (j + kFetchAhead >= kItemSlots)
                ok = warp_all_ok(mbar_wait(&meta->item_free[(j + kFetchAhead) % kItemSlots],
                                           ((j + kFetchAhead - kItemSlots) / kItemSlots) & 1, abort_flag, p.status));
            if (!ok) break;
            if (lane == 0) fetch(j + kFetchAhead);
            __syncwarp();
        }
        if (*abort_flag && lane == 0) {
            for (int sl = 0; sl < kLoadStages; ++sl)
                if (issued[sl] > 0) mbar_drain(&meta->kv_full[sl], (issued[sl] - 1) & 1);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        // Issues S_ns = Q K^T and PV_np = P V in whatever order their inputs become ready, so an
        // item's PV never waits for the next item's loads.  Order constraints: PV_j after S_j;
        // S_j after PV_{j-2} (its TMEM score buffer holds P_{j-2} until that MMA has read it;
        // tcgen05 MMAs of one thread run in issue order).
        if (lane == 0) {
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
            int ns = 0, np = 0;
            bool end_seen = false, ok = true;
            uint64_t idle_since = global_timer_ns();
            while (ok) {
                bool progressed = false;
                if (!end_seen && ns <= np + 1) {
                    const int it = ns % kItemSlots, sl = ns % kLoadStages, sb = ns & 1;
                    const uint32_t ph = (ns / kLoadStages) & 1;
                    if (mbar_test(smem_u32(&meta->item_full[it]), (ns / kItemSlots) & 1)) {
                        if (meta->slot[it].rec.w < 0) {
                            end_seen = true;
                            progressed = true;
                        } else if (mbar_test(smem_u32(&meta->q_full[sl]), ph) &&
                                   mbar_test(smem_u32(&meta->kv_full[sl]), ph)) {
                            tc_fence_after();
                            const uint32_t tS = tmem + sb * BS;
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint64_t a = sdesc_sw128(
                                    sQa + sl * C::kQBytes + (ks >> 2) * (128 * 128) + (ks & 3) * 32, 16, 1024);
                                const uint64_t bd = sdesc_sw128(
                                    sKa + sl * C::kKVBytes + (ks >> 2) * (BS * 128) + (ks & 3) * 32, 16, 1024);
                                umma_bf16(tS, a, bd, C::kIdescS, ks > 0 ? 1u : 0u);
                            }
                            umma_commit(&meta->s_full[sb]);
                            umma_commit(&meta->q_empty[sl]);
                            ++ns;
                            progressed = true;
                        }
                    }
                }
                if (np < ns) {
                    const int w = np & 1;
                    if (mbar_test(smem_u32(&meta->p_full[w]), (np >> 1) & 1) &&
                        (np < 2 || mbar_test(smem_u32(&meta->o_free[w]), ((np >> 1) - 1) & 1))) {
                        tc_fence_after();
                        const uint32_t tO = tmem + 128 + w * D;
                        const int vs = np % kLoadStages;
#pragma unroll
                        for (int ks = 0; ks < BS / 16; ++ks) {
                            const uint32_t a = tmem + w * BS + ks * 8;
                            const uint64_t bd = sdesc_sw128(sVa + vs * C::kKVBytes + ks * 16 * 128, BS * 128, 1024);
                            umma_bf16_tmem_a(tO, a, bd, C::kIdescPV, ks > 0 ? 1u : 0u);
                        }
                        umma_commit(&meta->pv_done[w]);
                        umma_commit(&meta->kv_empty[vs]);
                        ++np;
                        progressed = true;
                    }
                }
                if (end_seen && np == ns) break;
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
            if (!ok) {
                umma_commit(&meta->drain);
                mbar_drain(&meta->drain, 0);
            }
        }
    } else if (warp >= 10) {
        // ---------------------------------------------------------------- Q-row gather
        // Warp 11 copies rows 0..63 of each item's Q tile (row r = token * G + head) into the
        // 128-byte-swizzled K-major tile the MMA reads, warp 10 rows 64..127; rows past the item are
        // zero-filled.  Each lane's copies land on q_full through its own arrival.  Both follow the
        // producer's item sequence: the item's slot stays valid until its softmax group frees it,
        // which needs these copies (q_full) first.
        const int r0 = warp == 11 ? 0 : 64;
        bool ok = true;
        for (int j = 0; ok; ++j) {
            const int sl = j % kLoadStages, it = j % kItemSlots;
            const uint32_t ph = ((j / kLoadStages) - 1) & 1;
            ok = warp_all_ok(mbar_wait(&meta->item_full[it], (j / kItemSlots) & 1, abort_flag, p.status));
            if (!ok) break;
            const InvItem *item = &meta->slot[it];
            const int4 rec = item->rec;
            if (rec.w < 0) break;
            const int hk = rec.x % p.Hkv;
            if (j >= kLoadStages) ok = warp_all_ok(mbar_wait(&meta->q_empty[sl], ph, abort_flag, p.status));
            if (!ok) break;
            gather_q_rows<D>(p, item, hk, rec.w * p.G, r0, smem_u32(sQ + sl * C::kQBytes), lane);
            cp_async_mbar_arrive(&meta->q_full[sl]);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // this lane's copies have all landed
    } else {
        // ---------------------------------------------------------------- softmax groups (warps 2-9)
        const int grp = (warp - 2) >> 2;        // 0: warps 2-5, 1: warps 6-9
        const int quad = warp & 3;              // TMEM lane quadrant of this warp
        const int r = quad * 32 + lane;         // tile row
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t tS = lane_base + grp * BS;
        const uint32_t tO = lane_base + 128 + grp * D;
        uint4 *stg = reinterpret_cast<uint4 *>(smem + C::kOffStage) + (warp - 2) * 128;  // 32 rows x 64 bytes
        bool ok = true;
        for (int j = grp; ok; j += 2) {
            const uint32_t ph = (j >> 1) & 1;
            const int it = j % kItemSlots;
            ok = warp_all_ok(mbar_wait(&meta->item_full[it], (j / kItemSlots) & 1, abort_flag, p.status));
            if (!ok) break;
            const int4 rec = meta->slot[it].rec;
            if (rec.w < 0) break;
            const int hk = rec.x % p.Hkv, b = rec.x / p.Hkv, s = rec.y, n = rec.w;
            const bool cached = p.batch <= kInvCuCache;
            const int q0 = cached ? s_cu[b] : __ldg(&p.cu_q[b]);
            const int sq = (cached ? s_cu[b + 1] : __ldg(&p.cu_q[b + 1])) - q0;
            const int sk = cached ? s_cu[kInvCuCache + 1 + b + 1] - s_cu[kInvCuCache + 1 + b]
                                  : __ldg(&p.cu_k[b + 1]) - __ldg(&p.cu_k[b]);
            const int tok = r / p.G, gg = r - tok * p.G;
            const bool valid = tok < n;
            int64_t t = 0;
            int kslot = 0, lo = 0, hi = -1;
            if (valid) {
                const int e = meta->slot[it].tok[tok];
                t = e >> 7;
                kslot = e & 127;
                const int i = (int)(t - q0), delta = sk - sq;
                lo = 0;
                hi = sk - 1;
                if (p.wl >= 0) lo = max(lo, i + delta - p.wl);
                if (p.causal) hi = min(hi, i + delta);
                if (p.wr >= 0) hi = min(hi, i + delta + p.wr);
            }
            ok = warp_all_ok(mbar_wait(&meta->s_full[grp], ph, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            float x[BS];
            {
                uint32_t raw[BS];
                tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(raw));
                if constexpr (BS == 64) tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < BS; ++e) x[e] = __uint_as_float(raw[e]);
            }
            const int kb = s * BS;
            if (valid && !(kb >= lo && kb + BS - 1 <= hi)) {  // the block straddles the row's edge
#pragma unroll
                for (int c = 0; c < BS; ++c) {
                    const int key = kb + c;
                    x[c] = (key >= lo && key <= hi) ? x[c] : -INFINITY;
                }
            }
            const float m = valid ? row_max3<BS>(x) * p.scale_log2 : -INFINITY;
            const float m_use = m == -INFINITY ? 0.f : m;
            uint32_t packed[BS / 2];
            const float l = scores_to_p<BS>(x, valid ? p.scale_log2 : 0.f, valid ? -m_use : -INFINITY, packed);
            if constexpr (BS == 64) {
                tmem_st32(tS, packed);
            } else {
                tmem_st16(tS, packed);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&meta->p_full[grp]);

            // Epilogue: the row's normalised partial and its (max, sum).
            ok = warp_all_ok(mbar_wait(&meta->pv_done[grp], ph, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            const int h = hk * p.G + gg;
            const int64_t pslot = (t * p.Hq + h) * p.topk + kslot;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            // The warp's 32 rows go out 32 columns (64 bytes of bf16) at a time through its staging
            // buffer: each lane writes its row's four 16-byte segments, then lane l stores segment
            // l % 4 of row 8i + l / 4, so one store instruction writes whole 64-byte row pieces.
            // Segment j of row r sits at (j + r / 2) % 4, which keeps both sides bank-conflict free.
            int64_t ps_i[4];
            bool vr_i[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int rr = 8 * i + (lane >> 2);
                ps_i[i] = __shfl_sync(0xffffffffu, (long long)pslot, rr);
                vr_i[i] = __shfl_sync(0xffffffffu, valid ? 1 : 0, rr) != 0;
            }
            // one 32-column chunk c of the row: pack, stage, store
            auto put_chunk = [&](int c, const uint32_t(&o)[32]) {
                uint32_t wv[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                __syncwarp();  // the previous chunk's segments have been read out
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    stg[lane * 4 + ((e + (lane >> 1)) & 3)] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int rr = 8 * i + (lane >> 2), seg = lane & 3;
                    const uint4 v = stg[rr * 4 + ((seg + (rr >> 1)) & 3)];
                    if (vr_i[i]) reinterpret_cast<uint4 *>(p.po + ps_i[i] * D + c * 32)[seg] = v;
                }
            };
#pragma unroll 1
            for (int c = 0; c < D / 32; c += 2) {  // two chunks per TMEM wait
                uint32_t oa[32], ob[32];
                tmem_ld32(tO + c * 32, oa);
                tmem_ld32(tO + (c + 1) * 32, ob);
                tmem_wait_ld();
                if (c + 2 >= D / 32) {  // O is in registers: the group's next P.V may overwrite it
                    tc_fence_before();
                    mbar_arrive(&meta->o_free[grp]);
                }
                put_chunk(c, oa);
                put_chunk(c + 1, ob);
            }
            if (valid) p.pml[pslot] = make_float2(m, l);

            mbar_arrive(&meta->item_free[it]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Merge of the block-major partials, one warp per row (token, head) of a tile that went block-major:
// M = max m_k, L = sum l_k 2^(m_k - M), out = sum (l_k 2^(m_k - M) / L) o_k, lse = (M + log2 L) ln 2
// over the row's partials: its block-major ones (the first slots of its range) and, when the tile
// has dense blocks, the query-major kernel's partial over them, left in out / lse (taken as
// (m, l) = (lse in base 2, 1)).  Lanes cover the head dimension in 16-byte chunks and split the
// partials between them; each lane loads a batch of its partials at once (independent loads in
// flight), folds them into a running max / sum / weighted chunk, and the lanes sharing a chunk
// combine at the end.  The partials are read once, with streaming loads (they are not reused).
// Three CTAs per SM (80 registers): the loads in flight are what this kernel's speed rests on.
constexpr int kMergeWarps = 8;
constexpr int kMergeBatch = 8;  // partials each lane loads before folding them in

template <int D>
__global__ void __launch_bounds__(32 * kMergeWarps, 3) fwd_merge_kernel(const FwdAttendParams p)
{
    constexpr int kChunks = D / 8;       // 16-byte chunks of a row
    constexpr int kSplit = 32 / kChunks; // lanes sharing a chunk, each over every kSplit-th partial
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    grid_dep_wait();
    // One CTA per query tile (the tile numbering of the other prefill kernels); only the tiles the
    // plan sent block-major (ucnt = -1) have partials to merge.
    const int tile = blockIdx.x;
    if (__ldcg(&p.ctrl->item_total) == 0) return;  // every row was written by the query-major kernel
    if (__ldcg(&p.ucnt[tile]) != -1) return;
    const int hk = tile % p.Hkv;
    const int rest = tile / p.Hkv;
    const int b = rest % p.batch;
    const int qt = p.nqt - 1 - rest / p.batch;
    const int q0 = p.cu_q[b], sq = p.cu_q[b + 1] - q0;
    const int tok0 = qt * p.Tq;
    const int ntok = min(p.Tq, sq - tok0);
    if (ntok <= 0) return;
    const int nrows = ntok * p.G;
    // the selection counts of this warp's rows (row e = warp + kMergeWarps * i, i = lane), read at once
    const int e_l = warp + kMergeWarps * lane;
    const int64_t tl_l = (int64_t)q0 + tok0 + e_l / p.G;
    const int cnt_l = e_l < nrows ? __ldg(&p.cnt[tl_l * p.Hkv + hk]) : 0;
    // entries of dense blocks (their partial is the query-major kernel's, in out / lse)
    const uint32_t dm_l = e_l < nrows && p.dmask ? __ldg(&p.dmask[tl_l * p.Hkv + hk]) : 0u;
    const int c = lane % kChunks, kq = lane / kChunks;
    for (int i = 0; warp + kMergeWarps * i < nrows; ++i) {
        const int e = warp + kMergeWarps * i;
        const int cnt = __shfl_sync(0xffffffffu, cnt_l, i);
        const uint32_t dm = __shfl_sync(0xffffffffu, dm_l, i);
        // a row that keeps no key, or keeps only dense blocks: the query-major kernel wrote it
        if (cnt == __popc(dm)) continue;
        const int tt = e / p.G, g = e - tt * p.G;
        const int64_t t = (int64_t)q0 + tok0 + tt;
        const int h = hk * p.G + g;
        const int64_t base = (t * p.Hq + h) * p.topk;
        // Lane (kq, c) merges partials kq, kq + kSplit, ... of chunk c: a batch of their (m, l) and
        // 16-byte chunks is loaded at once, then folded into a running (max, sum, weighted chunk).
        // With dense blocks, lanes kq = 0 start from the query-major partial: normalised in out, its
        // log-sum-exp in lse (as (m, l) = (lse in base 2, 1)).
        float Mx = -INFINITY, Ls = 0.f, acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        // (its two loads go out with the first batch of partials, not ahead of them)
        // The block-major partials fill the row's first nk slots (the scatter numbers a row's entries
        // that are not dense consecutively).
        bool qdone = !(dm != 0u && kq == 0);
        const int nk = cnt - __popc(dm);
        for (int k0 = kq; k0 < nk; k0 += kSplit * kMergeBatch) {
            float2 ml[kMergeBatch];
            uint4 v[kMergeBatch];
#pragma unroll
            for (int i = 0; i < kMergeBatch; ++i) {
                const int k = k0 + i * kSplit;
                ml[i] = k < nk ? __ldcs(&p.pml[base + k]) : make_float2(-INFINITY, 0.f);
                v[i] = k < nk ? __ldcs(reinterpret_cast<const uint4 *>(p.po + (base + k) * D) + c) : make_uint4(0u, 0u, 0u, 0u);
            }
            if (!qdone) {  // the query-major partial as (m, l) = (lse in base 2, 1), normalised chunk vq
                qdone = true;
                const float lq = p.lse[(int64_t)h * p.total_q + t];
                const uint4 vq = reinterpret_cast<const uint4 *>(p.out + (t * p.Hq + h) * D)[c];
                if (lq != -INFINITY) {
                    Mx = lq * 1.4426950408889634f;
                    Ls = 1.f;
                    const uint32_t vv[4] = {vq.x, vq.y, vq.z, vq.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vv[e]));
                        acc[2 * e] = x.x;
                        acc[2 * e + 1] = x.y;
                    }
                }
            }
            float bm = Mx;
#pragma unroll
            for (int i = 0; i < kMergeBatch; ++i)
                if (ml[i].y > 0.f) bm = fmaxf(bm, ml[i].x);
            if (bm == -INFINITY) continue;
            const float f = Mx == -INFINITY ? 0.f : ex2(Mx - bm);
            Ls *= f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] *= f;
            Mx = bm;
#pragma unroll
            for (int i = 0; i < kMergeBatch; ++i) {
                const float w = ml[i].y > 0.f ? ml[i].y * ex2(ml[i].x - bm) : 0.f;
                Ls += w;
                const uint32_t vv[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vv[e]));
                    acc[2 * e] = fmaf(w, x.x, acc[2 * e]);
                    acc[2 * e + 1] = fmaf(w, x.y, acc[2 * e + 1]);
                }
            }
        }
        // combine the kSplit lanes of each chunk (lanes c, c + kChunks, ...)
        float M = Mx;
#pragma unroll
        for (int o = kChunks; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float f = Mx == -INFINITY ? 0.f : ex2(Mx - M);
        float L = Ls * f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= f;
#pragma unroll
        for (int o = kChunks; o < 32; o <<= 1) {
            L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
        }
        const float invL = L > 0.f ? 1.f / L : 0.f;
        if (kq == 0) {
            uint4 w4;
            w4.x = pack_bf16x2(acc[0] * invL, acc[1] * invL);
            w4.y = pack_bf16x2(acc[2] * invL, acc[3] * invL);
            w4.z = pack_bf16x2(acc[4] * invL, acc[5] * invL);
            w4.w = pack_bf16x2(acc[6] * invL, acc[7] * invL);
            reinterpret_cast<uint4 *>(p.out + (t * p.Hq + h) * D)[c] = w4;
        }
        if (lane == 0) p.lse[(int64_t)h * p.total_q + t] = L > 0.f ? (M + log2f(L)) * kLn2i : -INFINITY;
    }
}

template <int D, int BS>
size_t inv_smem_bytes()
{
    static_assert(sizeof(InvMeta) <= 4608, "InvMeta must fit below the staging buffers");
    return 1024 + InvCfg<D, BS>::kOffCu + 2 * (kInvCuCache + 1) * 4;
}

template <int D, int BS>
cudaError_t launch_inv_t(const FwdGeom &g, const FwdAttendParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                         const CUtensorMap &tv, cudaStream_t st)
{
    const size_t smem = inv_smem_bytes<D, BS>();
    const cudaError_t e = ensure_smem_for(fwd_attend_inv_kernel<D, BS>, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const cudaError_t le =
        launch_kernel(fwd_attend_inv_kernel<D, BS>, dim3(sms), dim3(kInvThreadsAttn), smem, st, true, tq, tk, tv, p);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

}  // namespace

size_t fwd_attend_inv_smem_bytes(const FwdGeom &g)
{
    if (g.d == 64) return g.bs == 32 ? inv_smem_bytes<64, 32>() : inv_smem_bytes<64, 64>();
    return g.bs == 32 ? inv_smem_bytes<128, 32>() : inv_smem_bytes<128, 64>();
}

cudaError_t launch_fwd_merge(const FwdGeom &g, const FwdAttendParams &p, cudaStream_t st)
{
    const unsigned grid = (unsigned)g.tiles;
    if (g.d == 64) return launch_kernel(fwd_merge_kernel<64>, dim3(grid), dim3(32 * kMergeWarps), 0, st, true, p);
    return launch_kernel(fwd_merge_kernel<128>, dim3(grid), dim3(32 * kMergeWarps), 0, st, true, p);
}

cudaError_t launch_fwd_attend_inv(const FwdGeom &g, const FwdAttendParams &p, const CUtensorMap &tq,
                                  const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st)
{
    if (g.d == 64) return g.bs == 32 ? launch_inv_t<64, 32>(g, p, tq, tk, tv, st) : launch_inv_t<64, 64>(g, p, tq, tk, tv, st);
    return g.bs == 32 ? launch_inv_t<128, 32>(g, p, tq, tk, tv, st) : launch_inv_t<128, 64>(g, p, tq, tk, tv, st);
}

}  // namespace sfa
