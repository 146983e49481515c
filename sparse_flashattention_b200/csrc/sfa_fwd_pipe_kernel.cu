// Prefill attention kernel, pipelined query-major schedule (sm_100a).
//
// Persistent CTAs, two per SM, each computing one query tile at a time: Tq consecutive tokens of
// one sequence times the G query heads that share one kv head (Tq*G <= 128 rows, the M dimension
// of one tcgen05 MMA).  The CTA walks the ascending union of its rows' selected blocks (built by
// the prep kernel); per block s:
//
//   producer warp   TMA-loads K and V rows [s*bs, s*bs+bs) of the kv head into two-stage
//                   shared-memory rings (128-byte swizzle).  It fetches the next tile, stages
//                   its union and issues its Q and K/V loads while the current tile finishes,
//                   so a tile switch costs about one epilogue instead of a pipeline drain.
//   MMA warp        one thread issues tcgen05.mma: S = Q K^T into one of two TMEM score buffers
//                   and O += P V into the TMEM output accumulator, each as soon as its inputs
//                   are ready (PV of a block never waits for a later block's loads).  The thread
//                   keeps its loop to the bare issue work: the tensor core queue is shallow, so
//                   instructions between MMA groups show up as tensor-core idle time.
//   softmax warps   4 warps, one thread per row: read S from TMEM, apply the row's mask (block
//                   not selected by this row, bottom-right causal limit, window), keep the
//                   running max and sum in fp32 (base-2 domain), write P = 2^(s - m) as bf16 over
//                   its own scores in TMEM (the A operand of the PV MMA), rescale O in TMEM when
//                   the running max grows by more than 2^8, and write out / lse.
//
// TMEM: two score buffers of bs columns and an output accumulator of d columns (256 columns for
// d = 128, bs = 64), so two CTAs share an SM and each one's MMAs fill the other's waits.
//
// The method is the FlashAttention tiling with online softmax applied to the gathered blocks
// only, as the Ascend "Sparse FlashAttention" article describes the fused SFA operator; the
// mask/GQA/LSE semantics are those of the flash-attention-npu FlashAttention v2 docstrings.
//
// Every wait is bounded (sfa_device.cuh): on a timeout the CTA records SFA_DEV_TIMEOUT, drains
// its in-flight copies and MMAs, frees TMEM and exits.
#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kQThreads = 224;  // warp 0 producer, warp 1 MMA, warps 2..5 softmax / epilogue, warp 6 index
constexpr int kQStages = 2;     // K and V ring depth (two CTAs per SM bound the shared memory)
constexpr float kQRescaleLog2 = 8.0f;
constexpr float kQLn2 = 0.6931471805599453f;
constexpr size_t kQMaxSmem = 113 * 1024;  // two CTAs per SM

template <int D, int BS>
struct QCfg {
    static constexpr int kQBytes = 128 * D * 2;  // the tile's Q
    static constexpr int kKVBytes = BS * D * 2;  // one K (or V) block
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffV = kOffK + kQStages * kKVBytes;
    static constexpr int kOffMeta = kOffV + kQStages * kKVBytes;
    static constexpr int kTmemCols = (2 * BS + D) <= 128 ? 128 : 256;
    static constexpr int kColO = 2 * BS;
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, BS, false);
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
};

struct TileInfo {
    int done;  // no tile left: every role leaves its loop
    int nU;    // union blocks (< 0: a block-major tile, whose rows another kernel computes)
    int dense; // a block-major tile whose dense blocks run here: the union is those blocks, a row's
               // selection of them is a bit mask, and out / lse receive a partial the merge combines
    int b, hk, q0, sq, k0, sk, tok0, ntok;
    int blo;   // window mode: the union is blocks blo, blo+1, ..., blo+nU-1
};

// How a tile's blocks and each row's selection are known (sfa_internal.h): kPipePrep, canonical
// lists and union written by the prep kernel; kPipeFused, the index warp canonicalizes the raw
// selections itself; kPipeWindow, dense attention under the causal / window mask (every block that
// holds a key of the row's window is selected; no selection lists).
constexpr int kModePrep = kPipePrep, kModeFused = kPipeFused, kModeWindow = kPipeWindow;

struct QMeta {
    uint64_t q_full, q_empty;
    uint64_t k_full[kQStages], k_empty[kQStages];  // K of a block is free once its S MMA is done,
    uint64_t v_full[kQStages], v_empty[kQStages];  // V once its PV MMA is done
    uint64_t s_full[2], p_full[2], pv_done[2];
    uint64_t o_free;                    // the epilogue has read O
    uint64_t meta_full[2], meta_empty[2];  // tile metadata double buffer
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    TileInfo info[2];
};

// Shared memory after the Q tile and the K/V rings: the barriers, two copies of a tile's union
// ([2][umax]) and, in the fused mode, two copies of the tile's canonical lists ([2][Tq][topk]),
// their counts ([2][Tq]) and the union bitmap (one bit per key block).
struct QLayout {
    size_t off_union, off_lists, off_cnts, off_bm, bytes;
};

template <int D, int BS>
__host__ __device__ inline QLayout pipe_layout(int mode, int umax, int Tq, int topk, int nblk_max)
{
    QLayout l;
    const bool fused = mode == kModeFused;
    l.off_union = QCfg<D, BS>::kOffMeta + ((sizeof(QMeta) + 15) & ~size_t(15));
    l.off_lists = l.off_union + (mode == kModeWindow ? 0 : (size_t)2 * umax * 4);
    l.off_cnts = l.off_lists + (fused ? (size_t)2 * Tq * topk * 4 : 0);
    l.off_bm = l.off_cnts + (fused ? (size_t)2 * Tq * 4 : 0);
    l.bytes = l.off_bm + (fused ? (size_t)(nblk_max + 31) / 32 * 4 : 0);
    return l;
}

template <int D, int BS, int MODE>
__global__ void __launch_bounds__(kQThreads, 2)
    fwd_attend_pipe_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                           const __grid_constant__ CUtensorMap tmv, const FwdAttendParams p)
{
    using C = QCfg<D, BS>;
    constexpr bool FUSED = MODE == kModeFused;
    constexpr bool WIN = MODE == kModeWindow;
    extern __shared__ uint8_t pipe_smem_raw[];
    uint8_t *smem =
        reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(pipe_smem_raw) + 1023) & ~uintptr_t(1023));
    const int U = p.umax;
    const QLayout L = pipe_layout<D, BS>(MODE, U, p.Tq, p.topk, p.nblk_max);
    QMeta *meta = reinterpret_cast<QMeta *>(smem + C::kOffMeta);
    int *s_union = reinterpret_cast<int *>(smem + L.off_union);   // [2][U]
    int *s_lists = reinterpret_cast<int *>(smem + L.off_lists);   // fused: [2][Tq][topk]
    int *s_cnts = reinterpret_cast<int *>(smem + L.off_cnts);     // fused: [2][Tq]
    uint32_t *s_bm = reinterpret_cast<uint32_t *>(smem + L.off_bm);  // fused: union bitmap
    uint8_t *sQ = smem;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned full = 0xffffffffu;

    if (threadIdx.x == 0) {
        mbar_init(&meta->q_full, 1);
        mbar_init(&meta->q_empty, 1);
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&meta->k_full[s], 1);
            mbar_init(&meta->k_empty[s], 1);
            mbar_init(&meta->v_full[s], 1);
            mbar_init(&meta->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&meta->s_full[s], 1);
            mbar_init(&meta->p_full[s], 128);
            mbar_init(&meta->pv_done[s], 1);
            mbar_init(&meta->meta_full[s], 32);  // every index-warp lane arrives after its writes
            mbar_init(&meta->meta_empty[s], 6);  // the 4 softmax warps, the MMA thread, the producer
        }
        mbar_init(&meta->o_free, 128);
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
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
    }
    grid_dep_wait();  // everything above ran while the prep kernels were finishing

    // Tile k uses metadata buffer k & 1; barrier phases of the rings run on a per-CTA count of
    // blocks (jg), so the pipeline carries over from tile to tile.
    if (warp == 6) {
        // ------------------------------------------------------------------ index warp
        // Runs a tile ahead of the producer: takes the next tile from the counter, builds (fused
        // mode) or copies its block union and canonical lists into metadata buffer k & 1, and
        // publishes them.
        int k = 0;
        bool ok = true;
        while (ok) {
            const int m = k & 1;
            if (k >= 2) ok = mbar_wait(&meta->meta_empty[m], ((k >> 1) - 1) & 1, abort_flag, p.status);
            ok = __all_sync(full, ok);
            if (!ok) break;
            TileInfo &ti = meta->info[m];
            int *uni = s_union + m * U;
            // Next tile holding any query row: tiles past the end of shorter sequences are skipped
            // here, without a trip through the pipeline.
            int tile, hk, b, qt, q0, sq;
            while (true) {
                tile = 0;
                if (lane == 0) tile = atomicAdd(p.tile_counter, 1);
                tile = __shfl_sync(full, tile, 0);
                if (tile >= p.tiles) break;
                hk = tile % p.Hkv;
                const int rest = tile / p.Hkv;
                b = rest % p.batch;
                qt = p.nqt - 1 - rest / p.batch;  // tiles deepest into their sequences first
                q0 = p.cu_q[b];
                sq = p.cu_q[b + 1] - q0;
                if (qt * p.Tq < sq) break;
            }
            if (tile >= p.tiles) {
                if (lane == 0) ti.done = 1;
                mbar_arrive(&meta->meta_full[m]);
                break;
            }
            const int k0 = p.cu_k[b], sk = p.cu_k[b + 1] - k0;
            const int tok0 = qt * p.Tq;
            const int ntok = min(p.Tq, sq - tok0);
            int nU, blo = 0, dense = 0;
            if constexpr (WIN) {
                // Rows' key windows [lo(i), hi(i)] move right with i, so the tile's blocks are the
                // contiguous range from the first row's lo to the last row's hi.
                int nblk = (sk + BS - 1) / BS;
                if (sq > p.max_sq || nblk > p.nblk_max) {  // lengths beyond the caller's max_seqlen bounds
                    if (lane == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
                    nblk = min(nblk, p.nblk_max);
                }
                // With per-head windows, the range covers every head's window of the kv head
                // (all of them hold the last row's diagonal key, so their union has no gap).
                const int delta = sk - sq, i0 = tok0, i1 = tok0 + ntok - 1;
                const int cap = min(sk, nblk * BS) - 1;
                int lo = 0x7fffffff, hi = -1;
                const int nh = (p.wl_head || p.wr_head) ? p.G : 1;
                for (int g = lane; g < nh; g += 32) {
                    const int h = hk * p.G + g;
                    const int wl = p.wl_head ? __ldg(&p.wl_head[h]) : p.wl;
                    const int wr = p.wr_head ? __ldg(&p.wr_head[h]) : p.wr;
                    int l = 0, r = cap;
                    if (wl >= 0) l = max(l, i0 + delta - wl);
                    if (p.causal) r = min(r, i1 + delta);
                    if (wr >= 0) r = min(r, i1 + delta + wr);
                    if (r >= l) {
                        lo = min(lo, l);
                        hi = max(hi, r);
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    lo = min(lo, __shfl_xor_sync(full, lo, o));
                    hi = max(hi, __shfl_xor_sync(full, hi, o));
                }
                blo = hi >= lo ? lo / BS : 0;
                nU = hi >= lo ? hi / BS - blo + 1 : 0;
            } else if constexpr (FUSED) {
                // The tile's canonical lists (one token per lane at a time) and the ascending union
                // of their blocks, built here instead of by a prep kernel.
                int *lists = s_lists + m * p.Tq * p.topk;
                int *cnts = s_cnts + m * p.Tq;
                int nblk = (sk + BS - 1) / BS;
                if (sq > p.max_sq || nblk > p.nblk_max) {  // lengths beyond the caller's max_seqlen bounds
                    if (lane == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
                    nblk = min(nblk, p.nblk_max);
                }
                const int words = (nblk + 31) >> 5;
                for (int w = lane; w < words; w += 32) s_bm[w] = 0u;
                __syncwarp();
                bool bad = false;
                const int delta = sk - sq;
                for (int tt = lane; tt < ntok; tt += 32) {
                    const int i = tok0 + tt;
                    int lo = 0, hi = sk - 1;
                    if (p.wl >= 0) lo = max(lo, i + delta - p.wl);
                    if (p.causal) hi = min(hi, i + delta);
                    if (p.wr >= 0) hi = min(hi, i + delta + p.wr);
                    const int *raw = p.sel + ((int64_t)(q0 + i) * p.Hkv + hk) * p.topk;
                    int *dst = lists + tt * p.topk;
                    int cn;
                    if (p.topk <= 16) cn = canon_list_regs<16>(raw, p.topk, nblk, BS, sk, lo, hi, dst, 1, bad);
                    else if (p.topk <= 32) cn = canon_list_regs<32>(raw, p.topk, nblk, BS, sk, lo, hi, dst, 1, bad);
                    else cn = canon_list_insert(raw, p.topk, nblk, BS, sk, lo, hi, dst, 1, bad);
                    cnts[tt] = cn;
                    for (int e = 0; e < cn; ++e) atomicOr(&s_bm[dst[e] >> 5], 1u << (dst[e] & 31));
                }
                if (__any_sync(full, bad) && lane == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_INDEX);
                __syncwarp();
                // Bitmap -> ascending ids: 32 words at a time, word w of a chunk to lane w, a warp scan
                // of the bit counts places each word's ids.
                int total = 0;
                for (int c0 = 0; c0 < words; c0 += 32) {
                    const int w = c0 + lane;
                    uint32_t bits = w < words ? s_bm[w] : 0u;
                    const int c = __popc(bits);
                    int incl = c;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(full, incl, o);
                        if (lane >= o) incl += y;
                    }
                    int pos = total + incl - c;
                    while (bits) {
                        const int bit = __ffs(bits) - 1;
                        bits &= bits - 1;
                        uni[pos++] = w * 32 + bit;
                    }
                    total += __shfl_sync(full, incl, 31);
                }
                nU = total;
            } else {
                nU = p.ucnt[tile];
                if (nU < 0 && p.duni) {  // a block-major tile: its dense blocks are this kernel's
                    nU = p.dcnt[tile];
                    dense = 1;
                    for (int i = lane; i < nU; i += 32) uni[i] = p.duni[(int64_t)tile * kDenseMax + i];
                } else {
                    for (int i = lane; i < nU; i += 32) uni[i] = p.uni[(int64_t)tile * U + i];
                }
            }
            if (lane == 0) {
                ti.done = 0;
                ti.nU = nU;
                ti.dense = dense;
                ti.b = b;
                ti.hk = hk;
                ti.q0 = q0;
                ti.sq = sq;
                ti.k0 = k0;
                ti.sk = sk;
                ti.tok0 = tok0;
                ti.ntok = ntok;
                ti.blo = blo;
            }
            mbar_arrive(&meta->meta_full[m]);
            ++k;
        }
    } else if (warp == 0) {
        // ------------------------------------------------------------------ producer
        int k_st = 0, k_ph = 0, nk = 0, v_st = 0, v_ph = 0, nv = 0;  // ring stage, phase, loads issued
        int q_phases = 0;                                            // Q phases issued
        if (lane == 0) {
            int k = 0;
            bool ok = true;
            while (ok) {
                const int m = k & 1;
                ok = mbar_wait(&meta->meta_full[m], (k >> 1) & 1, abort_flag, p.status);
                if (!ok) break;
                const TileInfo &ti = meta->info[m];
                if (ti.done) break;
                const int *uni = s_union + m * U;
                const int n = max(ti.nU, 0), hk = ti.hk, q0 = ti.q0, k0 = ti.k0, tok0 = ti.tok0, blo = ti.blo;
                // Q, once the previous tile's score MMAs no longer read it (a box of Tq tokens x
                // G heads, Tq*G <= 128 rows).
                if (k >= 1) ok = mbar_wait(&meta->q_empty, (k - 1) & 1, abort_flag, p.status);
                if (ok) {
                    const uint32_t qbytes = n > 0 ? (uint32_t)D * (uint32_t)(p.G * p.Tq) * 2u : 0u;
                    mbar_arrive_expect_tx(&meta->q_full, qbytes);
                    if (n > 0)
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_3d(&tmq, &meta->q_full, sQ + c * (128 * 128), c * 64, hk * p.G, q0 + tok0);
                    q_phases = k + 1;
                }
                // K of block u+1 goes out ahead of V of block u: the score MMAs need only K.
                auto load_k = [&](int u) -> bool {
                    const int st = k_st;
                    if (nk >= kQStages && !mbar_wait(&meta->k_empty[st], k_ph ^ 1, abort_flag, p.status))
                        return false;
                    const int row = k0 + (WIN ? blo + u : uni[u]) * BS;
                    mbar_arrive_expect_tx(&meta->k_full[st], (uint32_t)C::kKVBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(&tmk, &meta->k_full[st], sK + st * C::kKVBytes + c * (BS * 128), c * 64, hk, row);
                    ++nk;
                    if (++k_st == kQStages) {
                        k_st = 0;
                        k_ph ^= 1;
                    }
                    return true;
                };
                auto load_v = [&](int u) -> bool {
                    const int st = v_st;
                    if (nv >= kQStages && !mbar_wait(&meta->v_empty[st], v_ph ^ 1, abort_flag, p.status))
                        return false;
                    const int row = k0 + (WIN ? blo + u : uni[u]) * BS;
                    mbar_arrive_expect_tx(&meta->v_full[st], (uint32_t)C::kKVBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(&tmv, &meta->v_full[st], sV + st * C::kKVBytes + c * (BS * 128), c * 64, hk, row);
                    ++nv;
                    if (++v_st == kQStages) {
                        v_st = 0;
                        v_ph ^= 1;
                    }
                    return true;
                };
                if (ok && n > 0) {
                    ok = load_k(0);
                    for (int u = 0; ok && u < n; ++u) {
                        if (u + 1 < n && !load_k(u + 1)) ok = false;
                        else if (!load_v(u)) ok = false;
                    }
                }
                if (!ok) break;
                mbar_arrive(&meta->meta_empty[m]);
                ++k;
            }
        }
        if (*abort_flag && lane == 0) {  // wind down: let every copy this CTA started land
            if (q_phases > 0) mbar_drain(&meta->q_full, (q_phases - 1) & 1);
            for (int st = 0; st < kQStages; ++st) {
                const int ck = nk > st ? (nk - st + kQStages - 1) / kQStages : 0;  // loads into this stage
                const int cv = nv > st ? (nv - st + kQStages - 1) / kQStages : 0;
                if (ck > 0) mbar_drain(&meta->k_full[st], (ck - 1) & 1);
                if (cv > 0) mbar_drain(&meta->v_full[st], (cv - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tO = tmem + C::kColO;
            // Descriptor bases: adding (byte offset >> 4) moves the 14-bit start address field
            // (every shared-memory address here is below 256 KB, so the field does not carry).
            const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dV0 = sdesc_sw128(smem_u32(sV), BS * 128, 1024);
            int k = 0, jg0 = 0;
            int s_st = 0, s_ph = 0, p_st = 0, p_ph = 0;  // ring stage / phase of the next S and PV
            bool ok = true;
            while (ok) {
                const int m = k & 1;
                ok = mbar_wait(&meta->meta_full[m], (k >> 1) & 1, abort_flag, p.status);
                if (!ok) break;
                const TileInfo &ti = meta->info[m];
                if (ti.done) break;
                const int n = max(ti.nU, 0);
                ok = mbar_wait(&meta->q_full, k & 1, abort_flag, p.status);
                if (!ok) break;
                // S of block u goes out once K u has landed and PV u-2 was issued (S u overwrites
                // the score buffer PV u-2 reads; one thread's MMAs run in issue order); PV u once
                // P u and V u are ready.  The tile's first PV overwrites O, so it also waits until
                // the previous tile's epilogue has read it.
                bool ofree = (k == 0);
                int ns = 0, np = 0;
                if (n == 0) umma_commit(&meta->q_empty);
                uint64_t idle_since = 0;
                int spins = 0;  // failed polls since the last issue; the clock is read only now and then
                while (ok && np < n) {
                    bool progressed = false;
                    if (ns < n && ns <= np + 1) {
                        const int jg = jg0 + ns, st = s_st;
                        if (mbar_test(smem_u32(&meta->k_full[st]), s_ph)) {
                            tc_fence_after();
                            const uint32_t tS = tmem + (jg & 1) * BS;
                            const uint64_t dK = dK0 + (uint64_t)((st * C::kKVBytes) >> 4);
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks)
                                umma_bf16(tS, dQ + (uint64_t)(((ks >> 2) * (128 * 128) + (ks & 3) * 32) >> 4),
                                          dK + (uint64_t)(((ks >> 2) * (BS * 128) + (ks & 3) * 32) >> 4), C::kIdescS,
                                          ks > 0 ? 1u : 0u);
                            umma_commit(&meta->s_full[jg & 1]);
                            umma_commit(&meta->k_empty[st]);
                            ++ns;
                            if (++s_st == kQStages) {
                                s_st = 0;
                                s_ph ^= 1;
                            }
                            if (ns == n) umma_commit(&meta->q_empty);  // the tile no longer reads Q
                            progressed = true;
                        }
                    }
                    if (np < ns) {
                        const int ig = jg0 + np, st = p_st;
                        if (mbar_test(smem_u32(&meta->p_full[ig & 1]), (ig >> 1) & 1) &&
                            mbar_test(smem_u32(&meta->v_full[st]), p_ph) &&
                            (ofree || mbar_test(smem_u32(&meta->o_free), (k - 1) & 1))) {
                            ofree = true;
                            tc_fence_after();
                            const uint64_t dV = dV0 + (uint64_t)((st * C::kKVBytes) >> 4);
#pragma unroll
                            for (int ks = 0; ks < BS / 16; ++ks)  // P (bf16) sits in the first BS/2 columns
                                umma_bf16_tmem_a(tO, tmem + (ig & 1) * BS + ks * 8, dV + (uint64_t)((ks * 16 * 128) >> 4),
                                                 C::kIdescPV, (np > 0 || ks > 0) ? 1u : 0u);
                            umma_commit(&meta->pv_done[ig & 1]);
                            umma_commit(&meta->v_empty[st]);
                            ++np;
                            if (++p_st == kQStages) {
                                p_st = 0;
                                p_ph ^= 1;
                            }
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
            if (!ok) {  // wind down: wait for the MMAs already issued
                umma_commit(&meta->drain);
                mbar_drain(&meta->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const int r = quad * 32 + lane;
        const int gt = (warp - 2) * 32 + lane;  // thread index within the 128
        const int tok = r / p.G, g = r % p.G;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t tO = lane_base + C::kColO;
        int k = 0, jg0 = 0;
        bool ok = true;
        while (ok) {
            const int m = k & 1;
            ok = warp_all_ok(mbar_wait(&meta->meta_full[m], (k >> 1) & 1, abort_flag, p.status));
            if (!ok) break;
            const TileInfo &ti = meta->info[m];
            if (ti.done) break;
            const int nU = ti.nU, n = max(nU, 0), ntok = ti.ntok, tok0 = ti.tok0;
            const int q0 = ti.q0, sq = ti.sq, sk = ti.sk, hk = ti.hk;
            const int *uni = s_union + m * U;
            if (nU < 0) {
                // The block-major kernel computes this tile's rows; only rows that keep no key at all
                // (no partial will ever arrive for them) are written here: output 0, lse -inf.
                for (int e = gt; e < ntok * p.G; e += 128) {
                    const int tt = e / p.G, gg = e - tt * p.G;
                    const int64_t t = (int64_t)q0 + tok0 + tt;
                    if (p.cnt[t * p.Hkv + hk] != 0) continue;
                    const int h = hk * p.G + gg;
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out + (t * p.Hq + h) * D);
                    for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
                    p.lse[(int64_t)h * p.total_q + t] = -INFINITY;
                }
            }
            const bool row_valid = nU >= 0 && tok < ntok;
            const int i = tok0 + tok;
            const int delta = sk - sq;
            // the row's window (per query head in the window mode when the caller gives per-head windows)
            const int wl = WIN && p.wl_head ? __ldg(&p.wl_head[hk * p.G + g]) : p.wl;
            const int wr = WIN && p.wr_head ? __ldg(&p.wr_head[hk * p.G + g]) : p.wr;
            int lo = 0, hi = sk - 1;
            if (wl >= 0) lo = max(lo, i + delta - wl);
            if (p.causal) hi = min(hi, i + delta);
            if (wr >= 0) hi = min(hi, i + delta + wr);
            // This row's canonical (ascending) block list: in shared memory (fused mode), else read
            // from the prep kernel's output in global memory one entry ahead of its use.
            const int64_t t = (int64_t)q0 + i;
            const int *mylist = s_lists + (m * p.Tq + (row_valid ? tok : 0)) * p.topk;
            const int32_t *gl = p.sel_c + (row_valid && MODE == kModePrep ? (t * p.Hkv + hk) * p.topk : 0);
            const bool dense = !WIN && !FUSED && ti.dense;
            const uint32_t dsel = dense && row_valid ? __ldg(&p.dsel[t * p.Hkv + hk]) : 0u;
            const int mycnt = !row_valid || WIN || dense ? 0 : FUSED ? s_cnts[m * p.Tq + tok] : p.cnt[t * p.Hkv + hk];
            int nxt = (MODE == kModePrep && mycnt > 0) ? gl[0] : -1;
            int ptr = 0;
            float m_run = -INFINITY;  // running max of s*scale*log2e
            float l_run = 0.f;

            for (int j = 0; j < n; ++j) {
                const int jg = jg0 + j;
                const int s = WIN ? ti.blo + j : uni[j];
                bool selected;
                if constexpr (WIN) {
                    selected = row_valid && s * BS <= hi && s * BS + BS - 1 >= lo;
                } else if constexpr (FUSED) {
                    selected = ptr < mycnt && mylist[ptr] == s;
                    if (selected) ++ptr;
                } else if (dense) {
                    selected = (dsel >> j) & 1u;
                } else {
                    selected = nxt == s;
                    if (selected) {
                        ++ptr;
                        nxt = ptr < mycnt ? gl[ptr] : -1;
                    }
                }
                ok = warp_all_ok(mbar_wait(&meta->s_full[jg & 1], (jg >> 1) & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                const uint32_t tS = lane_base + (jg & 1) * BS;
                if (!__any_sync(full, selected)) {
                    // None of this warp's 32 rows selected the block: their P is zero, their running
                    // max and sum do not change, and the scores need not be read.
                    uint32_t zero[BS / 2];
#pragma unroll
                    for (int e = 0; e < BS / 2; ++e) zero[e] = 0u;
                    if constexpr (BS == 64) {
                        tmem_st32(tS, zero);
                    } else {
                        tmem_st16(tS, zero);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&meta->p_full[jg & 1]);
                    continue;
                }
                float xs[BS];
                {
                    uint32_t raw[BS];
                    tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(raw));
                    if constexpr (BS == 64) tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32));
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < BS; ++e) xs[e] = __uint_as_float(raw[e]);
                }
                // Rows that did not select this block contribute nothing (handled arithmetically
                // below); selected rows are masked element by element only where the block
                // straddles their causal / window edge.
                const int kb = s * BS;
                if (selected && !(kb >= lo && kb + BS - 1 <= hi)) {
#pragma unroll
                    for (int c = 0; c < BS; ++c) {
                        const int key = kb + c;
                        xs[c] = (key >= lo && key <= hi) ? xs[c] : -INFINITY;
                    }
                }
                const float mx = selected ? row_max3<BS>(xs) : -INFINITY;
                const float m_new = mx * p.scale_log2;
                const bool need = m_new > m_run + kQRescaleLog2;
                // O must be rescaled only for rows whose earlier blocks contributed (m_run finite);
                // a row's O is exactly 0 until its first kept key.
                const bool need_o = need && m_run != -INFINITY;
                float factor = 1.f;
                if (need) {
                    factor = m_run == -INFINITY ? 0.f : ex2(m_run - m_new);
                    m_run = m_new;
                    l_run *= factor;
                }
                if (j > 0 && __any_sync(full, need_o)) {
                    const int pg = jg - 1;
                    ok = warp_all_ok(mbar_wait(&meta->pv_done[pg & 1], (pg >> 1) & 1, abort_flag, p.status));
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
                l_run += scores_to_p<BS>(xs, selected ? p.scale_log2 : 0.f, selected ? -m_use : -INFINITY, packed);
                // P overwrites the first BS/2 columns of its own score buffer (already in registers).
                // S of block jg completing implies PV jg-2, which read the previous P there, has too.
                if constexpr (BS == 64) {
                    tmem_st32(tS, packed);
                } else {
                    tmem_st16(tS, packed);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&meta->p_full[jg & 1]);
            }
            if (!ok) break;

            // ------------------------------------------------------------ epilogue
            if (nU >= 0 && ntok > 0) {
                if (n > 0) {
                    const int lg = jg0 + n - 1;
                    ok = warp_all_ok(mbar_wait(&meta->pv_done[lg & 1], (lg >> 1) & 1, abort_flag, p.status));
                    if (!ok) break;
                    tc_fence_after();
                }
                const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
                const int h = hk * p.G + g;
                __nv_bfloat16 *orow = p.out + (t * p.Hq + h) * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    if (n > 0) {
                        tmem_ld32(tO + c * 32, o);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = 0u;
                    }
                    if (row_valid) {
                        uint32_t wv[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
                    }
                }
                if (row_valid)
                    p.lse[(int64_t)h * p.total_q + t] = l_run > 0.f ? (m_run + log2f(l_run)) * kQLn2 : -INFINITY;
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

template <int D, int BS, int MODE>
cudaError_t launch_pipe_t(const FwdAttendParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                          cudaStream_t st)
{
    const size_t smem = 1024 + pipe_layout<D, BS>(MODE, p.umax, p.Tq, p.topk, p.nblk_max).bytes;
    const cudaError_t e = ensure_smem_for(fwd_attend_pipe_kernel<D, BS, MODE>, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = p.tiles < 2 * sms ? p.tiles : 2 * sms;
    // The fused and window modes follow a memset of the tile counter, not a kernel: no early start.
    return launch_kernel(fwd_attend_pipe_kernel<D, BS, MODE>, dim3(grid > 0 ? grid : 1), dim3(kQThreads), smem, st,
                         MODE == kModePrep, tq, tk, tv, p);
}

template <int D, int BS>
cudaError_t launch_pipe_d(const FwdAttendParams &p, int mode, const CUtensorMap &tq, const CUtensorMap &tk,
                          const CUtensorMap &tv, cudaStream_t st)
{
    if (mode == kModeWindow) return launch_pipe_t<D, BS, kModeWindow>(p, tq, tk, tv, st);
    return mode == kModeFused ? launch_pipe_t<D, BS, kModeFused>(p, tq, tk, tv, st)
                              : launch_pipe_t<D, BS, kModePrep>(p, tq, tk, tv, st);
}

}  // namespace

bool fwd_pipe_fits(const FwdGeom &g, int mode)
{
    QLayout l;
    if (g.d == 64)
        l = g.bs == 32 ? pipe_layout<64, 32>(mode, g.umax, g.Tq, g.topk, g.nblk_max)
                       : pipe_layout<64, 64>(mode, g.umax, g.Tq, g.topk, g.nblk_max);
    else
        l = g.bs == 32 ? pipe_layout<128, 32>(mode, g.umax, g.Tq, g.topk, g.nblk_max)
                       : pipe_layout<128, 64>(mode, g.umax, g.Tq, g.topk, g.nblk_max);
    return 1024 + l.bytes <= kQMaxSmem;
}

cudaError_t launch_fwd_attend_pipe(const FwdGeom &g, const FwdAttendParams &p, int mode, const CUtensorMap &tq,
                                   const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st)
{
    if (g.d == 64)
        return g.bs == 32 ? launch_pipe_d<64, 32>(p, mode, tq, tk, tv, st) : launch_pipe_d<64, 64>(p, mode, tq, tk, tv, st);
    return g.bs == 32 ? launch_pipe_d<128, 32>(p, mode, tq, tk, tv, st) : launch_pipe_d<128, 64>(p, mode, tq, tk, tv, st);
}

}  // namespace sfa
