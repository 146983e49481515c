// Host side of libsfa.so: argument validation, workspace layout, TMA descriptor encoding and
// kernel launches for the C ABI declared in include/sfa.h.  Nothing here allocates device
// memory or synchronises with the device.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>

#include "sfa_internal.h"

using namespace sfa;

namespace sfa {

cudaError_t ensure_smem(const void *kernel, size_t bytes)
{
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> set;  // (kernel, device) -> limit set there
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    size_t &cur = set[{kernel, dev}];
    if (bytes <= cur) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) cur = bytes;
    return e;
}

}  // namespace sfa

namespace {

thread_local int g_last_launches = 0;

constexpr size_t kAlign = 256;

size_t align_up(size_t x)
{
    return (x + kAlign - 1) / kAlign * kAlign;
}

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Workspaces: every array in one starts on a multiple of kAlign from its base.
bool aligned256(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & (kAlign - 1)) == 0;
}

// ----------------------------------------------------------------------------------------
// Prefill geometry
// ----------------------------------------------------------------------------------------
int fwd_geometry(int batch, int max_sq, int max_sk, int total_q, int Hq, int Hkv, int d, int topk, int bs,
                 FwdGeom &g)
{
    if (batch < 0 || max_sq < 0 || max_sk < 0 || total_q < 0 || Hq <= 0 || Hkv <= 0 || topk <= 0 || bs <= 0)
        return SFA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return SFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SFA_ERR_UNSUPPORTED;
    if (bs != 32 && bs != 64) return SFA_ERR_UNSUPPORTED;
    if (topk > 128) return SFA_ERR_UNSUPPORTED;
    const int G = Hq / Hkv;
    if (G > 128) return SFA_ERR_UNSUPPORTED;
    const int64_t nblk_max = ((int64_t)max_sk + bs - 1) / bs;
    if (nblk_max > 65536) return SFA_ERR_UNSUPPORTED;
    g = FwdGeom{};
    g.batch = batch;
    g.max_sq = max_sq;
    g.max_sk = max_sk;
    g.total_q = total_q;
    g.Hq = Hq;
    g.Hkv = Hkv;
    g.d = d;
    g.topk = topk;
    g.bs = bs;
    g.G = G;
    g.Tq = 128 / G;
    g.nqt = (max_sq + g.Tq - 1) / g.Tq;
    const int64_t tiles = (int64_t)g.nqt * batch * Hkv;
    if (tiles > (1ll << 31) - 1) return SFA_ERR_UNSUPPORTED;
    g.tiles = (int)tiles;
    g.nblk_max = (int)std::max<int64_t>(nblk_max, 1);
    g.umax = (int)std::max<int64_t>(1, std::min<int64_t>(nblk_max, (int64_t)g.Tq * topk));
    // Block-major schedule for sparse windows: windows of 64 tiles; its block histogram lives in
    // shared memory, and (token, slot) pairs pack the token into 24 bits.
    g.W = g.Tq * 64;
    g.nwin = (max_sq + g.W - 1) / g.W;
    g.groups = g.nwin * batch * Hkv;
    // A window goes block-major when its tiles' unions hold over 4x its selected blocks (the fitted cost
    // of a block-major row-block, its partial merge included, is about 3.7 query-major row-blocks).  With
    // at most 10*topk blocks per sequence the schedule (and its planning kernels) is left off: the
    // windows of such sequences reach that ratio only in their last tiles, where it did not pay.
    g.inv = (g.nblk_max <= 2048 && g.nblk_max > 10 * topk && total_q < (1 << 24) &&
             fwd_attend_inv_smem_bytes(g) <= 227 * 1024)
                ? 1
                : 0;
    size_t off = 0;
    g.off_sel_c = off;
    off = align_up(off + (size_t)total_q * Hkv * topk * 4);
    g.off_cnt = off;
    off = align_up(off + (size_t)total_q * Hkv * 4);
    g.off_ucnt = off;
    off = align_up(off + (size_t)g.tiles * 4);
    g.off_union = off;
    off = align_up(off + (size_t)g.tiles * g.umax * 4);
    g.off_tilectr = off;
    off = align_up(off + 8);
    if (g.inv) {
        const size_t gb = (size_t)g.groups * g.nblk_max;
        g.cap_items = ((int64_t)total_q * Hkv * topk + g.Tq - 1) / g.Tq + (int64_t)gb;
        g.off_zero = off;  // ctrl and group statistics: cleared per call
        g.off_ctrl = off;
        off = align_up(off + sizeof(InvCtrl));
        g.off_gstat = off;
        off = align_up(off + (size_t)g.groups * sizeof(GroupStat));
        g.zero_bytes = off - g.off_zero;
        g.off_tcount = off;  // written whole by the prep kernel
        off = align_up(off + (size_t)g.tiles * g.nblk_max * 4);
        g.off_gfirst = off;
        off = align_up(off + gb * 4);
        g.off_duni = off;
        off = align_up(off + (size_t)g.tiles * kDenseMax * 4);
        g.off_dcnt = off;
        off = align_up(off + (size_t)g.tiles * 4);
        g.off_dsel = off;  // dsel then dmask
        off = align_up(off + (size_t)2 * total_q * Hkv * 4);
        g.off_items = off;
        off = align_up(off + (size_t)g.cap_items * sizeof(InvItem));
        g.off_pml = off;
        off = align_up(off + (size_t)total_q * Hq * topk * 8);
        g.off_po = off;
        off = align_up(off + (size_t)total_q * Hq * topk * d * 2);
    }
    g.bytes = total_q == 0 ? 0 : off;
    return SFA_OK;
}

// ----------------------------------------------------------------------------------------
// TMA descriptors
// ----------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A (rows, heads, d) bf16 tensor viewed as 3-D {d, heads, rows}; box {64, box_heads, box_rows},
// 128-byte swizzle (matches the UMMA K-major / MN-major SWIZZLE_128B canonical layouts).
bool encode_3d(CUtensorMap &m, const void *base, int d, int heads, int64_t rows, int box_heads, int box_rows)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// A (rows, d) bf16 matrix as a 2-D map {d, rows} with a {64, 1} box, 128-byte swizzle: the form
// tile::gather4 loads use (four arbitrary rows per copy).
bool encode_rows(CUtensorMap &m, const void *base, int d, int64_t rows)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64u, 1u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int check_window(int causal, int wl, int wr)
{
    if (causal != 0 && causal != 1) return SFA_ERR_INVALID_ARG;
    if (wl < -1 || wr < -1) return SFA_ERR_INVALID_ARG;
    return SFA_OK;
}

int fwd_prep_impl(const FwdGeom &g, const int32_t *cu_q, const int32_t *cu_k, const int32_t *sel, int causal, int wl,
                  int wr, void *ws, int32_t *status, cudaStream_t st)
{
    uint8_t *w = static_cast<uint8_t *>(ws);
    if (g.inv && cudaMemsetAsync(w + g.off_zero, 0, g.zero_bytes, st) != cudaSuccess) return SFA_ERR_CUDA;
    FwdPrepParams p{};
    p.cu_q = cu_q;
    p.cu_k = cu_k ? cu_k : cu_q;
    p.sel = sel;
    p.tile_counter = reinterpret_cast<int32_t *>(w + g.off_tilectr);
    p.batch = g.batch;
    p.Hkv = g.Hkv;
    p.topk = g.topk;
    p.bs = g.bs;
    p.causal = causal;
    p.wl = wl;
    p.wr = wr;
    p.Tq = g.Tq;
    p.nqt = g.nqt;
    p.umax = g.umax;
    p.max_sq = g.max_sq;
    p.nblk_max = g.nblk_max;
    p.total_q = g.total_q;
    p.sel_c = reinterpret_cast<int32_t *>(w + g.off_sel_c);
    p.cnt = reinterpret_cast<int32_t *>(w + g.off_cnt);
    p.ucnt = reinterpret_cast<int32_t *>(w + g.off_ucnt);
    p.uni = reinterpret_cast<int32_t *>(w + g.off_union);
    p.W = g.W;
    p.gstat = g.inv ? reinterpret_cast<GroupStat *>(w + g.off_gstat) : nullptr;
    p.tcount = g.inv ? reinterpret_cast<int32_t *>(w + g.off_tcount) : nullptr;
    // dense blocks of block-major tiles go to the pipelined query-major kernel (not the one-tile one)
    const bool dense = g.inv && g.topk <= 32 && fwd_pipe_fits(g, kPipePrep);
    p.duni = dense ? reinterpret_cast<int32_t *>(w + g.off_duni) : nullptr;
    p.dcnt = dense ? reinterpret_cast<int32_t *>(w + g.off_dcnt) : nullptr;
    p.dsel = dense ? reinterpret_cast<uint32_t *>(w + g.off_dsel) : nullptr;
    p.status = status;
    if (launch_fwd_prep(g, p, st) != cudaSuccess) return SFA_ERR_CUDA;
    if (!g.inv) return SFA_OK;
    // Which windows go block-major, and their items.
    FwdPlanParams pl{};
    pl.ucnt = p.ucnt;
    pl.gstat = p.gstat;
    pl.tcount = p.tcount;
    pl.gfirst = reinterpret_cast<int32_t *>(w + g.off_gfirst);
    pl.batch = g.batch;
    pl.Hkv = g.Hkv;
    pl.Tq = g.Tq;
    pl.nqt = g.nqt;
    pl.W = g.W;
    pl.nblk_max = g.nblk_max;
    pl.cu_q = cu_q;
    pl.cu_k = p.cu_k;
    pl.items = reinterpret_cast<InvItem *>(w + g.off_items);
    pl.ctrl = reinterpret_cast<InvCtrl *>(w + g.off_ctrl);
    if (launch_fwd_plan(g, pl, st) != cudaSuccess) return SFA_ERR_CUDA;
    FwdScatterParams sc{};
    sc.cu_q = cu_q;
    sc.sel_c = p.sel_c;
    sc.cnt = p.cnt;
    sc.ucnt = p.ucnt;
    sc.gfirst = pl.gfirst;
    sc.tcount = p.tcount;
    sc.dmask = dense ? p.dsel + (size_t)g.total_q * g.Hkv : nullptr;
    sc.batch = g.batch;
    sc.Hkv = g.Hkv;
    sc.topk = g.topk;
    sc.Tq = g.Tq;
    sc.nqt = g.nqt;
    sc.W = g.W;
    sc.nblk_max = g.nblk_max;
    sc.items = pl.items;
    return launch_fwd_scatter(g, sc, st) == cudaSuccess ? SFA_OK : SFA_ERR_CUDA;
}

// The attention stage.  sel == nullptr: the canonical sets come from the prep kernel's output in
// the workspace.  sel != nullptr (fused, only without the block-major schedule): the pipelined
// kernel canonicalizes the raw selections itself and the prep kernel does not run.
int fwd_attend_impl(const FwdGeom &g, const void *q, const void *k, const void *v, const int32_t *cu_q,
                    const int32_t *cu_k, int total_k, int causal, int wl, int wr, float scale, void *ws,
                    int32_t *status, void *out, float *lse, cudaStream_t st, const int32_t *sel = nullptr)
{
    const bool fused = sel != nullptr;
    const bool pipe = fwd_pipe_fits(g, fused ? kPipeFused : kPipePrep);
    if (fused && (!pipe || g.inv)) return SFA_ERR_UNSUPPORTED;
    if (!pipe && fwd_attend_smem_bytes(g) > 227 * 1024) return SFA_ERR_UNSUPPORTED;
    CUtensorMap tq, tk, tv;
    if (!encode_3d(tq, q, g.d, g.Hq, g.total_q, g.G, g.Tq)) return SFA_ERR_CUDA;
    if (!encode_3d(tk, k, g.d, g.Hkv, total_k, 1, g.bs)) return SFA_ERR_CUDA;
    if (!encode_3d(tv, v, g.d, g.Hkv, total_k, 1, g.bs)) return SFA_ERR_CUDA;
    FwdAttendParams p{};
    p.cu_q = cu_q;
    p.cu_k = cu_k ? cu_k : cu_q;
    const uint8_t *w = static_cast<const uint8_t *>(ws);
    p.sel_c = reinterpret_cast<const int32_t *>(w + g.off_sel_c);
    p.cnt = reinterpret_cast<const int32_t *>(w + g.off_cnt);
    p.ucnt = reinterpret_cast<const int32_t *>(w + g.off_ucnt);
    p.uni = reinterpret_cast<const int32_t *>(w + g.off_union);
    p.batch = g.batch;
    p.total_q = g.total_q;
    p.Hq = g.Hq;
    p.Hkv = g.Hkv;
    p.G = g.G;
    p.Tq = g.Tq;
    p.nqt = g.nqt;
    p.topk = g.topk;
    p.umax = g.umax;
    p.causal = causal;
    p.wl = wl;
    p.wr = wr;
    const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)g.d);
    p.scale_log2 = (float)(sc * 1.4426950408889634);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = status;
    p.tiles = g.tiles;
    p.tile_counter = reinterpret_cast<int32_t *>(const_cast<uint8_t *>(w) + g.off_tilectr);
    p.sel = sel;
    p.bs = g.bs;
    p.max_sq = g.max_sq;
    p.nblk_max = g.nblk_max;
    if (g.inv && g.topk <= 32 && pipe) {  // the dense blocks of block-major tiles (see the prep)
        const uint8_t *wd = static_cast<const uint8_t *>(ws);
        p.duni = reinterpret_cast<const int32_t *>(wd + g.off_duni);
        p.dcnt = reinterpret_cast<const int32_t *>(wd + g.off_dcnt);
        p.dsel = reinterpret_cast<const uint32_t *>(wd + g.off_dsel);
        p.dmask = p.dsel + (size_t)g.total_q * g.Hkv;
    }
    if (fused && cudaMemsetAsync(p.tile_counter, 0, 2 * sizeof(int32_t), st) != cudaSuccess) return SFA_ERR_CUDA;
    if ((pipe ? launch_fwd_attend_pipe(g, p, fused ? kPipeFused : kPipePrep, tq, tk, tv, st)
              : launch_fwd_attend(g, p, tq, tk, tv, st)) !=
        cudaSuccess)
        return SFA_ERR_CUDA;
    if (!g.inv) return SFA_OK;
    uint8_t *wm = static_cast<uint8_t *>(ws);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.items = reinterpret_cast<const InvItem *>(wm + g.off_items);
    p.ctrl = reinterpret_cast<InvCtrl *>(wm + g.off_ctrl);
    p.po = reinterpret_cast<__nv_bfloat16 *>(wm + g.off_po);
    p.pml = reinterpret_cast<float2 *>(wm + g.off_pml);
    CUtensorMap tq2;  // q as (total_q * Hq) rows of d, one-row boxes for the 4-row gathers
    if (!encode_rows(tq2, q, g.d, (int64_t)g.total_q * g.Hq)) return SFA_ERR_CUDA;
    if (launch_fwd_attend_inv(g, p, tq2, tk, tv, st) != cudaSuccess) return SFA_ERR_CUDA;
    return launch_fwd_merge(g, p, st) == cudaSuccess ? SFA_OK : SFA_ERR_CUDA;
}

int fwd_common_checks(const int32_t *cu_q, const int32_t *cu_k, int total_q, int total_k, int max_sq, int max_sk,
                      int causal, int wl, int wr)
{
    if (!cu_q) return SFA_ERR_INVALID_ARG;
    if (total_k < 0) return SFA_ERR_INVALID_ARG;
    if (!cu_k && total_k != total_q) return SFA_ERR_INVALID_ARG;
    if (!cu_k && max_sk != max_sq) return SFA_ERR_INVALID_ARG;
    return check_window(causal, wl, wr);
}

// ----------------------------------------------------------------------------------------
// Backward geometry: the forward's prep region (canonical lists, unions, tile counter) followed by
// the backward's own arrays.
// ----------------------------------------------------------------------------------------
int bwd_geometry(int batch, int max_sq, int max_sk, int total_q, int Hq, int Hkv, int d, int topk, int bs,
                 BwdGeom &g)
{
    int rc = fwd_geometry(batch, max_sq, max_sk, total_q, Hq, Hkv, d, topk, bs, g.f);
    if (rc != SFA_OK) return rc;
    g.f.inv = 0;  // the backward walks the query tiles; no block-major forward schedule
    const int64_t total_sel = (int64_t)total_q * Hkv * topk;
    if ((int64_t)total_q * Hq >= (1ll << 31) || total_sel >= (1ll << 31)) return SFA_ERR_UNSUPPORTED;
    const int64_t R = (int64_t)batch * Hkv * g.f.nblk_max;
    const int64_t words = std::max<int64_t>(1, ((int64_t)max_sq + 31) / 32);
    if (R >= (1ll << 31) || R * words >= (1ll << 40)) return SFA_ERR_UNSUPPORTED;
    g.R = (int)R;
    g.words = (int)words;
    const int64_t per_piece = (int64_t)kBwdPieceChunks * g.f.Tq;
    // A row of c tokens makes ceil(c / per_piece) <= c / per_piece + 1 pieces; the rows of more than
    // per_piece tokens (at most total_sel / (per_piece + 1) of them) need one partial slot per piece.
    g.max_pieces = total_sel / per_piece + std::min(R, total_sel) + 1;
    g.max_slots = total_sel / per_piece + total_sel / (per_piece + 1) + 2;
    size_t off = align_up(g.f.off_tilectr + 8);
    g.off_delta = off;
    off = align_up(off + (size_t)total_q * Hq * 4);
    g.off_zero = off;
    g.off_bits = off;
    off = align_up(off + (size_t)R * words * 4);
    g.off_rowcnt = off;
    off = align_up(off + (size_t)R * 4);
    g.off_flags = off;
    off = align_up(off + (size_t)g.max_slots * 4);
    g.zero_bytes = off - g.off_zero;
    g.off_ctrl = off;
    off = align_up(off + sizeof(BwdCtrl));
    g.off_rowoff = off;
    off = align_up(off + (size_t)R * 4);
    g.off_toks = off;
    off = align_up(off + (size_t)total_sel * 4);
    g.off_pieces = off;
    off = align_up(off + (size_t)g.max_pieces * sizeof(BwdPiece));
    g.off_part = off;
    off = align_up(off + (size_t)g.max_slots * 2 * bs * d * 4);
    g.bytes = total_q == 0 ? 0 : off;
    return SFA_OK;
}

// ----------------------------------------------------------------------------------------
// Decode geometry
// ----------------------------------------------------------------------------------------
int num_sms()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Split count: each split is one warp's chunk of a (sequence, kv head) token list; the splits of
// one (sequence, kv head) run decode_split_warps_per_block() to a CTA, and each CTA first
// deduplicates the whole selection.  Fill one wave of num_SMs * CTAs-per-SM slots: as many CTAs
// per (sequence, kv head) as fit in that wave, at least one, with at least 64 tokens per split.
int choose_splits(int B, int Hkv, int d, int topk)
{
    const int units = B * Hkv;
    const int wpb = decode_split_warps_per_block();
    const int slots = num_sms() * decode_split_blocks_per_sm(d);
    const int cps = std::max(1, std::min(slots / std::max(units, 1), topk / (wpb * 64)));
    return std::max(1, std::min(cps * wpb, topk / 64));
}

int dec_geometry(int B, int Hq, int Hkv, int d, int topk, int num_splits, DecGeom &g)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || topk <= 0 || num_splits < 0) return SFA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return SFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SFA_ERR_UNSUPPORTED;
    if (Hq / Hkv > 16) return SFA_ERR_UNSUPPORTED;
    if (topk > 65536) return SFA_ERR_UNSUPPORTED;
    g = DecGeom{};
    g.B = B;
    g.Hq = Hq;
    g.Hkv = Hkv;
    g.d = d;
    g.topk = topk;
    g.G = Hq / Hkv;
    g.S = num_splits > 0 ? std::min(num_splits, topk) : choose_splits(B, Hkv, d, topk);
    size_t off = 0;
    g.off_tok = off;
    off = align_up(off + (size_t)B * Hkv * topk * 4);
    g.off_cnt = off;
    off = align_up(off + (size_t)B * Hkv * 4);
    g.off_po = off;
    off = align_up(off + (size_t)B * Hq * g.S * d * 4);
    g.off_plse = off;
    off = align_up(off + (size_t)B * Hq * g.S * 4);
    g.bytes = B == 0 ? 0 : off;
    return SFA_OK;
}

int dec_prep_impl(const DecGeom &g, const int32_t *seqlens, const int32_t *sel, int max_pages, int page, int wl,
                  void *ws, int32_t *status, cudaStream_t st)
{
    const int64_t max_len = (int64_t)max_pages * page;
    if (max_len > (1 << 20)) return SFA_ERR_UNSUPPORTED;
    DecPrepParams p{};
    p.seqlens = seqlens;
    p.sel = sel;
    p.topk = g.topk;
    p.max_len = (int)max_len;
    p.Hkv = g.Hkv;
    p.wl = wl;
    uint8_t *w = static_cast<uint8_t *>(ws);
    p.tok_c = reinterpret_cast<int32_t *>(w + g.off_tok);
    p.cnt = reinterpret_cast<int32_t *>(w + g.off_cnt);
    p.status = status;
    return launch_decode_prep(g, p, st) == cudaSuccess ? SFA_OK : SFA_ERR_CUDA;
}

// fused: the split kernel deduplicates sel itself (no prep launch); else it reads the prep kernel's
// canonical sets from the workspace.
int dec_attend_impl(const DecGeom &g, const void *q, const void *kc, const void *vc, const int32_t *bt, int max_pages,
                    int num_pages, int page, const int32_t *seqlens, const int32_t *sel, int wl, bool fused,
                    float scale, void *ws, int32_t *status, void *out, float *lse, cudaStream_t st,
                    bool fp8 = false, const float *kd = nullptr, const float *vd = nullptr)
{
    if ((int64_t)num_pages * page * g.Hkv > (int64_t)INT32_MAX) return SFA_ERR_UNSUPPORTED;
    uint8_t *w = static_cast<uint8_t *>(ws);
    DecSplitParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.kc = static_cast<const __nv_bfloat16 *>(kc);
    p.vc = static_cast<const __nv_bfloat16 *>(vc);
    p.bt = bt;
    p.tok_c = reinterpret_cast<const int32_t *>(w + g.off_tok);
    p.cnt = reinterpret_cast<const int32_t *>(w + g.off_cnt);
    p.seqlens = seqlens;
    p.sel = sel;
    p.fused = fused ? 1 : 0;
    p.wl = wl;
    p.B = g.B;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
    p.page = page;
    p.page_shift = -1;
    for (int sh = 0; sh < 31; ++sh)
        if ((1 << sh) == page) p.page_shift = sh;
    p.Hq = g.Hq;
    p.Hkv = g.Hkv;
    p.G = g.G;
    p.topk = g.topk;
    p.S = g.S;
    const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)g.d);
    p.scale_log2 = (float)(sc * 1.4426950408889634);
    p.po = reinterpret_cast<float *>(w + g.off_po);
    p.plse = reinterpret_cast<float *>(w + g.off_plse);
    p.out_direct = static_cast<__nv_bfloat16 *>(out);
    p.lse_direct = lse;
    p.fp8 = fp8 ? 1 : 0;
    p.kd = kd;
    p.vd = vd;
    p.status = status;
    if (launch_decode_split(g, p, st) != cudaSuccess) return SFA_ERR_CUDA;
    if (g.S <= decode_split_warps_per_block()) return SFA_OK;  // combined inside the split kernel
    DecCombineParams c{};
    c.po = p.po;
    c.plse = p.plse;
    c.Hq = g.Hq;
    c.S = g.S;
    c.out = static_cast<__nv_bfloat16 *>(out);
    c.lse = lse;
    return launch_decode_combine(g, c, st) == cudaSuccess ? SFA_OK : SFA_ERR_CUDA;
}

}  // namespace

namespace {

// sfa_decode and sfa_decode_fp8: fp8 caches hold E4M3 codes with descales kd / vd (B, Hkv) or nullptr.
int decode_impl(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                int max_pages_per_seq, int num_pages, int page_size, const int32_t *cache_seqlens,
                const int32_t *sel_tok_idx, int topk_tok, int B, int Hq, int Hkv, int d, int window_left, float scale,
                int num_splits, void *workspace, size_t workspace_bytes, int32_t *status_dev, void *out, float *lse,
                sfa_stream_t stream, bool fp8, const float *kd, const float *vd)
{
    g_last_launches = 0;
    DecGeom g;
    int rc = dec_geometry(B, Hq, Hkv, d, topk_tok, num_splits, g);
    if (rc != SFA_OK) return rc;
    if (page_size <= 0 || max_pages_per_seq <= 0 || num_pages < 0 || window_left < -1) return SFA_ERR_INVALID_ARG;
    if (B == 0) return SFA_OK;
    if (!q || !k_cache || !v_cache || !block_table || !cache_seqlens || !sel_tok_idx || !workspace || !out || !lse)
        return SFA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return SFA_ERR_INVALID_ARG;
    if (fp8 && ((kd && (reinterpret_cast<uintptr_t>(kd) & 3u)) || (vd && (reinterpret_cast<uintptr_t>(vd) & 3u))))
        return SFA_ERR_INVALID_ARG;
    if (workspace_bytes < g.bytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (g.bytes > 0 && !aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    // Selections of up to decode_fused_max_topk() positions are deduplicated inside the split
    // kernel; longer ones go through the prep kernel first.
    const bool fused = topk_tok <= decode_fused_max_topk();
    if (!fused) {
        rc = dec_prep_impl(g, cache_seqlens, sel_tok_idx, max_pages_per_seq, page_size, window_left, workspace,
                           status_dev, stream);
        if (rc != SFA_OK) return rc;
    } else if ((int64_t)max_pages_per_seq * page_size > (1 << 20)) {
        return SFA_ERR_UNSUPPORTED;
    }
    rc = dec_attend_impl(g, q, k_cache, v_cache, block_table, max_pages_per_seq, num_pages, page_size, cache_seqlens,
                         sel_tok_idx, window_left, fused, scale, workspace, status_dev, out, lse, stream, fp8, kd, vd);
    if (rc == SFA_OK) g_last_launches = (fused ? 0 : 1) + (g.S <= decode_split_warps_per_block() ? 1 : 2);
    return rc;
}

}  // namespace

extern "C" {

size_t sfa_fwd_workspace_size(int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int Hq, int Hkv, int d,
                              int topk, int block_size)
{
    FwdGeom g;
    if (fwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size, g) != SFA_OK) return 0;
    return g.bytes;
}

int sfa_fwd_workspace_offsets(int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int Hq, int Hkv, int d,
                              int topk, int block_size, size_t *off_sel_c, size_t *off_cnt)
{
    FwdGeom g;
    const int rc = fwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size, g);
    if (rc != SFA_OK) return rc;
    if (off_sel_c) *off_sel_c = g.off_sel_c;
    if (off_cnt) *off_cnt = g.off_cnt;
    return SFA_OK;
}

int sfa_fwd_prep(const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int batch, int max_seqlen_q,
                 int max_seqlen_k, int total_q, int Hq, int Hkv, int d, const int32_t *sel_idx, int topk,
                 int block_size, int causal, int window_left, int window_right, void *workspace,
                 size_t workspace_bytes, int32_t *status_dev, sfa_stream_t stream)
{
    g_last_launches = 0;
    FwdGeom g;
    int rc = fwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size, g);
    if (rc != SFA_OK) return rc;
    if (!cu_seqlens_q || (total_q > 0 && !sel_idx)) return SFA_ERR_INVALID_ARG;
    if ((rc = check_window(causal, window_left, window_right)) != SFA_OK) return rc;
    if (total_q == 0 || batch == 0) return SFA_OK;
    if (!workspace) return SFA_ERR_INVALID_ARG;
    if (workspace_bytes < g.bytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (g.bytes > 0 && !aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    rc = fwd_prep_impl(g, cu_seqlens_q, cu_seqlens_k, sel_idx, causal, window_left, window_right, workspace,
                       status_dev, stream);
    if (rc == SFA_OK) g_last_launches = 1 + 2 * g.inv;
    return rc;
}

int sfa_fwd_attend(const void *q, const void *k, const void *v, const int32_t *cu_seqlens_q,
                   const int32_t *cu_seqlens_k, int batch, int max_seqlen_q, int max_seqlen_k, int total_q,
                   int total_k, int Hq, int Hkv, int d, int topk, int block_size, int causal, int window_left,
                   int window_right, float scale, void *workspace, size_t workspace_bytes, int32_t *status_dev,
                   void *out, float *lse, sfa_stream_t stream)
{
    g_last_launches = 0;
    FwdGeom g;
    int rc = fwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size, g);
    if (rc != SFA_OK) return rc;
    if ((rc = fwd_common_checks(cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k, causal,
                                window_left, window_right)) != SFA_OK)
        return rc;
    if (total_q == 0 || batch == 0) return SFA_OK;
    if (!q || !k || !v || !out || !lse || !workspace) return SFA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SFA_ERR_INVALID_ARG;
    if (total_k == 0) return SFA_ERR_UNSUPPORTED;
    if (workspace_bytes < g.bytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (g.bytes > 0 && !aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    rc = fwd_attend_impl(g, q, k, v, cu_seqlens_q, cu_seqlens_k, total_k, causal, window_left, window_right, scale,
                         workspace, status_dev, out, lse, stream);
    if (rc == SFA_OK) g_last_launches = 1 + 2 * g.inv;
    return rc;
}

int sfa_fwd(const void *q, const void *k, const void *v, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
            int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d,
            const int32_t *sel_idx, int topk, int block_size, int causal, int window_left, int window_right,
            float scale, void *workspace, size_t workspace_bytes, int32_t *status_dev, void *out, float *lse,
            sfa_stream_t stream)
{
    g_last_launches = 0;
    FwdGeom g;
    int rc = fwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size, g);
    if (rc != SFA_OK) return rc;
    if ((rc = fwd_common_checks(cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k, causal,
                                window_left, window_right)) != SFA_OK)
        return rc;
    if (total_q == 0 || batch == 0) return SFA_OK;
    if (!q || !k || !v || !out || !lse || !workspace || !sel_idx) return SFA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SFA_ERR_INVALID_ARG;
    if (total_k == 0) return SFA_ERR_UNSUPPORTED;
    if (workspace_bytes < g.bytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (g.bytes > 0 && !aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    if (!fwd_pipe_fits(g, kPipePrep) && fwd_attend_smem_bytes(g) > 227 * 1024) return SFA_ERR_UNSUPPORTED;
    if (!g.inv && fwd_pipe_fits(g, kPipeFused)) {
        // One launch: the attention kernel canonicalizes each tile's selections itself.
        rc = fwd_attend_impl(g, q, k, v, cu_seqlens_q, cu_seqlens_k, total_k, causal, window_left, window_right,
                             scale, workspace, status_dev, out, lse, stream, sel_idx);
        if (rc == SFA_OK) g_last_launches = 1;
        return rc;
    }
    rc = fwd_prep_impl(g, cu_seqlens_q, cu_seqlens_k, sel_idx, causal, window_left, window_right, workspace,
                       status_dev, stream);
    if (rc != SFA_OK) return rc;
    rc = fwd_attend_impl(g, q, k, v, cu_seqlens_q, cu_seqlens_k, total_k, causal, window_left, window_right, scale,
                         workspace, status_dev, out, lse, stream);
    if (rc == SFA_OK) g_last_launches = 2 + 4 * g.inv;
    return rc;
}

size_t sfa_bwd_workspace_size(int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int Hq, int Hkv, int d,
                              int topk, int block_size)
{
    BwdGeom g;
    if (bwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size, g) != SFA_OK) return 0;
    return g.bytes;
}

int sfa_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int batch, int max_seqlen_q, int max_seqlen_k,
            int total_q, int total_k, int Hq, int Hkv, int d, const int32_t *sel_idx, int topk, int block_size,
            int causal, int window_left, int window_right, float scale, void *workspace, size_t workspace_bytes,
            int32_t *status_dev, void *dq, void *dk, void *dv, sfa_stream_t stream)
{
    g_last_launches = 0;
    BwdGeom g;
    int rc = bwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, topk, block_size, g);
    if (rc != SFA_OK) return rc;
    if ((rc = fwd_common_checks(cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k, causal,
                                window_left, window_right)) != SFA_OK)
        return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (total_k > 0 && (!dk || !dv || !aligned16(dk) || !aligned16(dv))) return SFA_ERR_INVALID_ARG;
    if (total_q == 0 || batch == 0) {  // no query: every key's gradient is zero
        if (total_k > 0) {
            const size_t bytes = (size_t)total_k * Hkv * d * 2;
            if (cudaMemsetAsync(dk, 0, bytes, st) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, st) != cudaSuccess)
                return SFA_ERR_CUDA;
        }
        return SFA_OK;
    }
    if (!q || !k || !v || !out || !dout || !lse || !workspace || !sel_idx || !dq) return SFA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq))
        return SFA_ERR_INVALID_ARG;
    if (total_k == 0) return SFA_ERR_UNSUPPORTED;
    // The dQ kernel keeps two copies of a tile's block union in shared memory beside its rings.
    if (bwd_dq_smem_bytes(g) > 227 * 1024 || bwd_dkdv_smem_bytes(g) > 227 * 1024) return SFA_ERR_UNSUPPORTED;
    if (workspace_bytes < g.bytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (g.bytes > 0 && !aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    uint8_t *w = static_cast<uint8_t *>(workspace);
    if (cudaMemsetAsync(w + g.off_zero, 0, g.zero_bytes, st) != cudaSuccess) return SFA_ERR_CUDA;
    rc = fwd_prep_impl(g.f, cu_seqlens_q, cu_seqlens_k, sel_idx, causal, window_left, window_right, workspace,
                       status_dev, st);
    if (rc != SFA_OK) return rc;
    CUtensorMap tq, tdo, tk, tv;
    if (!encode_3d(tq, q, d, Hq, total_q, g.f.G, g.f.Tq) || !encode_3d(tdo, dout, d, Hq, total_q, g.f.G, g.f.Tq) ||
        !encode_3d(tk, k, d, Hkv, total_k, 1, block_size) || !encode_3d(tv, v, d, Hkv, total_k, 1, block_size))
        return SFA_ERR_CUDA;
    BwdParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.out = static_cast<const __nv_bfloat16 *>(out);
    p.dout = static_cast<const __nv_bfloat16 *>(dout);
    p.lse = lse;
    p.cu_q = cu_seqlens_q;
    p.cu_k = cu_seqlens_k ? cu_seqlens_k : cu_seqlens_q;
    p.sel_c = reinterpret_cast<const int32_t *>(w + g.f.off_sel_c);
    p.cnt = reinterpret_cast<const int32_t *>(w + g.f.off_cnt);
    p.ucnt = reinterpret_cast<const int32_t *>(w + g.f.off_ucnt);
    p.uni = reinterpret_cast<const int32_t *>(w + g.f.off_union);
    p.batch = batch;
    p.total_q = total_q;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = g.f.G;
    p.Tq = g.f.Tq;
    p.nqt = g.f.nqt;
    p.topk = topk;
    p.umax = g.f.umax;
    p.tiles = g.f.tiles;
    p.nblk_max = g.f.nblk_max;
    p.max_sq = max_seqlen_q;
    p.words = g.words;
    p.R = g.R;
    p.causal = causal;
    p.wl = window_left;
    p.wr = window_right;
    const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)d);
    p.scale = (float)sc;
    p.scale_log2 = (float)(sc * 1.4426950408889634);
    p.delta = reinterpret_cast<float *>(w + g.off_delta);
    p.bits = reinterpret_cast<uint32_t *>(w + g.off_bits);
    p.rowcnt = reinterpret_cast<int32_t *>(w + g.off_rowcnt);
    p.rowoff = reinterpret_cast<int32_t *>(w + g.off_rowoff);
    p.toks = reinterpret_cast<int32_t *>(w + g.off_toks);
    p.pieces = reinterpret_cast<BwdPiece *>(w + g.off_pieces);
    p.ctrl = reinterpret_cast<BwdCtrl *>(w + g.off_ctrl);
    p.flags = reinterpret_cast<int32_t *>(w + g.off_flags);
    p.part = reinterpret_cast<float *>(w + g.off_part);
    p.max_pieces = g.max_pieces;
    p.max_slots = g.max_slots;
    p.tile_counter = reinterpret_cast<int32_t *>(w + g.f.off_tilectr);
    p.dq = static_cast<__nv_bfloat16 *>(dq);
    p.dk = static_cast<__nv_bfloat16 *>(dk);
    p.dv = static_cast<__nv_bfloat16 *>(dv);
    p.status = status_dev;
    if (launch_bwd_delta(g, p, st) != cudaSuccess || launch_bwd_index(g, p, st) != cudaSuccess ||
        launch_bwd_plan(g, p, st) != cudaSuccess || launch_bwd_fill(g, p, st) != cudaSuccess ||
        launch_bwd_dq(g, p, tq, tdo, tk, tv, st) != cudaSuccess ||
        launch_bwd_dkdv(g, p, tk, tv, st) != cudaSuccess)
        return SFA_ERR_CUDA;
    g_last_launches = 7;
    return SFA_OK;
}

size_t sfa_index_topk_workspace_size(int B, int Hkv, int max_pages_per_seq, int page_size)
{
    if (B <= 0 || Hkv <= 0 || max_pages_per_seq <= 0 || page_size <= 0) return 0;
    return (size_t)B * Hkv * max_pages_per_seq * page_size * 8;
}

int sfa_index_topk(const void *q, const void *k_cache, const int32_t *block_table, int max_pages_per_seq,
                   int num_pages, int page_size, const int32_t *cache_seqlens, int B, int Hq, int Hkv, int d, int topk,
                   int n_local, void *workspace, size_t workspace_bytes, int32_t *status_dev, int32_t *sel_out,
                   sfa_stream_t stream)
{
    g_last_launches = 0;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || topk <= 0 || n_local < 0 || max_pages_per_seq < 0 || num_pages < 0 ||
        page_size <= 0)
        return SFA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return SFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SFA_ERR_UNSUPPORTED;
    if (Hq / Hkv > 1024) return SFA_ERR_UNSUPPORTED;  // past that, fp64 no longer holds the scores exactly
    if ((int64_t)max_pages_per_seq * page_size > (1 << 20) || topk > (1 << 20)) return SFA_ERR_UNSUPPORTED;
    if (B == 0) return SFA_OK;
    if (!q || !k_cache || !block_table || !cache_seqlens || !sel_out || !workspace) return SFA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache)) return SFA_ERR_INVALID_ARG;
    if (workspace_bytes < sfa_index_topk_workspace_size(B, Hkv, max_pages_per_seq, page_size))
        return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    IndexParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.kc = static_cast<const __nv_bfloat16 *>(k_cache);
    p.bt = block_table;
    p.seqlens = cache_seqlens;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = Hq / Hkv;
    p.d = d;
    p.max_pages = max_pages_per_seq;
    p.num_pages = num_pages;
    p.page = page_size;
    p.topk = topk;
    p.n_local = n_local;
    p.max_len = (int64_t)max_pages_per_seq * page_size;
    p.keys = static_cast<unsigned long long *>(workspace);
    p.sel = sel_out;
    p.status = status_dev;
    if (launch_index_topk(p, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SFA_ERR_CUDA;
    g_last_launches = 2;
    return SFA_OK;
}

int sfa_kv_append(const void *k_new, const void *v_new, int seqlen_new, void *k_cache, void *v_cache,
                  const int32_t *block_table, int max_pages_per_seq, int num_pages, int page_size,
                  const int32_t *cache_seqlens, int B, int Hkv, int d, int32_t *status_dev, sfa_stream_t stream)
{
    g_last_launches = 0;
    if (B < 0 || seqlen_new < 0 || Hkv <= 0 || d <= 0 || max_pages_per_seq < 0 || num_pages < 0 || page_size <= 0)
        return SFA_ERR_INVALID_ARG;
    if (d % 8 != 0) return SFA_ERR_UNSUPPORTED;
    if (B == 0 || seqlen_new == 0) return SFA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !cache_seqlens) return SFA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache)) return SFA_ERR_INVALID_ARG;
    KvAppendParams p{};
    p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    p.k_cache = static_cast<__nv_bfloat16 *>(k_cache);
    p.v_cache = static_cast<__nv_bfloat16 *>(v_cache);
    p.bt = block_table;
    p.seqlens = cache_seqlens;
    p.B = B;
    p.S = seqlen_new;
    p.Hkv = Hkv;
    p.d = d;
    p.max_pages = max_pages_per_seq;
    p.num_pages = num_pages;
    p.page = page_size;
    p.status = status_dev;
    if (launch_kv_append(p, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SFA_ERR_CUDA;
    g_last_launches = 1;
    return SFA_OK;
}

int sfa_decode_num_splits(int B, int Hq, int Hkv, int d, int topk_tok, int num_splits)
{
    DecGeom g;
    if (dec_geometry(B, Hq, Hkv, d, topk_tok, num_splits, g) != SFA_OK) return 0;
    return g.S;
}

size_t sfa_decode_workspace_size(int B, int Hq, int Hkv, int d, int topk_tok, int num_splits)
{
    DecGeom g;
    if (dec_geometry(B, Hq, Hkv, d, topk_tok, num_splits, g) != SFA_OK) return 0;
    return g.bytes;
}

int sfa_decode_workspace_offsets(int B, int Hq, int Hkv, int d, int topk_tok, int num_splits, size_t *off_tok_c,
                                 size_t *off_cnt)
{
    DecGeom g;
    const int rc = dec_geometry(B, Hq, Hkv, d, topk_tok, num_splits, g);
    if (rc != SFA_OK) return rc;
    if (off_tok_c) *off_tok_c = g.off_tok;
    if (off_cnt) *off_cnt = g.off_cnt;
    return SFA_OK;
}

int sfa_decode_prep(const int32_t *cache_seqlens, const int32_t *sel_tok_idx, int topk_tok, int max_pages_per_seq,
                    int page_size, int B, int Hq, int Hkv, int d, int window_left, int num_splits, void *workspace,
                    size_t workspace_bytes, int32_t *status_dev, sfa_stream_t stream)
{
    g_last_launches = 0;
    DecGeom g;
    int rc = dec_geometry(B, Hq, Hkv, d, topk_tok, num_splits, g);
    if (rc != SFA_OK) return rc;
    if (page_size <= 0 || max_pages_per_seq <= 0 || window_left < -1) return SFA_ERR_INVALID_ARG;
    if (B == 0) return SFA_OK;
    if (!cache_seqlens || !sel_tok_idx || !workspace) return SFA_ERR_INVALID_ARG;
    if (workspace_bytes < g.bytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (g.bytes > 0 && !aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    rc = dec_prep_impl(g, cache_seqlens, sel_tok_idx, max_pages_per_seq, page_size, window_left, workspace, status_dev,
                       stream);
    if (rc == SFA_OK) g_last_launches = 1;
    return rc;
}

int sfa_decode_attend(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                      int max_pages_per_seq, int num_pages, int page_size, int topk_tok, int B, int Hq, int Hkv, int d,
                      float scale, int num_splits, void *workspace, size_t workspace_bytes, int32_t *status_dev,
                      void *out, float *lse, sfa_stream_t stream)
{
    g_last_launches = 0;
    DecGeom g;
    int rc = dec_geometry(B, Hq, Hkv, d, topk_tok, num_splits, g);
    if (rc != SFA_OK) return rc;
    if (page_size <= 0 || max_pages_per_seq <= 0 || num_pages < 0) return SFA_ERR_INVALID_ARG;
    if (B == 0) return SFA_OK;
    if (!q || !k_cache || !v_cache || !block_table || !workspace || !out || !lse) return SFA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return SFA_ERR_INVALID_ARG;
    if (workspace_bytes < g.bytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (g.bytes > 0 && !aligned256(workspace)) return SFA_ERR_INVALID_ARG;
    rc = dec_attend_impl(g, q, k_cache, v_cache, block_table, max_pages_per_seq, num_pages, page_size, nullptr,
                         nullptr, -1, false, scale, workspace, status_dev, out, lse, stream);
    if (rc == SFA_OK) g_last_launches = g.S <= decode_split_warps_per_block() ? 1 : 2;
    return rc;
}

int sfa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
               int max_pages_per_seq, int num_pages, int page_size, const int32_t *cache_seqlens,
               const int32_t *sel_tok_idx, int topk_tok, int B, int Hq, int Hkv, int d, int window_left, float scale,
               int num_splits, void *workspace, size_t workspace_bytes, int32_t *status_dev, void *out, float *lse,
               sfa_stream_t stream)
{
    return decode_impl(q, k_cache, v_cache, block_table, max_pages_per_seq, num_pages, page_size, cache_seqlens,
                       sel_tok_idx, topk_tok, B, Hq, Hkv, d, window_left, scale, num_splits, workspace, workspace_bytes,
                       status_dev, out, lse, stream, false, nullptr, nullptr);
}

int sfa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const float *k_descale,
                   const float *v_descale, const int32_t *block_table, int max_pages_per_seq, int num_pages,
                   int page_size, const int32_t *cache_seqlens, const int32_t *sel_tok_idx, int topk_tok, int B,
                   int Hq, int Hkv, int d, int window_left, float scale, int num_splits, void *workspace,
                   size_t workspace_bytes, int32_t *status_dev, void *out, float *lse, sfa_stream_t stream)
{
    return decode_impl(q, k_cache, v_cache, block_table, max_pages_per_seq, num_pages, page_size, cache_seqlens,
                       sel_tok_idx, topk_tok, B, Hq, Hkv, d, window_left, scale, num_splits, workspace, workspace_bytes,
                       status_dev, out, lse, stream, true, k_descale, v_descale);
}

// A cache of batch_cache sequences of seqlen_cache rows each is a paged cache of batch_cache pages of
// seqlen_cache rows whose block table has one column, cache_batch_idx: row j of sequence b is then
// k_cache[cache_batch_idx[b]][j], the non-paged indexing of flash_attn_with_kvcache.
int sfa_decode_kvcache(const void *q, const void *k_cache, const void *v_cache, int batch_cache, int seqlen_cache,
                       const int32_t *cache_batch_idx, const int32_t *cache_seqlens, const int32_t *sel_tok_idx,
                       int topk_tok, int B, int Hq, int Hkv, int d, int window_left, float scale, int num_splits,
                       void *workspace, size_t workspace_bytes, int32_t *status_dev, void *out, float *lse,
                       sfa_stream_t stream)
{
    return sfa_decode(q, k_cache, v_cache, cache_batch_idx, 1, batch_cache, seqlen_cache, cache_seqlens, sel_tok_idx,
                      topk_tok, B, Hq, Hkv, d, window_left, scale, num_splits, workspace, workspace_bytes, status_dev,
                      out, lse, stream);
}

int sfa_kv_append_kvcache(const void *k_new, const void *v_new, int seqlen_new, void *k_cache, void *v_cache,
                          int batch_cache, int seqlen_cache, const int32_t *cache_batch_idx,
                          const int32_t *cache_seqlens, int B, int Hkv, int d, int32_t *status_dev,
                          sfa_stream_t stream)
{
    return sfa_kv_append(k_new, v_new, seqlen_new, k_cache, v_cache, cache_batch_idx, 1, batch_cache, seqlen_cache,
                         cache_seqlens, B, Hkv, d, status_dev, stream);
}

size_t sfa_window_fwd_workspace_size(void)
{
    return 256;
}

int sfa_window_fwd(const void *q, const void *k, const void *v, const int32_t *cu_seqlens_q,
                   const int32_t *cu_seqlens_k, int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                   int Hq, int Hkv, int d, int causal, int window_left, int window_right,
                   const int32_t *window_left_per_head, const int32_t *window_right_per_head, float scale,
                   void *workspace, size_t workspace_bytes, int32_t *status_dev, void *out, float *lse,
                   sfa_stream_t stream)
{
    g_last_launches = 0;
    // The window kernel tiles keys in 64-token blocks; no selection (topk 1 only sizes the geometry).
    FwdGeom g;
    int rc = fwd_geometry(batch, max_seqlen_q, max_seqlen_k, total_q, Hq, Hkv, d, 1, 64, g);
    if (rc != SFA_OK) return rc;
    if ((rc = fwd_common_checks(cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k, causal,
                                window_left, window_right)) != SFA_OK)
        return rc;
    if (total_q == 0 || batch == 0) return SFA_OK;
    if (!q || !k || !v || !out || !lse || !workspace) return SFA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SFA_ERR_INVALID_ARG;
    if (total_k == 0) return SFA_ERR_UNSUPPORTED;
    if (workspace_bytes < sfa_window_fwd_workspace_size()) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (!fwd_pipe_fits(g, kPipeWindow)) return SFA_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    CUtensorMap tq, tk, tv;
    if (!encode_3d(tq, q, g.d, g.Hq, g.total_q, g.G, g.Tq)) return SFA_ERR_CUDA;
    if (!encode_3d(tk, k, g.d, g.Hkv, total_k, 1, g.bs)) return SFA_ERR_CUDA;
    if (!encode_3d(tv, v, g.d, g.Hkv, total_k, 1, g.bs)) return SFA_ERR_CUDA;
    FwdAttendParams p{};
    p.cu_q = cu_seqlens_q;
    p.cu_k = cu_seqlens_k ? cu_seqlens_k : cu_seqlens_q;
    p.batch = g.batch;
    p.total_q = g.total_q;
    p.Hq = g.Hq;
    p.Hkv = g.Hkv;
    p.G = g.G;
    p.Tq = g.Tq;
    p.nqt = g.nqt;
    p.topk = g.topk;
    p.umax = g.umax;
    p.causal = causal;
    p.wl = window_left;
    p.wr = window_right;
    p.wl_head = window_left_per_head;
    p.wr_head = window_right_per_head;
    const double sc = scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)g.d);
    p.scale_log2 = (float)(sc * 1.4426950408889634);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    p.status = status_dev;
    p.tiles = g.tiles;
    p.tile_counter = static_cast<int32_t *>(workspace);
    p.bs = g.bs;
    p.max_sq = g.max_sq;
    p.nblk_max = g.nblk_max;
    if (cudaMemsetAsync(p.tile_counter, 0, 2 * sizeof(int32_t), st) != cudaSuccess) return SFA_ERR_CUDA;
    if (launch_fwd_attend_pipe(g, p, kPipeWindow, tq, tk, tv, st) != cudaSuccess) return SFA_ERR_CUDA;
    g_last_launches = 1;
    return SFA_OK;
}

int sfa_gated_combine(const void *o_cmp, const float *g_cmp, const void *o_slc, const float *g_slc, const void *o_win,
                      const float *g_win, int total_q, int Hq, int d, void *out, sfa_stream_t stream)
{
    g_last_launches = 0;
    if (total_q < 0 || Hq <= 0) return SFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SFA_ERR_UNSUPPORTED;
    CombineParams p{};
    const void *os[3] = {o_cmp, o_slc, o_win};
    const float *gs[3] = {g_cmp, g_slc, g_win};
    int given = 0;
    for (int b = 0; b < 3; ++b) {
        if (!os[b] || !gs[b]) continue;
        if (!aligned16(os[b])) return SFA_ERR_INVALID_ARG;
        p.o[given] = static_cast<const __nv_bfloat16 *>(os[b]);
        p.g[given] = gs[b];
        ++given;
    }
    if (given == 0) return SFA_ERR_INVALID_ARG;
    if (total_q == 0) return SFA_OK;
    if (!out || !aligned16(out)) return SFA_ERR_INVALID_ARG;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.rows = (int64_t)total_q * Hq;
    if (launch_gated_combine(p, d, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SFA_ERR_CUDA;
    g_last_launches = 1;
    return SFA_OK;
}

const char *sfa_status_string(int status)
{
    switch (status) {
    case SFA_OK: return "SFA_OK";
    case SFA_ERR_INVALID_ARG: return "SFA_ERR_INVALID_ARG: invalid argument";
    case SFA_ERR_UNSUPPORTED: return "SFA_ERR_UNSUPPORTED: valid but not supported by this library";
    case SFA_ERR_WORKSPACE_TOO_SMALL: return "SFA_ERR_WORKSPACE_TOO_SMALL: workspace below the required size";
    case SFA_ERR_CUDA: return "SFA_ERR_CUDA: a CUDA launch or driver call failed";
    default: return "unknown sfa_status";
    }
}

int sfa_last_launch_count(void)
{
    return g_last_launches;
}

}  // extern "C"
