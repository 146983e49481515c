// Internal interfaces between the C-ABI host layer (sfa_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "sfa.h"  // include/ is on the include path

namespace sfa {

// ---------------------------------------------------------------------------------------
// Prefill
// ---------------------------------------------------------------------------------------
// A query tile is Tq consecutive tokens of one sequence times the G query heads of one kv
// head: Tq * G <= 128 rows, the M dimension of one tcgen05 MMA.  Tiles are numbered
// tile = (qt_rev * batch + b) * Hkv + hk with qt = nqt - 1 - qt_rev, so the tiles deepest
// into their sequences (the ones with the most blocks under a causal mask) start first.
// Block-major windows: a tile's blocks that at least a quarter of its 128 rows select ("dense", at
// most kDenseMax of them, ascending) run query-major for the tile; the rest go to block-major items.
constexpr int kDenseMax = 32;

struct FwdGeom {
    int batch, max_sq, max_sk, total_q, Hq, Hkv, d, topk, bs;
    int G, Tq, nqt, tiles, nblk_max, umax;
    // Block-major schedule for sparse query windows (inv = 0 when this call cannot use it):
    // a window is W consecutive tokens of one sequence; for one (window, sequence, kv head)
    // group the prep lists, per selected block, the window's tokens that selected it, and cuts
    // those lists into items of at most Tq tokens.
    int inv, W, nwin, groups;
    int64_t cap_items;
    size_t off_sel_c, off_cnt, off_ucnt, off_union, off_tilectr;
    size_t off_zero, zero_bytes;  // the part of the workspace cleared before every prep
    size_t off_ctrl, off_gstat, off_tcount, off_gfirst, off_duni, off_dcnt, off_dsel, off_items, off_pml, off_po;
    size_t bytes;
};

// Control words of the block-major schedule (cleared before every prep).
struct InvCtrl {
    int item_total;  // items planned so far
    int pad[3];
};

// Per (window, sequence, kv head) group: selected row-blocks and union tile row-blocks.
struct GroupStat {
    unsigned long long useful, uni;
};

// One block-major item as stored in the workspace and copied whole into shared memory.
struct InvItem {
    int4 rec;      // {b * Hkv + hk, block, first K row of the sequence, tokens}; tokens < 0 ends the work
    int tok[128];  // (token << 7) | position of the block in the token's canonical list
};

struct FwdPrepParams {
    const int32_t *cu_q, *cu_k, *sel;
    int32_t *tile_counter;  // cleared here (two ints) for the attend kernel
    int batch, Hkv, topk, bs, causal, wl, wr, Tq, nqt, umax, max_sq, nblk_max, total_q;
    int32_t *sel_c, *cnt, *ucnt, *uni;
    // block-major statistics (nullptr when the schedule is off): per group, and per tile the number of
    // its tokens that selected each block ([tiles][nblk_max])
    int W;
    GroupStat *gstat;
    int32_t *tcount;
    // the tile's dense blocks ([tiles][kDenseMax], count per tile) and per (token, kv head) two masks:
    // the dense blocks it selected (bit j: the tile's dense block j) and its canonical entries that are
    // dense (bit e: entry e), [2][total_q * Hkv]
    int32_t *duni, *dcnt;
    uint32_t *dsel;
    int32_t *status;
};

struct FwdPlanParams {
    int32_t *ucnt;
    const GroupStat *gstat;
    int32_t *tcount;  // per-tile counts in; for block-major windows, each tile's first list position out
    int32_t *gfirst;
    int batch, Hkv, Tq, nqt, W, nblk_max;
    const int32_t *cu_q, *cu_k;
    InvItem *items;
    InvCtrl *ctrl;
};

struct FwdScatterParams {
    const int32_t *cu_q, *sel_c, *cnt, *ucnt, *gfirst;
    const int32_t *tcount;  // each tile's first position in every block's token list
    const uint32_t *dmask;  // per (token, kv head): canonical entries of dense blocks (not in items)
    int batch, Hkv, topk, Tq, nqt, W, nblk_max;
    InvItem *items;
};

struct FwdAttendParams {
    const int32_t *cu_q, *cu_k;
    const int32_t *sel_c, *cnt, *ucnt, *uni;
    int batch, total_q, Hq, Hkv, G, Tq, nqt, topk, umax, tiles;
    // Selections as given (the pipelined kernel's fused mode canonicalizes them itself)
    const int32_t *sel;
    int bs, max_sq, nblk_max;
    int32_t *tile_counter;  // next query tile to hand out; [1] counts CTAs done.  The prep kernel
                            // clears both; the attend kernel's last CTA clears them again.
    int causal, wl, wr;
    const int32_t *wl_head, *wr_head;  // window mode: per-q-head windows (nullptr: wl / wr for all heads)
    float scale_log2;  // softmax scale * log2(e)
    __nv_bfloat16 *out;
    float *lse;
    int32_t *status;
    // block-major schedule
    const __nv_bfloat16 *q;  // (total_q, Hq, d): the block-major kernel gathers its rows with cp.async
    const InvItem *items;
    InvCtrl *ctrl;
    __nv_bfloat16 *po;  // partial outputs, (total_q, Hq, topk, d) bf16, normalised
    float2 *pml;        // partial (max, sum) in the base-2 scaled domain, (total_q, Hq, topk)
    // dense blocks of block-major tiles (the query-major kernel attends over them and leaves its result
    // in out / lse, one more partial for the merge); nullptr when the schedule is off
    const int32_t *duni, *dcnt;
    const uint32_t *dsel, *dmask;
};

// ---------------------------------------------------------------------------------------
// Prefill backward
// ---------------------------------------------------------------------------------------
// dQ runs query-major over the forward's tiles and unions (the prep kernel's canonical lists);
// dK / dV run block-major: for every (sequence, kv head, key block) "row" the ascending list of
// the sequence's tokens that selected the block, cut into pieces of at most kBwdPieceChunks
// chunks of Tq tokens.  Each piece of a row longer than one piece writes an fp32 partial; the
// piece that finishes last sums the row's partials in piece order, so the result does not depend
// on timing and no piece waits for another.
constexpr int kBwdPieceChunks = 16;

struct BwdPiece {
    int row;        // (b * Hkv + hk) * nblk_max + block
    int tok_begin;  // first entry of the row's token list this piece takes
    int ntok;       // entries it takes
    int idx, npieces;
    int slot;       // first of the row's npieces partial slots (-1: a one-piece row)
    int pad[2];
};

struct BwdCtrl {
    int npieces;  // pieces planned
    int counter;  // next piece to hand out
    int pad[2];
};

struct BwdGeom {
    FwdGeom f;                 // query tiling, canonical lists and unions (block-major schedule off)
    int R, words;              // rows = batch * Hkv * nblk_max; bitmap words per row = ceil(max_sq / 32)
    int64_t max_pieces, max_slots;
    size_t off_delta, off_bits, off_rowcnt, off_flags, off_ctrl, off_rowoff, off_toks, off_pieces, off_part;
    size_t off_zero, zero_bytes;  // bitmap, row counts and partial flags: cleared before every call
    size_t bytes;
};

struct BwdParams {
    const __nv_bfloat16 *q, *out, *dout;  // q and dout: the dK/dV kernel gathers their rows
    const float *lse;     // (Hq, total_q), natural log
    const int32_t *cu_q, *cu_k;
    const int32_t *sel_c, *cnt, *ucnt, *uni;
    int batch, total_q, Hq, Hkv, G, Tq, nqt, topk, umax, tiles, nblk_max, max_sq, words, R;
    int causal, wl, wr;
    float scale, scale_log2;
    float *delta;         // (Hq, total_q): rowsum(dO o O)
    uint32_t *bits;       // [R][words] token bitmaps
    int32_t *rowcnt, *rowoff, *toks;
    BwdPiece *pieces;
    BwdCtrl *ctrl;
    int32_t *flags;       // [max_slots], at a row's first slot: its pieces finished so far
    float *part;          // [max_slots][2][bs][d] partials (dK, dV) of the pieces of multi-piece rows
    int64_t max_pieces, max_slots;
    int32_t *tile_counter;
    __nv_bfloat16 *dq, *dk, *dv;
    int32_t *status;
};

cudaError_t launch_bwd_delta(const BwdGeom &g, const BwdParams &p, cudaStream_t st);
cudaError_t launch_bwd_index(const BwdGeom &g, const BwdParams &p, cudaStream_t st);
cudaError_t launch_bwd_plan(const BwdGeom &g, const BwdParams &p, cudaStream_t st);
cudaError_t launch_bwd_fill(const BwdGeom &g, const BwdParams &p, cudaStream_t st);
cudaError_t launch_bwd_dq(const BwdGeom &g, const BwdParams &p, const CUtensorMap &tq, const CUtensorMap &tdo,
                          const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st);
cudaError_t launch_bwd_dkdv(const BwdGeom &g, const BwdParams &p, const CUtensorMap &tk, const CUtensorMap &tv,
                            cudaStream_t st);
size_t bwd_dq_smem_bytes(const BwdGeom &g);
size_t bwd_dkdv_smem_bytes(const BwdGeom &g);

// ---------------------------------------------------------------------------------------
// Decode
// ---------------------------------------------------------------------------------------
struct DecGeom {
    int B, Hq, Hkv, d, topk, S, G;
    size_t off_tok, off_cnt, off_po, off_plse, bytes;
};

struct DecPrepParams {
    const int32_t *seqlens, *sel;
    int topk, max_len, Hkv, wl;
    int32_t *tok_c, *cnt;
    int32_t *status;
};

struct DecSplitParams {
    const __nv_bfloat16 *q, *kc, *vc;
    const int32_t *bt, *tok_c, *cnt;  // canonical sets from the prep kernel (fused == 0)
    const int32_t *seqlens, *sel;     // raw selections, deduplicated in the kernel (fused == 1)
    int fused, wl;
    int B, max_pages, num_pages, page, Hq, Hkv, G, topk, S;  // CTA c of (b, kv head) runs splits 6c..6c+5
    int page_shift;  // log2(page) when page is a power of two, else -1
    int fp8;         // caches hold E4M3 codes (1 byte per value); kd / vd: descales (B, Hkv) or nullptr (1)
    const float *kd, *vd;
    float scale_log2;
    float *po, *plse;  // partial outputs (B, Hq, S, d) and natural-log lse (B, Hq, S)
    __nv_bfloat16 *out_direct;  // S <= 4: the CTA combines its splits and writes out / lse itself
    float *lse_direct;
    int32_t *status;
};

struct DecCombineParams {
    const float *po, *plse;
    int Hq, S;
    __nv_bfloat16 *out;
    float *lse;
};

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the current device.  The
// limit is a per-device attribute, so the value already set is remembered per (kernel, device)
// under a lock; a launch on another device (or from another host thread) sets it there too.
cudaError_t ensure_smem(const void *kernel, size_t bytes);
template <typename K>
inline cudaError_t ensure_smem_for(K *kernel, size_t bytes)
{
    return ensure_smem(reinterpret_cast<const void *>(kernel), bytes);
}

// Launchers (return the launch's cudaError_t).
// Kernel launch on `st`; with pdl the kernel may start while the previous kernel in the stream is
// finishing (it must call grid_dep_wait() before reading that kernel's results).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 bool pdl, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

cudaError_t launch_fwd_prep(const FwdGeom &g, const FwdPrepParams &p, cudaStream_t st);
cudaError_t launch_fwd_attend(const FwdGeom &g, const FwdAttendParams &p, const CUtensorMap &tq,
                              const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st);
size_t fwd_attend_smem_bytes(const FwdGeom &g);
// Pipelined query-major kernel (tile switches overlapped with the previous tile's tail): whether
// its shared memory (which holds two copies of a tile's union) fits two CTAs per SM for this
// geometry; when it does not, fwd_attend_kernel runs instead.
// mode 0: canonical lists and unions from the prep kernel; 1 (fused): the kernel builds each tile's
// canonical lists and union from the raw selections itself (no prep kernel; the caller clears the
// tile counter), for calls without the block-major schedule; 2 (window): dense attention under the
// causal / window mask, every block holding a key of a row's window selected (no selection at all).
constexpr int kPipePrep = 0, kPipeFused = 1, kPipeWindow = 2;
bool fwd_pipe_fits(const FwdGeom &g, int mode);
cudaError_t launch_fwd_attend_pipe(const FwdGeom &g, const FwdAttendParams &p, int mode, const CUtensorMap &tq,
                                   const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st);
cudaError_t launch_fwd_plan(const FwdGeom &g, const FwdPlanParams &p, cudaStream_t st);
cudaError_t launch_fwd_scatter(const FwdGeom &g, const FwdScatterParams &p, cudaStream_t st);
cudaError_t launch_fwd_attend_inv(const FwdGeom &g, const FwdAttendParams &p, const CUtensorMap &tq,
                                  const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st);
cudaError_t launch_fwd_merge(const FwdGeom &g, const FwdAttendParams &p, cudaStream_t st);
size_t fwd_attend_inv_smem_bytes(const FwdGeom &g);

// Gated mix of up to three branch outputs (o[b] == nullptr: branch absent).
struct CombineParams {
    const __nv_bfloat16 *o[3];
    const float *g[3];
    __nv_bfloat16 *out;
    int64_t rows;  // total_q * Hq
};
cudaError_t launch_gated_combine(const CombineParams &p, int d, cudaStream_t st);

// Decode index producer (exact FP8 scores, top-k positions per (sequence, kv head)).
struct IndexParams {
    const __nv_bfloat16 *q, *kc;  // (B, Hq, d), (num_pages, page, Hkv, d)
    const int32_t *bt, *seqlens;  // (B, max_pages), (B)
    int B, Hq, Hkv, G, d, max_pages, num_pages, page, topk, n_local;
    int64_t max_len;              // max_pages * page: the key array's stride per (sequence, kv head)
    unsigned long long *keys;     // workspace [B * Hkv][max_len]
    int32_t *sel;                 // (B, Hkv, topk)
    int32_t *status;
};
cudaError_t launch_index_topk(const IndexParams &p, cudaStream_t st);

// In-place paged KV-cache append.
struct KvAppendParams {
    const __nv_bfloat16 *k_new, *v_new;  // (B, S, Hkv, d)
    __nv_bfloat16 *k_cache, *v_cache;    // (num_pages, page, Hkv, d)
    const int32_t *bt, *seqlens;         // (B, max_pages), (B)
    int B, S, Hkv, d, max_pages, num_pages, page;
    int32_t *status;
};
cudaError_t launch_kv_append(const KvAppendParams &p, cudaStream_t st);

cudaError_t launch_decode_prep(const DecGeom &g, const DecPrepParams &p, cudaStream_t st);
cudaError_t launch_decode_split(const DecGeom &g, const DecSplitParams &p, cudaStream_t st);
cudaError_t launch_decode_combine(const DecGeom &g, const DecCombineParams &p, cudaStream_t st);
int decode_split_blocks_per_sm(int d);
int decode_split_warps_per_block();
int decode_fused_max_topk();

}  // namespace sfa
