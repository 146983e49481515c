/*
 * sfa.h — C ABI of libsfa.so: top-k sparse FlashAttention forward on NVIDIA B200 (sm_100a).
 *
 * Two operations, each also available as its separate stages:
 *
 *   sfa_fwd     varlen prefill.  Every query token attends only to the key blocks its
 *               (token, kv head) selection lists, shared by the G = Hq/Hkv query heads of
 *               that kv head.  Sources: the Ascend "Sparse FlashAttention" article (ggplus
 *               blog post), section "这到底是个啥？Sparse FlashAttention架构初探" — gather the
 *               K/V rows named by the top-k indices into a compact sub-matrix and run plain
 *               attention on those entries only; the "Relaxed-System-Lab/Flash-Sparse-Attention"
 *               project page, quick-start (block_size / topk / init_blocks / local_blocks NSA
 *               selection, cu_seqlens varlen input); flash-attention-npu "FlashAttention v2"
 *               docstrings of flash_attn_varlen_func (layouts, bottom-right causal mask, window,
 *               GQA mapping, softmax_lse).
 *   sfa_decode  paged top-k decode, one query token per sequence.  Sources: the
 *               Flash-Sparse-Attention README (gitcode mirror), feature list ("Top-k gather
 *               KV-cache decode", "Split-KV", "Paged Attention"); flash-attention-npu
 *               flash_attn_with_kvcache docstrings (paged cache + block_table, cache_seqlens,
 *               num_splits with 0 = automatic, softmax_lse).
 *
 * Built around them, each documented at its declaration: the backward (sfa_bwd), the NSA
 * sliding-window branch and gated mix (sfa_window_fwd, sfa_gated_combine), the decode over FP8
 * caches (sfa_decode_fp8), an allocation-free decode (sfa_decode_noalloc), decode and KV append
 * over non-paged caches addressed by cache_batch_idx (sfa_decode_kvcache, sfa_kv_append_kvcache),
 * the paged KV append (sfa_kv_append) and the decode index producer (sfa_index_topk).
 *
 * Semantics common to both (the plain reading of those pages):
 *   - q head h reads kv head h / (Hq/Hkv); Hq must be a multiple of Hkv.
 *   - For a query at local position i of a sequence with lengths (sq, sk), delta = sk - sq.
 *     Key j is kept iff it is selected and  causal => j <= i+delta;  window_left >= 0 =>
 *     j >= i+delta-window_left;  window_right >= 0 => j <= i+delta+window_right.
 *   - Softmax over the kept keys of  scale * q.k ; scale <= 0 means 1/sqrt(d).
 *   - A row with no kept key outputs exactly 0 and lse = -inf.
 *   - lse is the natural-log logsumexp of scale*q.k over the kept keys.
 *   - A selection is a set: -1 slots are padding, duplicates and order do not matter.
 *
 * Conventions of this ABI:
 *   - Every pointer argument except the workspace size queries is a DEVICE pointer of the
 *     current CUDA device, owned by the caller.  The library allocates no device memory,
 *     never synchronises the host and launches everything on `stream` (cudaStream_t; NULL is
 *     the legacy default stream), so the calls can be captured in a CUDA graph.
 *   - bf16 tensors are contiguous row-major with the last dimension contiguous, 16-byte
 *     aligned base addresses.
 *   - Return value: a synchronous sfa_status.  Argument errors are detected on the host
 *     before anything is launched.  SFA_ERR_CUDA means a launch failed (the CUDA error is
 *     left for the caller's next runtime call to report).
 *   - Data errors found on the device are OR-ed into *status_dev (int32, may be NULL) as
 *     SFA_DEV_* bits and the offending entry is ignored: an out-of-range block/token id,
 *     a block_table entry outside [0, num_pages), a sequence longer than the bound given,
 *     or a pipeline wait that exceeded its time limit (the kernel then stops early; its
 *     outputs are undefined).  Kernels never trap.
 *   - Calls on one workspace must not overlap in time (use one workspace per stream).
 *   - A workspace starts on a 256-byte boundary (as cudaMalloc and the PyTorch caching
 *     allocator return); another base is SFA_ERR_INVALID_ARG.
 */
#ifndef SFA_H_
#define SFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sfa_stream_t; /* same type as cudaStream_t */

typedef enum sfa_status {
    SFA_OK = 0,
    SFA_ERR_INVALID_ARG = 1,         /* NULL pointer, negative size, Hq % Hkv != 0, misaligned base */
    SFA_ERR_UNSUPPORTED = 2,         /* valid but outside what this library supports: see the limits below */
    SFA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes below the matching *_workspace_size() */
    SFA_ERR_CUDA = 4                 /* a CUDA launch or driver call failed */
} sfa_status;

enum {
    SFA_DEV_BAD_INDEX = 1,  /* a block / token id neither -1 nor inside its sequence: ignored */
    SFA_DEV_BAD_PAGE = 2,   /* a block_table entry outside [0, num_pages): its tokens are dropped */
    SFA_DEV_TIMEOUT = 4,    /* a pipeline wait passed its time limit: outputs undefined */
    SFA_DEV_BAD_SEQLEN = 8  /* a sequence longer than max_seqlen_q/k (or than the block table): the
                               excess is not computed / its ids are treated as out of range */
};

/* Supported by this library: bf16 inputs; d in {64, 128}; prefill block_size in {32, 64},
 * 1 <= topk <= 128, G = Hq/Hkv <= 128, ceil(max_seqlen_k / block_size) <= 65536;
 * decode G <= 16, page_size >= 1, 1 <= topk_tok <= 65536, max_pages_per_seq*page_size
 * <= 2^20; backward the forward's d and block_size; KV append d a multiple of 8; index top-k G <= 1024,
 * max_pages_per_seq*page_size <= 2^20.  Anything else returns SFA_ERR_UNSUPPORTED. */

/* ----------------------------------------------------------------------------------------
 * Prefill
 * -------------------------------------------------------------------------------------- */

/* Bytes of device workspace sfa_fwd / sfa_fwd_prep / sfa_fwd_attend need for these sizes
 * (0 only when total_q == 0).  max_seqlen_q / max_seqlen_k bound every sequence's length. */
size_t sfa_fwd_workspace_size(int batch, int max_seqlen_q, int max_seqlen_k, int total_q,
                              int Hq, int Hkv, int d, int topk, int block_size);

/* Byte offsets, inside that workspace, of the canonical selection written by sfa_fwd_prep:
 * sel_c int32 (total_q, Hkv, topk) — per (token, kv head) the ascending distinct block ids
 * that are blocks of the sequence and hold at least one key the mask keeps, then -1 — and
 * cnt int32 (total_q, Hkv) — how many.  Returns SFA_OK or SFA_ERR_INVALID_ARG. */
int sfa_fwd_workspace_offsets(int batch, int max_seqlen_q, int max_seqlen_k, int total_q,
                              int Hq, int Hkv, int d, int topk, int block_size,
                              size_t *off_sel_c, size_t *off_cnt);

/* Full prefill forward: the result of sfa_fwd_prep followed by sfa_fwd_attend on the same
 * workspace (when the call needs no block-major plan it is one kernel that canonicalises each
 * query tile's selections itself; the workspace then only carries its tile counter).
 *   q            bf16 (total_q, Hq, d)
 *   k, v         bf16 (total_k, Hkv, d)
 *   cu_seqlens_q int32 (batch+1), prefix sums from 0; cu_seqlens_k likewise, or NULL for
 *                "same as q" (then total_k must equal total_q)
 *   sel_idx      int32 (total_q, Hkv, topk): block ids of the sequence's own K coordinates,
 *                block s = keys [s*block_size, min((s+1)*block_size, sk)); -1 = unused slot
 *   out          bf16 (total_q, Hq, d);  lse  fp32 (Hq, total_q)
 * max_seqlen_q/k are host-side bounds used to size the grid (no device->host read). */
int sfa_fwd(const void *q, const void *k, const void *v,
            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
            int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
            int Hq, int Hkv, int d,
            const int32_t *sel_idx, int topk, int block_size,
            int causal, int window_left, int window_right, float scale,
            void *workspace, size_t workspace_bytes, int32_t *status_dev,
            void *out, float *lse, sfa_stream_t stream);

/* Stage 1 alone: canonicalise the selection (validate, drop padding / out-of-range ids /
 * blocks with no kept key, dedupe, sort ascending, count) and build, per query tile, the
 * ascending union of its rows' blocks.  Writes only the workspace. */
int sfa_fwd_prep(const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                 int batch, int max_seqlen_q, int max_seqlen_k, int total_q,
                 int Hq, int Hkv, int d, const int32_t *sel_idx, int topk, int block_size,
                 int causal, int window_left, int window_right,
                 void *workspace, size_t workspace_bytes, int32_t *status_dev, sfa_stream_t stream);

/* Stage 2 alone: the attention kernel (TMA gather of K/V blocks, tcgen05 QK^T and PV with
 * TMEM accumulators, masked online softmax, epilogue) on a workspace filled by
 * sfa_fwd_prep with the same arguments. */
int sfa_fwd_attend(const void *q, const void *k, const void *v,
                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                   int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                   int Hq, int Hkv, int d, int topk, int block_size,
                   int causal, int window_left, int window_right, float scale,
                   void *workspace, size_t workspace_bytes, int32_t *status_dev,
                   void *out, float *lse, sfa_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Prefill backward
 * The gradients of sfa_fwd's attention: with P the probabilities recomputed from the forward's
 * lse, dP = dO V^T, dS = P o (dP - rowsum(dO o O)), dQ = scale dS K, dK = scale dS^T Q and
 * dV = P^T dO, every product restricted to the keys each row selected and its mask keeps (the
 * FlashAttentionScoreGrad case study of the Ascend "Sparse FlashAttention" article for P, dP, dS
 * and dQ; dK and dV by the same chain rule; the flash-sparse-attention README's backward example
 * for what is differentiated).
 * -------------------------------------------------------------------------------------- */

/* Bytes of device workspace sfa_bwd needs (0 when total_q == 0 or the sizes are unsupported).
 * It grows with batch * Hkv * ceil(max_seqlen_k / block_size) * ceil(max_seqlen_q / 32) (the
 * token bitmaps that invert the selection) and with total_q * Hkv * topk. */
size_t sfa_bwd_workspace_size(int batch, int max_seqlen_q, int max_seqlen_k, int total_q,
                              int Hq, int Hkv, int d, int topk, int block_size);

/* Backward of sfa_fwd.  Inputs are sfa_fwd's (same layouts, selection, mask, scale) plus:
 *   out   bf16 (total_q, Hq, d), the forward's output;  lse fp32 (Hq, total_q), its LSE
 *   dout  bf16 (total_q, Hq, d), the gradient of the loss with respect to out
 * Outputs (written in full; the caller owns them): dq bf16 (total_q, Hq, d), dk and dv bf16
 * (total_k, Hkv, d).  A key no row keeps gets dk = dv = 0; a row that keeps no key gets dq = 0.
 * Sizes as sfa_fwd (d in {64, 128}, block_size in {32, 64}), and a tile's block union must fit the
 * dQ kernel's shared memory (else SFA_ERR_UNSUPPORTED).  Deterministic: the sums run
 * in a fixed order whatever the timing.  Seven kernels and one memset on `stream`; status bits as
 * sfa_fwd (SFA_DEV_BAD_SEQLEN also when a token of a sequence is past max_seqlen_q). */
int sfa_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
            const float *lse, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
            int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
            int Hq, int Hkv, int d, const int32_t *sel_idx, int topk, int block_size,
            int causal, int window_left, int window_right, float scale,
            void *workspace, size_t workspace_bytes, int32_t *status_dev,
            void *dq, void *dk, void *dv, sfa_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Paged top-k decode
 * -------------------------------------------------------------------------------------- */

/* The split count sfa_decode uses for num_splits (0 = automatic choice). */
int sfa_decode_num_splits(int B, int Hq, int Hkv, int d, int topk_tok, int num_splits);

/* Bytes of device workspace for sfa_decode with these sizes; num_splits as passed there. */
size_t sfa_decode_workspace_size(int B, int Hq, int Hkv, int d, int topk_tok, int num_splits);

/* Byte offsets inside the decode workspace of the canonical token sets written by
 * sfa_decode_prep: tok_c int32 (B, Hkv, topk_tok) ascending distinct positions in
 * [0, cache_seqlens[b]) (and >= L-1-window_left when window_left >= 0), then -1; and
 * cnt int32 (B, Hkv). */
int sfa_decode_workspace_offsets(int B, int Hq, int Hkv, int d, int topk_tok, int num_splits,
                                 size_t *off_tok_c, size_t *off_cnt);

/* Paged top-k decode = split-KV attention and LSE combine.  Each (sequence, kv head)'s
 * selection is deduplicated and sorted inside the split kernel when topk_tok <= 2048; longer
 * selections first go through the prep kernel.  The splits of one (sequence, kv head) run six
 * to a CTA; with num_splits <= 6 the CTA also merges them (one launch), otherwise a combine
 * kernel follows.
 *   q             bf16 (B, Hq, d): the new token of each sequence, at position L_b - 1
 *   k_cache,
 *   v_cache       bf16 (num_pages, page_size, Hkv, d)
 *   block_table   int32 (B, max_pages_per_seq): logical page p of sequence b lives in
 *                 physical page block_table[b][p]
 *   cache_seqlens int32 (B): L_b, tokens in the cache (the new token included)
 *   sel_tok_idx   int32 (B, Hkv, topk_tok): logical token positions, -1 = unused slot
 *   window_left   -1 = unbounded, else keep positions >= L_b - 1 - window_left
 *   num_splits    0 = automatic, else the number of key chunks per (b, kv head)
 *   out           bf16 (B, Hq, d);  lse  fp32 (B, Hq) */
int sfa_decode(const void *q, const void *k_cache, const void *v_cache,
               const int32_t *block_table, int max_pages_per_seq, int num_pages, int page_size,
               const int32_t *cache_seqlens, const int32_t *sel_tok_idx, int topk_tok,
               int B, int Hq, int Hkv, int d, int window_left, float scale, int num_splits,
               void *workspace, size_t workspace_bytes, int32_t *status_dev,
               void *out, float *lse, sfa_stream_t stream);

/* Stage 1 alone: canonical token sets into the workspace. */
int sfa_decode_prep(const int32_t *cache_seqlens, const int32_t *sel_tok_idx, int topk_tok,
                    int max_pages_per_seq, int page_size, int B, int Hq, int Hkv, int d,
                    int window_left, int num_splits,
                    void *workspace, size_t workspace_bytes, int32_t *status_dev, sfa_stream_t stream);

/* The attention stage alone, on the canonical sets sfa_decode_prep wrote into the workspace
 * (same arguments): the split kernel, which gathers through block_table and, with at most six
 * splits, also merges them; beyond six splits the LSE combine kernel follows. */
int sfa_decode_attend(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_table, int max_pages_per_seq, int num_pages, int page_size,
                      int topk_tok, int B, int Hq, int Hkv, int d, float scale, int num_splits,
                      void *workspace, size_t workspace_bytes, int32_t *status_dev,
                      void *out, float *lse, sfa_stream_t stream);

/* Paged top-k decode over FP8 caches: k_cache and v_cache hold FP8 E4M3 codes (1 byte per value,
 * (num_pages, page_size, Hkv, d), 16-byte aligned) and the cached value of sequence b, kv head h is
 * code * k_descale[b * Hkv + h] (keys) or code * v_descale[b * Hkv + h] (values): the descale
 * convention of the FlashAttention-3 docstrings (flash-attention-npu page, k_descale / v_descale of
 * shape (batch, kv heads)); FP8 caches are in the Flash-Sparse-Attention README feature list ("Fused
 * Quant").  k_descale / v_descale: fp32 device arrays (B, Hkv), or NULL for 1.  Every other argument,
 * the workspace (sfa_decode_workspace_size), the semantics, the launches and the status bits are
 * sfa_decode's; q, out and lse stay bf16 / fp32.  The E4M3 values are exact in bf16, so the kernel
 * computes with the cached values themselves: half the bytes per gathered row. */
int sfa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const float *k_descale,
                   const float *v_descale, const int32_t *block_table, int max_pages_per_seq, int num_pages,
                   int page_size, const int32_t *cache_seqlens, const int32_t *sel_tok_idx, int topk_tok, int B,
                   int Hq, int Hkv, int d, int window_left, float scale, int num_splits, void *workspace,
                   size_t workspace_bytes, int32_t *status_dev, void *out, float *lse, sfa_stream_t stream);

/* Paged top-k decode for callers that cannot allocate device memory.  The pages have no
 * counterpart to this call: it exists for callers such as serving engines whose device memory
 * pool is fixed before serving and forbids later allocation, or plugin hooks that receive only
 * input and output pointers.  Same arguments, semantics and kernels as sfa_decode, without the
 * workspace: the scratch lives in a static device array of 8 MiB that a GPU keeps, once it holds
 * it, until the process exits.
 *   - Returns SFA_ERR_WORKSPACE_TOO_SMALL when sfa_decode_workspace_size() of these arguments
 *     exceeds 8 MiB (nothing is launched).  It calls no allocation routine of any kind.
 *   - q (and every other tensor) must live on the current device; a q on another device, or a
 *     pointer the runtime does not know as device memory, returns SFA_ERR_INVALID_ARG.
 *   - The first call on each device looks the array's address up on that device (with it
 *     current).  With CUDA's lazy module loading (the default since CUDA 12.2) that lookup is
 *     also when the module is loaded onto the device and its 8 MiB are reserved, so the first
 *     call can fail if the device is out of memory.  Make that first call during start-up: before
 *     a memory pool is sized to take the rest of the device, and before any stream capture.
 *   - Every call on a device shares the one array, and each call rewrites every byte it reads
 *     from it, so nothing carries over between calls; two calls that overlap on the GPU
 *     (other streams, other host threads) race on it and give undefined results. */
int sfa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_table, int max_pages_per_seq, int num_pages, int page_size,
                       const int32_t *cache_seqlens, const int32_t *sel_tok_idx, int topk_tok,
                       int B, int Hq, int Hkv, int d, int window_left, float scale, int num_splits,
                       int32_t *status_dev, void *out, float *lse, sfa_stream_t stream);

/* Index producer for the decode (Lightning-Indexer style: the "Sparse FlashAttention" post on Ascend,
 * section "那个叫Lightning Indexer的家伙" — the current query scored against every key with FP8
 * dot products, the top-k positions kept).  Per (sequence b, kv head): score_j = sum over the G query
 * heads of the group of e4m3(q_h) . e4m3(k_j) for every cache position j < cache_seqlens[b]
 * (E4M3: round to nearest even, saturated at +-448, no scale factors), computed exactly; the last
 * n_local positions are always kept, the others by descending score, a tie to the lower position.
 *   q          bf16 (B, Hq, d);  k_cache bf16 (num_pages, page_size, Hkv, d);  block_table as sfa_decode
 *   sel_out    int32 (B, Hkv, topk): ascending positions, -1 padded — the sel_tok_idx of sfa_decode
 *   workspace  sfa_index_topk_workspace_size() bytes (one 64-bit key per position)
 * Positions whose page id is outside [0, num_pages) are no candidates (SFA_DEV_BAD_PAGE); a length
 * past the block table is cut to it (SFA_DEV_BAD_SEQLEN).  d in {64, 128}; max_pages_per_seq *
 * page_size <= 2^20; G = Hq / Hkv <= 1024 (the exactness bound).  Two kernels: the scores (one CTA per (sequence, kv head, run of 4096
 * positions)), then the selection (one CTA per (sequence, kv head)). */
size_t sfa_index_topk_workspace_size(int B, int Hkv, int max_pages_per_seq, int page_size);
int sfa_index_topk(const void *q, const void *k_cache, const int32_t *block_table, int max_pages_per_seq,
                   int num_pages, int page_size, const int32_t *cache_seqlens, int B, int Hq, int Hkv, int d, int topk,
                   int n_local, void *workspace, size_t workspace_bytes, int32_t *status_dev, int32_t *sel_out,
                   sfa_stream_t stream);

/* In-place append of new keys / values to the paged cache, as the k / v arguments of
 * flash_attn_with_kvcache (flash-attention-npu docstrings): row j of sequence b goes to logical
 * position cache_seqlens[b] + j, i.e. page block_table[b][pos / page_size], row pos % page_size.
 *   k_new, v_new  bf16 (B, seqlen_new, Hkv, d);  k_cache, v_cache  bf16 (num_pages, page_size, Hkv, d)
 * cache_seqlens is read, not updated: a decode over the appended cache passes cache_seqlens +
 * seqlen_new.  A position past the block table (SFA_DEV_BAD_SEQLEN) or whose page id is outside
 * [0, num_pages) (SFA_DEV_BAD_PAGE) is not written.  d a multiple of 8; 16-byte aligned tensors.
 * One kernel (none when B or seqlen_new is 0). */
int sfa_kv_append(const void *k_new, const void *v_new, int seqlen_new, void *k_cache, void *v_cache,
                  const int32_t *block_table, int max_pages_per_seq, int num_pages, int page_size,
                  const int32_t *cache_seqlens, int B, int Hkv, int d, int32_t *status_dev, sfa_stream_t stream);

/* Non-paged caches with a batch index, the cache_batch_idx argument of flash_attn_with_kvcache
 * (flash-attention-npu docstrings): k_cache / v_cache bf16 (batch_cache, seqlen_cache, Hkv, d) and
 * cache_batch_idx int32 (B): sequence b reads and appends row j at k_cache[cache_batch_idx[b]][j].
 * (The docstring's default, cache_batch_idx = None, is 0, 1, ..., B-1: pass that array.)  Such a
 * cache is the paged cache of batch_cache pages of seqlen_cache rows whose block table is
 * cache_batch_idx itself (one page per sequence), so these calls are sfa_decode / sfa_kv_append with
 * block_table = cache_batch_idx, max_pages_per_seq = 1, num_pages = batch_cache, page_size =
 * seqlen_cache: the same kernels, launches, workspace (sfa_decode_workspace_size), limits
 * (seqlen_cache <= 2^20) and status bits.  An index outside [0, batch_cache) sets
 * SFA_DEV_BAD_PAGE and drops the sequence's rows (decode: out 0, lse -inf; append: nothing
 * written); cache_seqlens[b] (+ the new rows) past seqlen_cache sets SFA_DEV_BAD_SEQLEN and the
 * excess is cut.  As the docstring warns, an append whose cache_batch_idx repeats an index writes
 * the same rows from several sequences: which one lands is unspecified. */
int sfa_decode_kvcache(const void *q, const void *k_cache, const void *v_cache, int batch_cache, int seqlen_cache,
                       const int32_t *cache_batch_idx, const int32_t *cache_seqlens, const int32_t *sel_tok_idx,
                       int topk_tok, int B, int Hq, int Hkv, int d, int window_left, float scale, int num_splits,
                       void *workspace, size_t workspace_bytes, int32_t *status_dev, void *out, float *lse,
                       sfa_stream_t stream);
int sfa_kv_append_kvcache(const void *k_new, const void *v_new, int seqlen_new, void *k_cache, void *v_cache,
                          int batch_cache, int seqlen_cache, const int32_t *cache_batch_idx,
                          const int32_t *cache_seqlens, int B, int Hkv, int d, int32_t *status_dev,
                          sfa_stream_t stream);

/* ---------------------------------------------------------------------------------------
 * NSA branches beside the selected attention (the "Relaxed-System-Lab/Flash-Sparse-Attention"
 * project page, quick-start: window_size alongside block_size / topk; the Flash-Sparse-Attention
 * README feature list: causal and local window attention, gated attention).
 * --------------------------------------------------------------------------------------- */

/* Bytes of device workspace sfa_window_fwd needs (a tile counter it clears itself). */
size_t sfa_window_fwd_workspace_size(void);

/* Sliding-window branch: every query attends to all keys its mask keeps — the common semantics
 * above with every key selected (bottom-right causal limit when causal; window_left /
 * window_right as in the flash-attention-npu docstrings, -1 = unbounded; a plain causal or full
 * attention when no window is given).  window_left_per_head / window_right_per_head: int32 (Hq)
 * device arrays or NULL; when given, q head h uses element h instead of window_left /
 * window_right (negative = unbounded) — per-head windows as in the Flash-Sparse-Attention README
 * ("Flex Local Window Attention").  Layouts, lengths, status word and errors as sfa_fwd; there is
 * no selection.  out bf16 (total_q, Hq, d); lse fp32 (Hq, total_q).  One kernel. */
int sfa_window_fwd(const void *q, const void *k, const void *v,
                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                   int batch, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                   int Hq, int Hkv, int d, int causal, int window_left, int window_right,
                   const int32_t *window_left_per_head, const int32_t *window_right_per_head, float scale,
                   void *workspace, size_t workspace_bytes, int32_t *status_dev,
                   void *out, float *lse, sfa_stream_t stream);

/* Gated mix of the branch outputs: out[t,h,:] = sum over the given branches c of
 * g_c[t,h] * o_c[t,h,:] (fp32 arithmetic, bf16 round-to-nearest result).  Each o_c is bf16
 * (total_q, Hq, d) and each g_c fp32 (total_q, Hq), e.g. the compressed, selected and window
 * branches with the caller's gate values; a branch whose o or g pointer is NULL is left out (at
 * least one must be given).  d in {64, 128}; 16-byte aligned bf16 tensors.  One kernel. */
int sfa_gated_combine(const void *o_cmp, const float *g_cmp, const void *o_slc, const float *g_slc,
                      const void *o_win, const float *g_win, int total_q, int Hq, int d, void *out,
                      sfa_stream_t stream);

/* Human-readable name of an sfa_status value (static string). */
const char *sfa_status_string(int status);

/* Number of kernel launches the last successful call on this host thread made (prefill: 1,
 * or 6 when the call uses the block-major schedule; decode: 1 with at most 6 splits, else 2,
 * plus 1 when topk_tok > 2048; a stage: its own count; window branch, gated mix, KV append, index top-k: 1; backward: 7). */
int sfa_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SFA_H_ */
