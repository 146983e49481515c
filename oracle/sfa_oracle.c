/*
 * fp64 CPU oracle for top-k sparse FlashAttention (prefill and paged decode).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * helper with the CUDA path (sparse_flashattention_b200/csrc); the two meet only
 * in the seeded input arrays.
 *
 * What it computes is the plain definition, one (query, head) row at a time:
 * standard softmax attention restricted to the explicit set of selected keys that
 * survive the mask.  Sources:
 *  - "Sparse FlashAttention" on Ascend (ggplus blog post), section "这到底是个啥？
 *    Sparse FlashAttention架构初探": the operator pulls the K/V rows named by the
 *    top-k indices into a compact sub-matrix and runs ordinary attention on those
 *    entries only; FlashAttention itself is exact (equal to standard attention).
 *  - flash-attention-npu, "FlashAttention v2" API docstrings (flash_attn_func,
 *    flash_attn_varlen_func, flash_attn_with_kvcache): bottom-right aligned causal
 *    mask, sliding window [i+sk-sq-wl, i+sk-sq+wr], an all-masked row outputs 0,
 *    GQA head h -> kv head h / (Hq/Hkv), softmax_lse = per-row logsumexp of
 *    QK^T*scale, default scale 1/sqrt(d), varlen layout (total, H, d) with
 *    cu_seqlens, lse layout (H, total_q), paged cache (num_blocks, page, Hkv, d)
 *    addressed through block_table.
 *  - Ascend SFA page, ConstInfo listing: INVALID_IDX = -1 marks an unused top-k slot.
 *
 * Readings where the pages are silent (each is restated where it is used):
 *  - a selected block id s names keys [s*bs, min(s*bs+bs, sk)) of its own sequence;
 *  - the selection is a set: duplicates and order do not matter;
 *  - an id that is neither -1 nor in [0, ceil(sk/bs)) is an error: counted, ignored;
 *  - an all-masked row has lse = -inf (log of an empty sum);
 *  - decode token ids are logical positions in [0, cache_seqlens[b]); other ids are
 *    errors (counted, ignored); a block_table entry outside [0, num_pages) is an
 *    error (counted) and drops that token.
 *
 * Inputs q/k/v are bfloat16 bit patterns; every one converts to double exactly, so
 * each product q*k is exact in fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int cmp_int(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* Key j (sequence-local) survives the mask for local query i when, with delta = sk - sq:
 *   causal  => j <= i + delta          (causal mask aligned to the bottom-right corner)
 *   wl >= 0 => j >= i + delta - wl     (window left edge)
 *   wr >= 0 => j <= i + delta + wr     (window right edge)                          */
static int key_kept(int64_t j, int64_t i, int64_t delta, int causal, int wl, int wr)
{
    if (causal && j > i + delta) return 0;
    if (wl >= 0 && j < i + delta - wl) return 0;
    if (wr >= 0 && j > i + delta + wr) return 0;
    return 1;
}

/* Standard softmax attention of one query row over an explicit list of key rows.
 * krows[a] / vrows[a] point at the d bf16 values of key a.  Empty list: out = 0,
 * lse = -inf. */
static void attend_row(const uint16_t *qrow, const uint16_t *const *krows, const uint16_t *const *vrows,
                       int n, int d, double scale, double *scores, double *out, double *lse)
{
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int a = 0; a < n; ++a) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += bf16_value(qrow[c]) * bf16_value(krows[a][c]);
        s *= scale;
        scores[a] = s;
        if (s > m) m = s;
    }
    double z = 0.0;
    for (int a = 0; a < n; ++a) {
        scores[a] = exp(scores[a] - m);
        z += scores[a];
    }
    for (int a = 0; a < n; ++a) {
        double p = scores[a] / z;
        for (int c = 0; c < d; ++c) out[c] += p * bf16_value(vrows[a][c]);
    }
    *lse = m + log(z);
}

static int owner_of(const int32_t *cu, int batch, int64_t t)
{
    for (int b = 0; b < batch; ++b)
        if (t < cu[b + 1]) return b;
    return batch - 1;
}

/* ---------------------------------------------------------------------------------------------
 * Prefill
 * ------------------------------------------------------------------------------------------- */

typedef struct {
    const uint16_t *q, *k, *v;
    const int32_t *cu_q, *cu_k;
    int batch, Hq, Hkv, d;
    const int32_t *sel;
    int topk, bs, causal, wl, wr;
    double scale;
    const int64_t *rows; /* flat row ids t*Hq + h, or NULL for every row */
    int64_t nrows;
    double *out, *lse;
    int nthreads, max_sk;
} fwd_job;

typedef struct {
    const fwd_job *J;
    int tid;
    int64_t bad;
} fwd_thread;

/* Build the kept-key list of (token t, kv head hk): union over the row's selected blocks of
 * keys [s*bs, min(s*bs+bs, sk)), intersected with the mask, ascending.  Returns the count;
 * *bad counts ids that are neither -1 nor a block of the sequence. */
static int fwd_keyset(const fwd_job *J, int64_t t, int hk, unsigned char *mark, int *keys, int64_t *bad)
{
    int b = owner_of(J->cu_q, J->batch, t);
    int64_t i = t - J->cu_q[b];
    int64_t sq = J->cu_q[b + 1] - J->cu_q[b];
    int64_t sk = J->cu_k[b + 1] - J->cu_k[b];
    int64_t delta = sk - sq;
    int64_t nblk = (sk + J->bs - 1) / J->bs;
    const int32_t *slist = J->sel + (t * J->Hkv + hk) * (int64_t)J->topk;
    int n = 0;
    for (int e = 0; e < J->topk; ++e) {
        int s = slist[e];
        if (s == -1) continue;
        if (s < 0 || s >= nblk) { (*bad)++; continue; }
        int64_t j0 = (int64_t)s * J->bs, j1 = j0 + J->bs < sk ? j0 + J->bs : sk;
        for (int64_t j = j0; j < j1; ++j) {
            if (mark[j]) continue; /* already taken through a duplicate id */
            mark[j] = 1;
            if (key_kept(j, i, delta, J->causal, J->wl, J->wr)) keys[n++] = (int)j;
        }
    }
    for (int e = 0; e < J->topk; ++e) {
        int s = slist[e];
        if (s < 0 || s >= nblk) continue;
        int64_t j0 = (int64_t)s * J->bs, j1 = j0 + J->bs < sk ? j0 + J->bs : sk;
        memset(mark + j0, 0, (size_t)(j1 - j0));
    }
    qsort(keys, (size_t)n, sizeof(int), cmp_int);
    return n;
}

static void *fwd_worker(void *arg)
{
    fwd_thread *th = (fwd_thread *)arg;
    const fwd_job *J = th->J;
    const int G = J->Hq / J->Hkv;
    const int total_q = J->cu_q[J->batch];
    const int64_t nrows = J->rows ? J->nrows : (int64_t)total_q * J->Hq;
    const int cap = J->max_sk > 0 ? J->max_sk : 1;
    unsigned char *mark = (unsigned char *)calloc((size_t)cap, 1);
    int *keys = (int *)malloc(sizeof(int) * (size_t)cap);
    double *scores = (double *)malloc(sizeof(double) * (size_t)cap);
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)cap);
    int64_t bad = 0;

    for (int64_t r = th->tid; r < nrows; r += J->nthreads) {
        int64_t flat = J->rows ? J->rows[r] : r;
        int64_t t = flat / J->Hq;
        int h = (int)(flat % J->Hq);
        int hk = h / G; /* GQA: q head h reads kv head h / (Hq/Hkv) */
        int64_t bad_row = 0;
        int n = fwd_keyset(J, t, hk, mark, keys, &bad_row);
        if (h % G == 0) bad += bad_row; /* count each (token, kv head) once */
        int b = owner_of(J->cu_q, J->batch, t);
        for (int a = 0; a < n; ++a) {
            int64_t krow = ((int64_t)J->cu_k[b] + keys[a]) * J->Hkv + hk;
            kr[a] = J->k + krow * J->d;
            vr[a] = J->v + krow * J->d;
        }
        double l;
        attend_row(J->q + flat * (int64_t)J->d, kr, vr, n, J->d, J->scale, scores,
                   J->out + (J->rows ? r : flat) * (int64_t)J->d, &l);
        if (J->rows) J->lse[r] = l;
        else J->lse[(int64_t)h * total_q + t] = l; /* lse layout (Hq, total_q) */
    }
    free(mark); free(keys); free(scores); free(kr); free(vr);
    th->bad = bad;
    return NULL;
}

static int max_len(const int32_t *cu, int batch)
{
    int m = 0;
    for (int b = 0; b < batch; ++b)
        if (cu[b + 1] - cu[b] > m) m = cu[b + 1] - cu[b];
    return m;
}

/* Prefill attention.  rows == NULL: every row, out (total_q, Hq, d), lse (Hq, total_q).
 * rows != NULL: only the listed flat rows t*Hq+h, out (nrows, d), lse (nrows).
 * cu_k == NULL means the same as cu_q.  scale <= 0 means 1/sqrt(d).
 * Returns the number of out-of-range block ids seen (each (token, kv head) slot once when
 * every head of the group is computed). */
int64_t sfa_oracle_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       const int32_t *cu_q, const int32_t *cu_k, int batch, int Hq, int Hkv, int d,
                       const int32_t *sel, int topk, int bs, int causal, int wl, int wr, double scale,
                       const int64_t *rows, int64_t nrows, double *out, double *lse, int nthreads)
{
    fwd_job J;
    J.q = q; J.k = k; J.v = v; J.cu_q = cu_q; J.cu_k = cu_k ? cu_k : cu_q;
    J.batch = batch; J.Hq = Hq; J.Hkv = Hkv; J.d = d; J.sel = sel; J.topk = topk; J.bs = bs;
    J.causal = causal; J.wl = wl; J.wr = wr;
    J.scale = scale > 0 ? scale : 1.0 / sqrt((double)d);
    J.rows = rows; J.nrows = nrows; J.out = out; J.lse = lse;
    J.nthreads = nthreads < 1 ? 1 : nthreads;
    J.max_sk = max_len(J.cu_k, batch);
    pthread_t *ids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)J.nthreads);
    fwd_thread *ths = (fwd_thread *)calloc((size_t)J.nthreads, sizeof(fwd_thread));
    for (int i = 0; i < J.nthreads; ++i) {
        ths[i].J = &J;
        ths[i].tid = i;
        pthread_create(&ids[i], NULL, fwd_worker, &ths[i]);
    }
    int64_t bad = 0;
    for (int i = 0; i < J.nthreads; ++i) {
        pthread_join(ids[i], NULL);
        bad += ths[i].bad;
    }
    free(ids);
    free(ths);
    return bad;
}

/* Canonical selection of every (token, kv head): the ascending distinct block ids that are
 * blocks of the sequence and contain at least one key kept by the mask, then -1 padding;
 * cnt = how many.  Output layouts (total_q, Hkv, topk) and (total_q, Hkv).  Returns the
 * number of out-of-range ids. */
int64_t sfa_oracle_fwd_index(const int32_t *cu_q, const int32_t *cu_k, int batch, int Hkv,
                             const int32_t *sel, int topk, int bs, int causal, int wl, int wr,
                             int32_t *sel_c, int32_t *cnt)
{
    if (!cu_k) cu_k = cu_q;
    int64_t bad = 0;
    int total_q = cu_q[batch];
    int *buf = (int *)malloc(sizeof(int) * (size_t)(topk > 0 ? topk : 1));
    for (int64_t t = 0; t < total_q; ++t) {
        int b = owner_of(cu_q, batch, t);
        int64_t i = t - cu_q[b];
        int64_t sq = cu_q[b + 1] - cu_q[b], sk = cu_k[b + 1] - cu_k[b], delta = sk - sq;
        int64_t nblk = (sk + bs - 1) / bs;
        for (int hk = 0; hk < Hkv; ++hk) {
            const int32_t *row = sel + (t * Hkv + hk) * (int64_t)topk;
            int n = 0;
            for (int e = 0; e < topk; ++e) {
                int s = row[e];
                if (s == -1) continue;
                if (s < 0 || s >= nblk) { bad++; continue; }
                buf[n++] = s;
            }
            qsort(buf, (size_t)n, sizeof(int), cmp_int);
            int m = 0;
            for (int a = 0; a < n; ++a) {
                if (a > 0 && buf[a] == buf[a - 1]) continue; /* set semantics */
                int64_t j0 = (int64_t)buf[a] * bs, j1 = j0 + bs < sk ? j0 + bs : sk;
                int any = 0;
                for (int64_t j = j0; j < j1 && !any; ++j) any = key_kept(j, i, delta, causal, wl, wr);
                if (any) buf[m++] = buf[a];
            }
            int32_t *dst = sel_c + (t * Hkv + hk) * (int64_t)topk;
            for (int e = 0; e < topk; ++e) dst[e] = e < m ? buf[e] : -1;
            cnt[t * Hkv + hk] = m;
        }
    }
    free(buf);
    return bad;
}

/* ---------------------------------------------------------------------------------------------
 * Prefill backward: gradients of the selected attention with respect to q, k and v
 * -------------------------------------------------------------------------------------------
 * Sources: "Sparse FlashAttention" on Ascend (ggplus blog post), FlashAttentionScoreGrad case
 * study at the end of the post: recompute the probabilities P, then dP = dO V^T, dS = P o (dP -
 * rowsum(dO o O)), dQ = (dS K) * scale; the flash-sparse-attention README, "反向" (backward)
 * example: gradients of the selected attention flow to query, key and value.  The pages stop at
 * dQ; dK = scale * dS^T Q and dV = P^T dO are the same chain rule applied to the other two
 * operands (the plainest reading).  Per row (query t, head h) over its kept keys a — the same
 * key set as the forward:
 *   p_a  = exp(s_a - lse),  s_a = scale * q . k_a
 *   dp_a = dO . v_a;  D = sum_a p_a dp_a  (= dO . o);  ds_a = p_a (dp_a - D)
 *   dq   = scale * sum_a ds_a k_a;   dk_a += scale * ds_a q;   dv_a += p_a dO
 * A row with no kept key contributes nothing and has dq = 0.  Every key that no row keeps has
 * dk = dv = 0.  Work is split by (sequence, kv head): the rows of one split are the only writers of
 * its keys' dk / dv, so the sums need no locks and run in a fixed order. */

typedef struct {
    fwd_job F;              /* the forward's inputs and key-set rules */
    const uint16_t *dout;   /* (total_q, Hq, d) bf16 bits */
    double *dq, *dk, *dv;   /* (total_q, Hq, d), (total_k, Hkv, d), (total_k, Hkv, d) */
} bwd_job;

typedef struct {
    const bwd_job *J;
    int tid;
    int64_t bad;
} bwd_thread;

static void *bwd_worker(void *arg)
{
    bwd_thread *th = (bwd_thread *)arg;
    const bwd_job *J = th->J;
    const fwd_job *F = &J->F;
    const int G = F->Hq / F->Hkv, d = F->d;
    const int cap = F->max_sk > 0 ? F->max_sk : 1;
    unsigned char *mark = (unsigned char *)calloc((size_t)cap, 1);
    int *keys = (int *)malloc(sizeof(int) * (size_t)cap);
    double *p = (double *)malloc(sizeof(double) * (size_t)cap);
    double *dp = (double *)malloc(sizeof(double) * (size_t)cap);
    double *qv = (double *)malloc(sizeof(double) * (size_t)d);
    double *gv = (double *)malloc(sizeof(double) * (size_t)d);
    int64_t bad = 0;
    for (int job = th->tid; job < F->batch * F->Hkv; job += F->nthreads) {
        const int b = job / F->Hkv, hk = job % F->Hkv;
        for (int64_t t = F->cu_q[b]; t < F->cu_q[b + 1]; ++t) {
            int64_t bad_row = 0;
            const int n = fwd_keyset(F, t, hk, mark, keys, &bad_row);
            bad += bad_row;
            for (int g = 0; g < G; ++g) {
                const int h = hk * G + g;
                const int64_t flat = t * F->Hq + h;
                double *dqrow = J->dq + flat * d;
                for (int c = 0; c < d; ++c) dqrow[c] = 0.0;
                if (n == 0) continue;
                for (int c = 0; c < d; ++c) {
                    qv[c] = bf16_value(F->q[flat * d + c]);
                    gv[c] = bf16_value(J->dout[flat * d + c]);
                }
                /* probabilities, by the forward's definition (max-shifted for range) */
                double m = -INFINITY;
                for (int a = 0; a < n; ++a) {
                    const uint16_t *kr = F->k + (((int64_t)F->cu_k[b] + keys[a]) * F->Hkv + hk) * d;
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += qv[c] * bf16_value(kr[c]);
                    p[a] = s * F->scale;
                    if (p[a] > m) m = p[a];
                }
                double z = 0.0;
                for (int a = 0; a < n; ++a) {
                    p[a] = exp(p[a] - m);
                    z += p[a];
                }
                double D = 0.0;
                for (int a = 0; a < n; ++a) {
                    p[a] /= z;
                    const uint16_t *vr = F->v + (((int64_t)F->cu_k[b] + keys[a]) * F->Hkv + hk) * d;
                    double x = 0.0;
                    for (int c = 0; c < d; ++c) x += gv[c] * bf16_value(vr[c]);
                    dp[a] = x;
                    D += p[a] * x;
                }
                for (int a = 0; a < n; ++a) {
                    const int64_t krow = ((int64_t)F->cu_k[b] + keys[a]) * F->Hkv + hk;
                    const uint16_t *kr = F->k + krow * d;
                    const double ds = p[a] * (dp[a] - D);
                    double *dkrow = J->dk + krow * d, *dvrow = J->dv + krow * d;
                    for (int c = 0; c < d; ++c) {
                        dqrow[c] += F->scale * ds * bf16_value(kr[c]);
                        dkrow[c] += F->scale * ds * qv[c];
                        dvrow[c] += p[a] * gv[c];
                    }
                }
            }
        }
    }
    free(mark); free(keys); free(p); free(dp); free(qv); free(gv);
    th->bad = bad;
    return NULL;
}

/* Backward of sfa_oracle_fwd's attention (same arguments), given dout: dq (total_q, Hq, d) and
 * dk, dv (total_k, Hkv, d), all written in full.  Returns the number of out-of-range block ids
 * (each (token, kv head) slot once). */
int64_t sfa_oracle_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                       const int32_t *cu_q, const int32_t *cu_k, int batch, int Hq, int Hkv, int d,
                       const int32_t *sel, int topk, int bs, int causal, int wl, int wr, double scale,
                       double *dq, double *dk, double *dv, int nthreads)
{
    bwd_job J;
    memset(&J, 0, sizeof J);
    J.F.q = q; J.F.k = k; J.F.v = v; J.F.cu_q = cu_q; J.F.cu_k = cu_k ? cu_k : cu_q;
    J.F.batch = batch; J.F.Hq = Hq; J.F.Hkv = Hkv; J.F.d = d; J.F.sel = sel; J.F.topk = topk; J.F.bs = bs;
    J.F.causal = causal; J.F.wl = wl; J.F.wr = wr;
    J.F.scale = scale > 0 ? scale : 1.0 / sqrt((double)d);
    J.F.nthreads = nthreads < 1 ? 1 : nthreads;
    J.F.max_sk = max_len(J.F.cu_k, batch);
    J.dout = dout; J.dq = dq; J.dk = dk; J.dv = dv;
    const int64_t total_k = J.F.cu_k[batch];
    memset(dk, 0, sizeof(double) * (size_t)(total_k * Hkv * d));
    memset(dv, 0, sizeof(double) * (size_t)(total_k * Hkv * d));
    pthread_t *ids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)J.F.nthreads);
    bwd_thread *ths = (bwd_thread *)calloc((size_t)J.F.nthreads, sizeof(bwd_thread));
    for (int i = 0; i < J.F.nthreads; ++i) {
        ths[i].J = &J;
        ths[i].tid = i;
        pthread_create(&ids[i], NULL, bwd_worker, &ths[i]);
    }
    int64_t bad = 0;
    for (int i = 0; i < J.F.nthreads; ++i) {
        pthread_join(ids[i], NULL);
        bad += ths[i].bad;
    }
    free(ids);
    free(ths);
    return bad;
}

/* ---------------------------------------------------------------------------------------------
 * Paged decode (one new query token per sequence, at logical position L-1)
 * ------------------------------------------------------------------------------------------- */

typedef struct {
    const uint16_t *q, *kc, *vc;
    const int32_t *bt;
    int max_pages, num_pages, page;
    const int32_t *seqlens, *sel;
    int topk, B, Hq, Hkv, d, wl;
    double scale;
    double *out, *lse;
    int nthreads;
} dec_job;

typedef struct {
    const dec_job *J;
    int tid;
    int64_t bad_index, bad_page;
} dec_thread;

/* Canonical token set of (b, kv head): ascending distinct positions j with 0 <= j < L (and
 * j >= L-1-wl when wl >= 0).  Returns the count; *bad counts ids that are neither -1 nor in
 * [0, L). */
static int dec_tokens(const dec_job *J, int b, int hk, int *buf, int64_t *bad)
{
    int L = J->seqlens[b];
    const int32_t *row = J->sel + ((int64_t)b * J->Hkv + hk) * J->topk;
    int n = 0;
    for (int e = 0; e < J->topk; ++e) {
        int j = row[e];
        if (j == -1) continue;
        if (j < 0 || j >= L) { (*bad)++; continue; }
        if (J->wl >= 0 && j < L - 1 - J->wl) continue; /* outside the left window */
        buf[n++] = j;
    }
    qsort(buf, (size_t)n, sizeof(int), cmp_int);
    int m = 0;
    for (int a = 0; a < n; ++a)
        if (a == 0 || buf[a] != buf[a - 1]) buf[m++] = buf[a];
    return m;
}

static void *dec_worker(void *arg)
{
    dec_thread *th = (dec_thread *)arg;
    const dec_job *J = th->J;
    const int G = J->Hq / J->Hkv;
    int *toks = (int *)malloc(sizeof(int) * (size_t)(J->topk > 0 ? J->topk : 1));
    double *scores = (double *)malloc(sizeof(double) * (size_t)(J->topk > 0 ? J->topk : 1));
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)(J->topk > 0 ? J->topk : 1));
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)(J->topk > 0 ? J->topk : 1));
    for (int64_t r = th->tid; r < (int64_t)J->B * J->Hq; r += J->nthreads) {
        int b = (int)(r / J->Hq), h = (int)(r % J->Hq), hk = h / G;
        int64_t bad = 0;
        int n = dec_tokens(J, b, hk, toks, &bad);
        int m = 0;
        for (int a = 0; a < n; ++a) {
            int j = toks[a];
            int pg = J->bt[(int64_t)b * J->max_pages + j / J->page];
            if (pg < 0 || pg >= J->num_pages) { if (h % G == 0) th->bad_page++; continue; }
            int64_t rowi = (((int64_t)pg * J->page + j % J->page) * J->Hkv + hk) * J->d;
            kr[m] = J->kc + rowi;
            vr[m] = J->vc + rowi;
            m++;
        }
        if (h % G == 0) th->bad_index += bad;
        attend_row(J->q + r * J->d, kr, vr, m, J->d, J->scale, scores, J->out + r * J->d, &J->lse[r]);
    }
    free(toks); free(scores); free(kr); free(vr);
    return NULL;
}

/* Decode attention, out (B, Hq, d), lse (B, Hq).  bad[0] += out-of-range token ids,
 * bad[1] += tokens whose block_table entry is outside [0, num_pages). */
void sfa_oracle_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                       const int32_t *block_table, int max_pages, int num_pages, int page,
                       const int32_t *cache_seqlens, const int32_t *sel, int topk,
                       int B, int Hq, int Hkv, int d, int wl, double scale,
                       double *out, double *lse, int nthreads, int64_t *bad)
{
    dec_job J;
    J.q = q; J.kc = k_cache; J.vc = v_cache; J.bt = block_table; J.max_pages = max_pages;
    J.num_pages = num_pages; J.page = page; J.seqlens = cache_seqlens; J.sel = sel; J.topk = topk;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.d = d; J.wl = wl;
    J.scale = scale > 0 ? scale : 1.0 / sqrt((double)d);
    J.out = out; J.lse = lse; J.nthreads = nthreads < 1 ? 1 : nthreads;
    pthread_t *ids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)J.nthreads);
    dec_thread *ths = (dec_thread *)calloc((size_t)J.nthreads, sizeof(dec_thread));
    for (int i = 0; i < J.nthreads; ++i) {
        ths[i].J = &J;
        ths[i].tid = i;
        pthread_create(&ids[i], NULL, dec_worker, &ths[i]);
    }
    for (int i = 0; i < J.nthreads; ++i) {
        pthread_join(ids[i], NULL);
        bad[0] += ths[i].bad_index;
        bad[1] += ths[i].bad_page;
    }
    free(ids);
    free(ths);
}

/* Canonical token sets, (B, Hkv, topk) ascending then -1 padded, and counts (B, Hkv). */
int64_t sfa_oracle_decode_index(const int32_t *cache_seqlens, const int32_t *sel, int topk,
                                int B, int Hkv, int wl, int32_t *tok_c, int32_t *cnt)
{
    dec_job J;
    memset(&J, 0, sizeof J);
    J.seqlens = cache_seqlens; J.sel = sel; J.topk = topk; J.B = B; J.Hkv = Hkv; J.wl = wl;
    int *buf = (int *)malloc(sizeof(int) * (size_t)(topk > 0 ? topk : 1));
    int64_t bad = 0;
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk) {
            int n = dec_tokens(&J, b, hk, buf, &bad);
            int32_t *dst = tok_c + ((int64_t)b * Hkv + hk) * topk;
            for (int e = 0; e < topk; ++e) dst[e] = e < n ? buf[e] : -1;
            cnt[b * Hkv + hk] = n;
        }
    free(buf);
    return bad;
}
