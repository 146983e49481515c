// Index preparation: turn the caller's top-k selections into canonical sets.
//
// Prefill (one CTA per query tile): for every (token, kv head) of the tile keep the block ids
// that are -1-free, inside the sequence, and hold at least one key the mask keeps; sort them
// ascending without duplicates (a selection is a set); count them; and OR them into a bitmap
// whose ascending scan is the tile's union of blocks — the list the attention kernel walks.
// INVALID = -1 marks an unused slot (Ascend SFA article, ConstInfo listing); the mask is the
// bottom-right aligned causal mask plus window of the flash-attention-npu docstrings.
//
// Decode (one CTA per (sequence, kv head)): a bitmap over the positions [0, L) turns the
// selected token positions into an ascending duplicate-free list in O(L/32) work.
#include <climits>

#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kPrepThreads = 128;

// Exclusive scan of one int per thread over a 128- or 256-thread block; returns the total.
template <int NT>
__device__ int block_exclusive_scan(int v, int *scratch, int &excl)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < NT / 32 ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < NT / 32) scratch[lane] = w;  // inclusive per-warp totals
    }
    __syncthreads();
    const int before = warp > 0 ? scratch[warp - 1] : 0;
    excl = before + x - v;
    const int total = scratch[NT / 32 - 1];
    __syncthreads();
    return total;
}

// Bitmap words [0, words) -> ascending ids written to dst; returns the count.  All threads.
template <int NT>
__device__ int compact_bitmap(const uint32_t *bm, int words, int32_t *dst, int *scratch)
{
    const int per = (words + NT - 1) / NT;
    const int w0 = min(words, (int)threadIdx.x * per), w1 = min(words, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(bm[w]);
    int pos;
    const int total = block_exclusive_scan<NT>(c, scratch, pos);
    for (int w = w0; w < w1; ++w) {
        uint32_t bits = bm[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            dst[pos++] = w * 32 + b;
        }
    }
    return total;
}

__global__ void __launch_bounds__(kPrepThreads) fwd_prep_kernel(FwdPrepParams p)
{
    extern __shared__ uint32_t prep_smem[];
    __shared__ int scan_scratch[32];
    if (blockIdx.x == 0 && threadIdx.x < 2 && p.tile_counter) p.tile_counter[threadIdx.x] = 0;
    const int tile = blockIdx.x;
    const int hk = tile % p.Hkv;
    const int rest = tile / p.Hkv;
    const int b = rest % p.batch;
    const int qt = p.nqt - 1 - rest / p.batch;

    const int q0 = p.cu_q[b], sq = p.cu_q[b + 1] - q0;
    const int sk = p.cu_k[b + 1] - p.cu_k[b];
    const int tok0 = qt * p.Tq;
    const int ntok = min(p.Tq, sq - tok0);
    if (ntok <= 0) {
        if (threadIdx.x == 0) p.ucnt[tile] = 0;
        return;
    }
    int nblk = (sk + p.bs - 1) / p.bs;
    if (sq > p.max_sq || nblk > p.nblk_max) {  // lengths beyond the caller's max_seqlen bounds
        if (threadIdx.x == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
        nblk = min(nblk, p.nblk_max);
    }
    const int words = (p.nblk_max + 31) / 32;
    uint32_t *bm = prep_smem;
    // [Tq][rs] selections as given: an odd row stride rs keeps a warp's 32 rows on 32 banks when each
    // thread walks its own row
    const int rs = p.topk | 1;
    int *raw = reinterpret_cast<int *>(prep_smem + words);
    int *lists = raw + p.Tq * rs;                             // [topk][kPrepThreads] canonical
    int *hist = p.tcount ? lists + p.topk * kPrepThreads : nullptr;  // [nblk_max] this tile's tokens per block
    uint32_t *dbm = p.duni ? reinterpret_cast<uint32_t *>(hist + p.nblk_max) : nullptr;  // [words] dense blocks
    for (int w = threadIdx.x; w < words; w += kPrepThreads) bm[w] = 0;
    if (hist)
        for (int s = threadIdx.x; s < p.nblk_max; s += kPrepThreads) hist[s] = 0;
    const int64_t row0 = ((int64_t)(q0 + tok0) * p.Hkv + hk) * p.topk;
    const int64_t tok_stride = (int64_t)p.Hkv * p.topk;
    for (int e = threadIdx.x; e < ntok * p.topk; e += kPrepThreads) {
        const int tt = e / p.topk;
        raw[tt * rs + (e - tt * p.topk)] = p.sel[row0 + tt * tok_stride + (e - tt * p.topk)];
    }
    __syncthreads();

    const int tt = threadIdx.x;
    int n = 0;
    if (tt < ntok) {
        const int i = tok0 + tt;  // local query index
        const int delta = sk - sq;
        int lo = 0, hi = sk - 1;
        if (p.wl >= 0) lo = max(lo, i + delta - p.wl);
        if (p.causal) hi = min(hi, i + delta);
        if (p.wr >= 0) hi = min(hi, i + delta + p.wr);
        bool bad = false;
        // canonical list into column tt of lists ([slot][kPrepThreads])
        const int *r = raw + tt * rs;
        if (p.topk <= 16) n = canon_list_regs<16>(r, p.topk, nblk, p.bs, sk, lo, hi, lists + tt, kPrepThreads, bad);
        else if (p.topk <= 32) n = canon_list_regs<32>(r, p.topk, nblk, p.bs, sk, lo, hi, lists + tt, kPrepThreads, bad);
        else n = canon_list_insert(r, p.topk, nblk, p.bs, sk, lo, hi, lists + tt, kPrepThreads, bad);
        const int64_t t = (int64_t)q0 + i;
        p.cnt[t * p.Hkv + hk] = n;
        if (bad && p.status) atomicOr(p.status, SFA_DEV_BAD_INDEX);
    }
    // Union bitmap: lanes that hold the same block set its bit once.  With the block-major
    // schedule on, also count each block's selecting tokens of this tile (shared memory; the tile's
    // counts then go out whole, so no counter is shared between CTAs).
    const int grp = p.gstat ? ((tok0 / p.W) * p.batch + b) * p.Hkv + hk : 0;
    {
        const int maxn = __reduce_max_sync(0xffffffffu, n);
        const int lane = threadIdx.x & 31;
        for (int e = 0; e < maxn; ++e) {
            const int s = e < n ? lists[e * kPrepThreads + tt] : -1;
            const unsigned m = __match_any_sync(0xffffffffu, s);
            if (s >= 0 && lane == __ffs(m) - 1) {
                atomicOr(&bm[s >> 5], 1u << (s & 31));
                if (hist) atomicAdd(&hist[s], __popc(m));
            }
        }
        if (p.gstat) {
            const int wsum = __reduce_add_sync(0xffffffffu, n);
            if (lane == 0 && wsum) atomicAdd(&p.gstat[grp].useful, (unsigned long long)wsum);
        }
    }
    __syncthreads();  // every thread is done reading raw
    if (tt < ntok)
        for (int e = 0; e < p.topk; ++e) raw[tt * rs + e] = e < n ? lists[e * kPrepThreads + tt] : -1;
    __syncthreads();
    for (int e = threadIdx.x; e < ntok * p.topk; e += kPrepThreads) {
        const int t2 = e / p.topk;
        p.sel_c[row0 + t2 * tok_stride + (e - t2 * p.topk)] = raw[t2 * rs + (e - t2 * p.topk)];
    }
    if (dbm) {
        // Dense blocks: selected by at least a quarter of a full tile's rows (Tq / 4 tokens), at most
        // kDenseMax, ascending.  They run query-major for this tile (the query-major kernel leaves that
        // partial in out / lse), so they leave the tile's counts; each token notes which of the dense
        // blocks it selected and which of its canonical entries they are.  (The lists region is free
        // now and holds up to 2 * topk dense blocks: each needs Tq / 4 of the tile's Tq * topk entries.)
        for (int w = threadIdx.x; w < words; w += kPrepThreads) dbm[w] = 0;
        __syncthreads();
        for (int s = threadIdx.x; s < nblk; s += kPrepThreads)
            if (hist[s] > 0 && 4 * hist[s] >= p.Tq) atomicOr(&dbm[s >> 5], 1u << (s & 31));
        __syncthreads();
        const int nd = min(kDenseMax, compact_bitmap<kPrepThreads>(dbm, (nblk + 31) / 32, lists, scan_scratch));
        for (int j = threadIdx.x; j < nd; j += kPrepThreads) {
            hist[lists[j]] = -1 - j;
            p.duni[(int64_t)tile * kDenseMax + j] = lists[j];
        }
        if (threadIdx.x == 0) p.dcnt[tile] = nd;
        __syncthreads();
        if (tt < ntok) {
            uint32_t sel_bits = 0, entry_bits = 0;
            for (int e = 0; e < n; ++e) {
                const int v = hist[raw[tt * rs + e]];
                if (v < 0) {
                    sel_bits |= 1u << (-1 - v);
                    entry_bits |= 1u << e;
                }
            }
            const int64_t t = (int64_t)q0 + tok0 + tt;
            p.dsel[t * p.Hkv + hk] = sel_bits;
            p.dsel[(int64_t)p.total_q * p.Hkv + t * p.Hkv + hk] = entry_bits;
        }
    }
    if (hist)
        for (int s = threadIdx.x; s < p.nblk_max; s += kPrepThreads)
            p.tcount[(int64_t)tile * p.nblk_max + s] = max(hist[s], 0);
    const int total = compact_bitmap<kPrepThreads>(bm, (nblk + 31) / 32, p.uni + (int64_t)tile * p.umax,
                                                   scan_scratch);
    if (threadIdx.x == 0) {
        p.ucnt[tile] = total;
        if (p.gstat) atomicAdd(&p.gstat[grp].uni, (unsigned long long)total * ntok);
    }
    grid_dep_launch();
}

constexpr int kInvThreads = 256;

// Block-major plan, one CTA per (window, sequence, kv head) group and run of kInvThreads blocks.
// The window stays with the query-major kernel unless the union of its query tiles' blocks is
// over 4x its selected blocks (a block-major item moves several times the memory of a query-major
// tile per selected row-block: its bf16 partial is written and read back and its Q rows are
// gathered).  For a block-major window: mark its tiles (ucnt = -1); per block (one thread each)
// add up the window's tiles' counts, leaving in each tile's place its first position in the
// block's list; cut each block's list into items of at most Tq tokens, reserve the CTA's items,
// and write their records (tokens come from the scatter kernel).
__global__ void __launch_bounds__(kInvThreads) fwd_plan_kernel(FwdPlanParams p)
{
    __shared__ int scan_scratch[32];
    __shared__ int item_base;
    grid_dep_wait();
    const int g = blockIdx.x;
    const int s = blockIdx.y * kInvThreads + threadIdx.x;  // this thread's block
    const int hk = g % p.Hkv;
    const int b = (g / p.Hkv) % p.batch;
    const int w = g / (p.Hkv * p.batch);
    const int sq = p.cu_q[b + 1] - p.cu_q[b];
    const int t0 = w * p.W;
    if (t0 >= sq) return;
    const GroupStat st = p.gstat[g];
    if (st.uni <= 4ull * st.useful) return;  // the query-major kernel keeps this window
    const int nt = min(p.W, sq - t0);
    const int qt0 = t0 / p.Tq, qt1 = (t0 + nt - 1) / p.Tq;
    if (blockIdx.y == 0)
        for (int qt = qt0 + threadIdx.x; qt <= qt1; qt += kInvThreads)
            p.ucnt[((p.nqt - 1 - qt) * p.batch + b) * p.Hkv + hk] = -1;

    // The block's token count over the window's tiles, and in place of each tile's count the tile's
    // first position in the block's list (tiles in query order; eight tiles' counts loaded at once).
    int c = 0;
    if (s < p.nblk_max) {
        for (int q8 = qt0; q8 <= qt1; q8 += 8) {
            int v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = q8 + i <= qt1 ? p.tcount[(int64_t)(((p.nqt - 1 - (q8 + i)) * p.batch + b) * p.Hkv + hk) * p.nblk_max + s]
                                     : 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (q8 + i <= qt1) {
                    p.tcount[(int64_t)(((p.nqt - 1 - (q8 + i)) * p.batch + b) * p.Hkv + hk) * p.nblk_max + s] = c;
                    c += v[i];
                }
        }
    }
    // this CTA's items: reserved together, each block's consecutive
    int pos;
    const int nitems = block_exclusive_scan<kInvThreads>((c + p.Tq - 1) / p.Tq, scan_scratch, pos);
    if (threadIdx.x == 0) item_base = atomicAdd(&p.ctrl->item_total, nitems);
    __syncthreads();
    if (s < p.nblk_max) {
        const int i0 = item_base + pos;
        p.gfirst[(int64_t)g * p.nblk_max + s] = i0;
        const int k0 = p.cu_k[b];
        for (int i = 0; i * p.Tq < c; ++i)
            p.items[i0 + i].rec = make_int4(b * p.Hkv + hk, s, k0, min(p.Tq, c - i * p.Tq));
    }
}

// Block-major token lists, one CTA per query tile of a block-major window: every (token, block)
// of the tile's canonical selections takes the next position in its block's list, counted on from
// the tile's first position there (the plan's scan of the tiles' counts; shared-memory atomics, no
// counter shared between CTAs), which names the item (position / Tq) and the slot in it.
__global__ void __launch_bounds__(kPrepThreads) fwd_scatter_kernel(FwdScatterParams p)
{
    extern __shared__ int scatter_smem[];
    grid_dep_wait();
    const int tile = blockIdx.x;
    if (p.ucnt[tile] != -1) return;
    const int hk = tile % p.Hkv;
    const int rest = tile / p.Hkv;
    const int b = rest % p.batch;
    const int qt = p.nqt - 1 - rest / p.batch;
    const int q0 = p.cu_q[b], sq = p.cu_q[b + 1] - q0;
    const int tok0 = qt * p.Tq;
    const int ntok = min(p.Tq, sq - tok0);
    const int grp = ((tok0 / p.W) * p.batch + b) * p.Hkv + hk;
    int *pos_s = scatter_smem;                // next position of each block's list for this tile
    int *first_s = scatter_smem + p.nblk_max; // first item of each block
    for (int s = threadIdx.x; s < p.nblk_max; s += kPrepThreads) {
        pos_s[s] = p.tcount[(int64_t)tile * p.nblk_max + s];
        first_s[s] = p.gfirst[(int64_t)grp * p.nblk_max + s];
    }
    __syncthreads();
    const int tt = threadIdx.x;
    const int64_t t = (int64_t)q0 + tok0 + tt;
    const int n = tt < ntok ? p.cnt[t * p.Hkv + hk] : 0;
    const uint32_t dense = tt < ntok && p.dmask ? p.dmask[t * p.Hkv + hk] : 0u;  // run query-major
    const int32_t *row = p.sel_c + (t * p.Hkv + hk) * p.topk;
    // An entry's partial goes to slot (its rank among the token's entries that are not dense), so a
    // row's block-major partials fill the first slots of its range.
    for (int e = 0; e < n; ++e) {
        if ((dense >> e) & 1u) continue;
        const int s = row[e];
        const int pos = atomicAdd(&pos_s[s], 1);
        const int slot = e - __popc(dense & ((1u << e) - 1u));
        p.items[first_s[s] + pos / p.Tq].tok[pos % p.Tq] = (int)(t << 7) | slot;
    }
}

constexpr int kDecPrepThreads = 512;

__global__ void __launch_bounds__(kDecPrepThreads) decode_prep_kernel(DecPrepParams p)
{
    extern __shared__ uint32_t dprep_smem[];
    __shared__ int scan_scratch[32];
    const int b = blockIdx.x / p.Hkv, hk = blockIdx.x % p.Hkv;
    int L = p.seqlens[b];
    bool bad_len = false;
    if (L > p.max_len) {  // more tokens than the block table can address
        L = p.max_len;
        bad_len = true;
    }
    if (L < 0) L = 0;
    const int words = (L + 31) / 32;
    for (int w = threadIdx.x; w < words; w += kDecPrepThreads) dprep_smem[w] = 0;
    __syncthreads();
    const int32_t *row = p.sel + ((int64_t)b * p.Hkv + hk) * p.topk;
    bool bad = false;
    for (int e = threadIdx.x; e < p.topk; e += kDecPrepThreads) {
        const int j = row[e];
        if (j == -1) continue;
        if (j < 0 || j >= L) {
            bad = true;
            continue;
        }
        if (p.wl >= 0 && j < L - 1 - p.wl) continue;  // left of the window
        atomicOr(&dprep_smem[j >> 5], 1u << (j & 31));
    }
    if (bad && p.status) atomicOr(p.status, SFA_DEV_BAD_INDEX);
    if (bad_len && threadIdx.x == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
    __syncthreads();
    int32_t *dst = p.tok_c + ((int64_t)b * p.Hkv + hk) * p.topk;
    const int n = compact_bitmap<kDecPrepThreads>(dprep_smem, words, dst, scan_scratch);
    for (int e = n + threadIdx.x; e < p.topk; e += kDecPrepThreads) dst[e] = -1;
    if (threadIdx.x == 0) p.cnt[b * p.Hkv + hk] = n;
}

}  // namespace

cudaError_t launch_fwd_prep(const FwdGeom &g, const FwdPrepParams &p, cudaStream_t st)
{
    const size_t words = (size_t)(g.nblk_max + 31) / 32;
    const size_t smem = words * 4 + (size_t)g.Tq * (g.topk | 1) * 4 + (size_t)g.topk * kPrepThreads * 4 +
                        (p.tcount ? (size_t)g.nblk_max * 4 : 0) + (p.duni ? words * 4 : 0);
    if (smem > 48 * 1024) {
        const cudaError_t e = ensure_smem_for(fwd_prep_kernel, smem);
        if (e != cudaSuccess) return e;
    }
    fwd_prep_kernel<<<g.tiles, kPrepThreads, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_fwd_plan(const FwdGeom &g, const FwdPlanParams &p, cudaStream_t st)
{
    const dim3 grid(g.groups, (g.nblk_max + kInvThreads - 1) / kInvThreads);
    return launch_kernel(fwd_plan_kernel, grid, dim3(kInvThreads), 0, st, true, p);
}

cudaError_t launch_fwd_scatter(const FwdGeom &g, const FwdScatterParams &p, cudaStream_t st)
{
    const size_t smem = (size_t)g.nblk_max * 8;
    if (smem > 48 * 1024) {
        const cudaError_t e = ensure_smem_for(fwd_scatter_kernel, smem);
        if (e != cudaSuccess) return e;
    }
    return launch_kernel(fwd_scatter_kernel, dim3(g.tiles), dim3(kPrepThreads), smem, st, true, p);
}

cudaError_t launch_decode_prep(const DecGeom &g, const DecPrepParams &p, cudaStream_t st)
{
    const size_t smem = (size_t)((p.max_len + 31) / 32) * 4;
    if (smem > 48 * 1024) {
        const cudaError_t e = ensure_smem_for(decode_prep_kernel, smem);
        if (e != cudaSuccess) return e;
    }
    decode_prep_kernel<<<g.B * g.Hkv, kDecPrepThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sfa
