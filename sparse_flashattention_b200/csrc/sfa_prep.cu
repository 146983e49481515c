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

// One warp-wide op on per-lane keys (-1 = no key): lanes holding the same key are counted
// together and only the lowest of them touches shared memory.  Returns, for each lane, the
// first value it may use (the leader's old value plus the lane's rank among equal keys).
__device__ __forceinline__ int warp_aggregated_add(int *counters, int key)
{
    const int lane = threadIdx.x & 31;
    const unsigned m = __match_any_sync(0xffffffffu, key);
    const int leader = __ffs(m) - 1;
    const int rank = __popc(m & ((1u << lane) - 1));
    int base = 0;
    if (lane == leader && key >= 0) base = atomicAdd(&counters[key], __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    return base + rank;
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
    int *raw = reinterpret_cast<int *>(prep_smem + words);  // [Tq][topk] selections as given
    int *lists = raw + p.Tq * p.topk;                         // [topk][kPrepThreads] canonical
    for (int w = threadIdx.x; w < words; w += kPrepThreads) bm[w] = 0;
    const int64_t row0 = ((int64_t)(q0 + tok0) * p.Hkv + hk) * p.topk;
    const int64_t tok_stride = (int64_t)p.Hkv * p.topk;
    for (int e = threadIdx.x; e < ntok * p.topk; e += kPrepThreads) {
        const int tt = e / p.topk;
        raw[e] = p.sel[row0 + tt * tok_stride + (e - tt * p.topk)];
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
        const int *r = raw + tt * p.topk;
        if (p.topk <= 16) n = canon_list_regs<16>(r, p.topk, nblk, p.bs, sk, lo, hi, lists + tt, kPrepThreads, bad);
        else if (p.topk <= 32) n = canon_list_regs<32>(r, p.topk, nblk, p.bs, sk, lo, hi, lists + tt, kPrepThreads, bad);
        else n = canon_list_insert(r, p.topk, nblk, p.bs, sk, lo, hi, lists + tt, kPrepThreads, bad);
        const int64_t t = (int64_t)q0 + i;
        p.cnt[t * p.Hkv + hk] = n;
        if (bad && p.status) atomicOr(p.status, SFA_DEV_BAD_INDEX);
    }
    // Union bitmap: lanes that hold the same block set its bit once.  With the block-major
    // schedule on, also count each block's selecting tokens for the window's group.
    const int grp = p.gstat ? ((tok0 / p.W) * p.batch + b) * p.Hkv + hk : 0;
    {
        const int maxn = __reduce_max_sync(0xffffffffu, n);
        const int lane = threadIdx.x & 31;
        int32_t *gc = p.gstat ? p.gcount + (int64_t)grp * p.nblk_max : nullptr;
        for (int e = 0; e < maxn; ++e) {
            const int s = e < n ? lists[e * kPrepThreads + tt] : -1;
            const unsigned m = __match_any_sync(0xffffffffu, s);
            if (s >= 0 && lane == __ffs(m) - 1) {
                atomicOr(&bm[s >> 5], 1u << (s & 31));
                if (gc) atomicAdd(&gc[s], __popc(m));
            }
        }
        if (p.gstat) {
            const int wsum = __reduce_add_sync(0xffffffffu, n);
            if (lane == 0 && wsum) atomicAdd(&p.gstat[grp].useful, (unsigned long long)wsum);
        }
    }
    __syncthreads();  // every thread is done reading raw
    if (tt < ntok)
        for (int e = 0; e < p.topk; ++e) raw[tt * p.topk + e] = e < n ? lists[e * kPrepThreads + tt] : -1;
    __syncthreads();
    for (int e = threadIdx.x; e < ntok * p.topk; e += kPrepThreads) {
        const int t2 = e / p.topk;
        p.sel_c[row0 + t2 * tok_stride + (e - t2 * p.topk)] = raw[e];
    }
    const int total = compact_bitmap<kPrepThreads>(bm, (nblk + 31) / 32, p.uni + (int64_t)tile * p.umax,
                                                   scan_scratch);
    if (threadIdx.x == 0) {
        p.ucnt[tile] = total;
        if (p.gstat) atomicAdd(&p.gstat[grp].uni, (unsigned long long)total * ntok);
    }
    grid_dep_launch();
}

constexpr int kInvThreads = 256;

// Exclusive scan of v[0..n) in place (all threads); returns the total.
__device__ int block_scan_array(int *v, int n, int *scratch)
{
    const int per = (n + kInvThreads - 1) / kInvThreads;
    const int i0 = min(n, (int)threadIdx.x * per), i1 = min(n, i0 + per);
    int c = 0;
    for (int i = i0; i < i1; ++i) c += v[i];
    int pos;
    const int total = block_exclusive_scan<kInvThreads>(c, scratch, pos);
    for (int i = i0; i < i1; ++i) {
        const int x = v[i];
        v[i] = pos;
        pos += x;
    }
    __syncthreads();
    return total;
}

// Block-major plan, one CTA per (window, sequence, kv head) group.  The window stays with the
// query-major kernel unless the union of its query tiles' blocks is over 4x its selected
// blocks (a block-major item moves several times the memory of a query-major tile per selected
// row-block: its bf16 partial is written and read back and its Q rows are gathered).  For a
// block-major window: mark its tiles (ucnt = -1), cut each selected block's token list into
// items of at most Tq tokens, reserve them, and write their records (tokens come from the
// scatter kernel).
__global__ void __launch_bounds__(kInvThreads) fwd_plan_kernel(FwdPlanParams p)
{
    extern __shared__ int plan_smem[];
    __shared__ int scan_scratch[32];
    __shared__ int item_base;
    grid_dep_wait();
    const int g = blockIdx.x;
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
    for (int qt = qt0 + threadIdx.x; qt <= qt1; qt += kInvThreads)
        p.ucnt[((p.nqt - 1 - qt) * p.batch + b) * p.Hkv + hk] = -1;

    const int32_t *count = p.gcount + (int64_t)g * p.nblk_max;
    int *first = plan_smem;  // first item of each block, local to the group
    for (int s = threadIdx.x; s < p.nblk_max; s += kInvThreads) first[s] = (count[s] + p.Tq - 1) / p.Tq;
    __syncthreads();
    const int nitems = block_scan_array(first, p.nblk_max, scan_scratch);
    if (threadIdx.x == 0) item_base = atomicAdd(&p.ctrl->item_total, nitems);
    __syncthreads();
    int32_t *gfirst = p.gfirst + (int64_t)g * p.nblk_max;
    const int k0 = p.cu_k[b];
    for (int s = threadIdx.x; s < p.nblk_max; s += kInvThreads) {
        const int c = count[s];
        const int i0 = item_base + first[s];
        gfirst[s] = i0;
        for (int i = 0; i * p.Tq < c; ++i)
            p.items[i0 + i].rec = make_int4(b * p.Hkv + hk, s, k0, min(p.Tq, c - i * p.Tq));
    }
}

// Block-major token lists, one CTA per query tile of a block-major window: every (token, block)
// of the tile's canonical selections takes the next position in its block's list, which names
// the item (position / Tq) and the slot in it.
__global__ void __launch_bounds__(kPrepThreads) fwd_scatter_kernel(FwdScatterParams p)
{
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
    int32_t *cursor = p.gcursor + (int64_t)grp * p.nblk_max;
    const int32_t *first = p.gfirst + (int64_t)grp * p.nblk_max;
    const int tt = threadIdx.x;
    const int64_t t = (int64_t)q0 + tok0 + tt;
    const int n = tt < ntok ? p.cnt[t * p.Hkv + hk] : 0;
    const int32_t *row = p.sel_c + (t * p.Hkv + hk) * p.topk;
    const int maxn = __reduce_max_sync(0xffffffffu, n);
    for (int e = 0; e < maxn; ++e) {
        const int s = e < n ? row[e] : -1;
        // cursor is global here; warp_aggregated_add works on any address space
        const int pos = warp_aggregated_add(cursor, s);
        if (s >= 0) p.items[first[s] + pos / p.Tq].tok[pos % p.Tq] = (int)(t << 7) | e;
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
    const size_t smem = words * 4 + (size_t)g.Tq * g.topk * 4 + (size_t)g.topk * kPrepThreads * 4;
    if (smem > 48 * 1024) {
        const cudaError_t e = ensure_smem_for(fwd_prep_kernel, smem);
        if (e != cudaSuccess) return e;
    }
    fwd_prep_kernel<<<g.tiles, kPrepThreads, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_fwd_plan(const FwdGeom &g, const FwdPlanParams &p, cudaStream_t st)
{
    const size_t smem = (size_t)g.nblk_max * 4;
    return launch_kernel(fwd_plan_kernel, dim3(g.groups), dim3(kInvThreads), smem, st, true, p);
}

cudaError_t launch_fwd_scatter(const FwdGeom &g, const FwdScatterParams &p, cudaStream_t st)
{
    return launch_kernel(fwd_scatter_kernel, dim3(g.tiles), dim3(kPrepThreads), 0, st, true, p);
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
