// In-place append of new key / value rows to a paged KV cache: row j of sequence b goes to logical
// position cache_seqlens[b] + j, i.e. page block_table[b][pos / page_size], row pos % page_size —
// the k / v arguments of flash_attn_with_kvcache (flash-attention-npu page, "FlashAttention v2" API
// docstrings).  One thread per 16-byte piece of a (sequence, new row, kv head) row, K and V both;
// consecutive threads take consecutive pieces of a row (coalesced on both sides).
#include "sfa_device.cuh"

namespace sfa {

namespace {

__global__ void __launch_bounds__(256) kv_append_kernel(KvAppendParams p)
{
    const int per_row = p.d / 8;  // 16-byte pieces per (row, kv head)
    const int64_t total = (int64_t)p.B * p.S * p.Hkv * per_row;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = idx / per_row;  // (b, j, hk) in the layout of k_new
        const int piece = (int)(idx - row * per_row);
        const int hk = (int)(row % p.Hkv);
        const int64_t bj = row / p.Hkv;
        const int j = (int)(bj % p.S), b = (int)(bj / p.S);
        const int64_t pos = (int64_t)__ldg(&p.seqlens[b]) + j;
        const int64_t blk = pos / p.page;
        if (pos < 0 || blk >= p.max_pages) {
            if (piece == 0 && hk == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_SEQLEN);
            continue;
        }
        const int pg = __ldg(&p.bt[(int64_t)b * p.max_pages + blk]);
        if (pg < 0 || pg >= p.num_pages) {
            if (piece == 0 && hk == 0 && p.status) atomicOr(p.status, SFA_DEV_BAD_PAGE);
            continue;
        }
        const int64_t dst = (((int64_t)pg * p.page + pos % p.page) * p.Hkv + hk) * p.d + piece * 8;
        const int64_t src = row * p.d + piece * 8;
        *reinterpret_cast<uint4 *>(p.k_cache + dst) = __ldg(reinterpret_cast<const uint4 *>(p.k_new + src));
        *reinterpret_cast<uint4 *>(p.v_cache + dst) = __ldg(reinterpret_cast<const uint4 *>(p.v_new + src));
    }
}

}  // namespace

cudaError_t launch_kv_append(const KvAppendParams &p, cudaStream_t st)
{
    const int64_t total = (int64_t)p.B * p.S * p.Hkv * (p.d / 8);
    if (total == 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, 148 * 16);
    kv_append_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sfa
