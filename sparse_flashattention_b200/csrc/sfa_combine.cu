// Gated mix of NSA branch outputs: out[t,h,:] = sum_c g_c[t,h] * o_c[t,h,:].
//
// The Flash-Sparse-Attention module combines its compressed, selected and sliding-window
// attention branches per query token and head with gate values ("Relaxed-System-Lab/
// Flash-Sparse-Attention" project page, quick-start module arguments; README feature list,
// "Gated attention").  HBM-bound elementwise work: each thread takes one 16-byte chunk (8
// values) of a row from every branch, accumulates in fp32 and writes the bf16 chunk.
#include "sfa_device.cuh"

namespace sfa {

namespace {

constexpr int kCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) gated_combine_kernel(CombineParams p)
{
    constexpr int kChunks = D / 8;
    const int64_t e = (int64_t)blockIdx.x * kCombineThreads + threadIdx.x;  // (row, chunk)
    if (e >= p.rows * kChunks) return;
    const int64_t row = e / kChunks;
    const int c = (int)(e - row * kChunks);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int b = 0; b < 3; ++b) {
        if (!p.o[b]) continue;
        const float g = __ldg(&p.g[b][row]);
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p.o[b] + row * D) + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
            const float2 f = __bfloat1622float2(h);
            acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
            acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
        }
    }
    uint4 r;
    r.x = pack_bf16x2(acc[0], acc[1]);
    r.y = pack_bf16x2(acc[2], acc[3]);
    r.z = pack_bf16x2(acc[4], acc[5]);
    r.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4 *>(p.out + row * D)[c] = r;
}

}  // namespace

cudaError_t launch_gated_combine(const CombineParams &p, int d, cudaStream_t st)
{
    const int64_t work = p.rows * (d / 8);
    const unsigned grid = (unsigned)((work + kCombineThreads - 1) / kCombineThreads);
    if (grid == 0) return cudaSuccess;
    if (d == 64) gated_combine_kernel<64><<<grid, kCombineThreads, 0, st>>>(p);
    else gated_combine_kernel<128><<<grid, kCombineThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace sfa
