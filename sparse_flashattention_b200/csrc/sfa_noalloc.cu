// sfa_decode_noalloc: the paged top-k decode for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: an inference engine whose memory
// pool is fixed before serving starts and forbids any cudaMalloc afterwards, a plugin hook that
// only receives input and output pointers from a host framework that owns every allocation,
// or code that must not touch the allocator for latency reasons.  For them this entry point
// keeps its scratch in a file-scope device array that the CUDA module reserves on every GPU
// that loads the library, for the life of the process.  It allocates nothing and otherwise
// runs exactly the same kernels as sfa_decode.
#include <mutex>

#include "sfa_internal.h"

namespace {

// Largest decode workspace this entry point can serve (sfa_decode_workspace_size of the call).
constexpr size_t kNoAllocScratchBytes = 8u << 20;

// The scratch itself.  In host code this name is only a stand-in for the device symbol, never a
// device address: the address is looked up per device with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the device that holds `q`, which must be the current device:
// the kernels run on the current device and read the array there, so a call whose tensors live on
// another GPU is refused rather than pointed at the wrong GPU's array.  Looked up once per device.
int scratch_for_device_of(const void *q, void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SFA_ERR_CUDA;
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, q) != cudaSuccess) {
        (void)cudaGetLastError();  // clear the error a non-device pointer leaves behind
        return SFA_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return SFA_ERR_INVALID_ARG;
    if (attr.device != dev) return SFA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return SFA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SFA_OK;
}

}  // namespace

extern "C" int sfa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *block_table, int max_pages_per_seq, int num_pages, int page_size,
                                  const int32_t *cache_seqlens, const int32_t *sel_tok_idx, int topk_tok, int B,
                                  int Hq, int Hkv, int d, int window_left, float scale, int num_splits,
                                  int32_t *status_dev, void *out, float *lse, sfa_stream_t stream)
{
    const size_t need = sfa_decode_workspace_size(B, Hq, Hkv, d, topk_tok, num_splits);
    if (need > kNoAllocScratchBytes) return SFA_ERR_WORKSPACE_TOO_SMALL;
    if (!q) return SFA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    const int rc = scratch_for_device_of(q, &scratch);
    if (rc != SFA_OK) return rc;
    return sfa_decode(q, k_cache, v_cache, block_table, max_pages_per_seq, num_pages, page_size, cache_seqlens,
                      sel_tok_idx, topk_tok, B, Hq, Hkv, d, window_left, scale, num_splits, scratch,
                      kNoAllocScratchBytes, status_dev, out, lse, stream);
}
