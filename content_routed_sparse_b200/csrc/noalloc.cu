// crs_block_select_noalloc: block selection with its scratch in a static device array.
//
// Who this is for: callers that cannot allocate device memory when they call
// the library, for example an engine whose memory pool owns the whole device
// and rejects allocations after start-up, a plugin host that hands its plugins
// only input and output buffers, or a latency-bound loop where the cost and
// the implicit device synchronization of cudaMalloc/cudaFree are not allowed.
// Such a caller cannot provide the workspace crs_block_select asks for.  This
// entry point takes the same inputs and outputs and finds its scratch in
// g_noalloc_scratch, a fixed array that is part of the library image: every
// GPU that loads libcrs holds these 16 MiB until the process exits.
//
// The array's name is only a host-side stand-in for the device object; the
// device address is fetched once per device with cudaGetSymbolAddress (with
// that device current) the first time this entry point runs on it, and then
// reused.  The kernels (the same ones crs_block_select launches) overwrite
// every scratch entry before they read it, so nothing has to be cleared
// between calls; the array keeps the last call's contents.
#include <mutex>

#include "common.cuh"

namespace crs {

constexpr size_t kNoAllocScratchBytes = CRS_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set up once per device).
static int noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CRS_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return CRS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) return CRS_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return CRS_OK;
}

}  // namespace crs

extern "C" int crs_block_select_noalloc(const crs_block_sel_params *p, const void *Q,
                                        const float *mu, const float *xi, int32_t *tok_idx,
                                        int32_t *tok_count, void *stream) {
    int st = bs_validate(p);
    if (st) return st;
    if (crs_block_select_workspace_size(p) > crs::kNoAllocScratchBytes) return CRS_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = crs::noalloc_scratch(&scratch);
    if (st) return st;
    return crs_block_select(p, Q, mu, xi, tok_idx, tok_count, scratch, crs::kNoAllocScratchBytes,
                            stream);
}
