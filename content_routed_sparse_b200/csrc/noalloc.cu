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
// reused while the device's current context stays the same one (after a
// cudaDeviceReset the module is loaded again and the address is fetched anew).
// The kernels (the same ones crs_block_select launches) overwrite
// every scratch entry before they read it, so nothing has to be cleared
// between calls; the array keeps the last call's contents.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace crs {

constexpr size_t kNoAllocScratchBytes = CRS_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[kNoAllocMaxDevices] = {};
static unsigned long long g_noalloc_ctx_id[kNoAllocMaxDevices] = {};

// Unique id of the current context (cuCtxGetCurrent + cuCtxGetId, looked up once
// through the runtime: no link-time dependency on libcuda); 0 when unknown.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
static unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked = false;
    if (!looked) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        looked = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_noalloc_scratch on the current device: set up once per device
// and context, fetched again when the current context is not the one it was set up
// in (or cannot be identified).
static int noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CRS_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return CRS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    unsigned long long id = current_ctx_id();
    if (!g_noalloc_ptr[dev] || id == 0 || id != g_noalloc_ctx_id[dev]) {
        void *ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) return CRS_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
        if (id == 0) id = current_ctx_id();     // the lookup made the primary context current
        g_noalloc_ctx_id[dev] = id;
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
