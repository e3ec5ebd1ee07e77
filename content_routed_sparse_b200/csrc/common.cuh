// Shared device helpers for libcrs kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "crs.h"

namespace crs {

// Per-device error word (CRS_DEVERR_* bits), read and cleared by crs_get_device_error.
// The library is built as one translation unit (libcrs.cu), so this is its only definition.
__device__ uint32_t g_device_error = 0;

__device__ __forceinline__ void raise_error(uint32_t bit) { atomicOr(&g_device_error, bit); }

// Debug switch (crs_debug_force_wait_timeout): while non-zero, the bounded waits
// marked as forceable give up at once, so a test can drive the timeout path
// (error bit, diagnostic record, drain, early return) without a stuck barrier.
__device__ uint32_t g_force_wait_timeout = 0;

// Diagnostic record of the first failure a kernel reports about itself:
// [0] = kernel id + 1 (0: none), [1] = where (kernel-defined site), [2..4] =
// blockIdx.x/y/z, [5..] = kernel-defined values.  Read by crs_get_device_diag.
__device__ uint32_t g_device_diag[16] = {};
__device__ __forceinline__ void diag_record(uint32_t kernel, uint32_t site, uint32_t a,
                                            uint32_t b, uint32_t c, uint32_t d) {
    if (atomicCAS(&g_device_diag[0], 0u, kernel + 1u) == 0u) {
        g_device_diag[1] = site;
        g_device_diag[2] = blockIdx.x;
        g_device_diag[3] = blockIdx.y;
        g_device_diag[4] = blockIdx.z;
        g_device_diag[5] = a;
        g_device_diag[6] = b;
        g_device_diag[7] = c;
        g_device_diag[8] = d;
    }
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Order-preserving map of an fp32 score to uint32: a > b  <=>  key(a) > key(b)
// for non-NaN a, b, with -0 and +0 mapped to the same key.  NaN maps to 0,
// below every number.
__device__ __forceinline__ uint32_t score_key(float s) {
    if (s != s) return 0u;
    s = s + 0.0f;  // -0 -> +0
    uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// packed fp32 pairs (sm_100 f32x2 arithmetic) and a NaN-propagating ReLU
__device__ __forceinline__ uint64_t f32x2_pack(float x, float y) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float &x, float &y) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ float relu_nan(float x) {
    float r;
    asm("max.NaN.f32 %0, %1, 0f00000000;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float fmax_nan(float x, float y) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(x), "f"(y));
    return r;
}

constexpr int kMaxRounds = 8;   // LSH hash rounds supported by the attention kernels

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ long long ceil_div_ll(long long a, long long b) {
    return (a + b - 1) / b;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global -> shared copy (sm_80+ path, valid on sm_100a).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
// CTA-wide sum of one count per thread (blockDim.x a multiple of 32): warp sums
// go to one of two shared arrays and a single barrier publishes them.  Every
// thread makes the same sequence of calls with its own parity ph (flipped
// here), so an array is rewritten only after all threads passed the barrier of
// the call that followed its last reading.
__device__ __forceinline__ int cta_count(int local, int &ph) {
    __shared__ int cbuf[2][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ws = __reduce_add_sync(0xffffffffu, local);
    if (lane == 0) cbuf[ph][warp] = ws;
    __syncthreads();
    const int v = lane < (int)(blockDim.x >> 5) ? cbuf[ph][lane] : 0;
    ph ^= 1;
    return __reduce_add_sync(0xffffffffu, v);
}

__device__ __forceinline__ void cp_async16_zfill(void *smem, const void *gmem, bool valid) {
    int src_size = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
                 "l"(gmem), "r"(src_size));
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace crs

// Host-side helpers shared by the entry points.
#define CRS_TRY_CUDA(expr)                          \
    do {                                            \
        cudaError_t _e = (expr);                    \
        if (_e != cudaSuccess) return CRS_ERR_CUDA; \
    } while (0)

#define CRS_CHECK_LAUNCH()                                   \
    do {                                                     \
        if (cudaGetLastError() != cudaSuccess) return CRS_ERR_CUDA; \
    } while (0)

// ---------------------------------------------------------------------------
// Launch tracing: every kernel launch site opens a ProfScope.  Launches are
// always counted; while tracing is enabled (crs_profile_set) each launch is
// also bracketed by a pair of CUDA events recorded on its own stream, and
// crs_profile_collect turns them into per-kernel device times.
// ---------------------------------------------------------------------------
namespace crs {
enum KernelId {
    K_LSH_HASH = 0, K_LSH_SORT, K_LSH_ATTN, K_LSH_COMBINE, K_IDX_SLICE, K_IDX_MERGE,
    K_SA_MAIN, K_SA_MERGE, K_BLK_DESCRIBE, K_BLK_SCORE, K_BLK_PICK, K_LSH_ATTN_TC,
    K_IDX_PREFILL_TC, K_IDX_SELECT, K_NOALLOC, K_BLK_QUANTIZE, K_HISA, K_LSH_DECODE, K_ROUTE, K_LSH_CSR, K_LSH_ATTN_RING, K_COUNT
};
void prof_begin(int id, cudaStream_t s, void **ev_start);
void prof_end(int id, cudaStream_t s, void *ev_start);
void prof_add_launches(int id, int k);
// One scope counts one kernel launch; a scope that launches more kernels
// calls more(k) for the k further launches.
struct ProfScope {
    int id;
    cudaStream_t s;
    void *ev;
    ProfScope(int id_, cudaStream_t s_) : id(id_), s(s_), ev(nullptr) { prof_begin(id, s, &ev); }
    ~ProfScope() { prof_end(id, s, ev); }
    void more(int k) { prof_add_launches(id, k); }
};
}  // namespace crs
