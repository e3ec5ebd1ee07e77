// The candidate sets of the chunked LSH attention as an explicit CSR matrix
// (an inspection export for small inputs), sm_100a.
//
// [P1] PaperTrace 2.1.1 §2.1-2.2 and §1.1 Eq.(2): in round r, query i meets
// the key j when j sits in i's chunk or in the chunk before it (chunks of m
// sorted slots), shares i's bucket, and passes the causal (j <= i), self
// (j != i) and padding (j < valid_len) masks; "重复候选和归一化": the set over
// several rounds is their union, each key once.  §4 (the index tensors
// row_ptr / col_idx, perm, inverse_perm) names the CSR form.
//
// One CTA per query row: the (round, window slot) pairs are split over the
// threads; a pair met in an earlier round is dropped by the same first-round
// test the attention kernels use, so every key is counted once; the row's keys
// are collected in shared memory and sorted ascending (bitonic).
#include "common.cuh"

namespace crs {

constexpr int kCsrThreads = 256;
constexpr int kCsrMax = 2 * 128 * kMaxRounds;   // window slots x rounds: 2048

struct CsrArgs {
    const int32_t *bucket, *perm, *inv_perm, *valid_len;
    int64_t *row_ptr;
    int32_t *col_idx;
    int H, n, m, rounds, causal, no_self;
};

// Key j of window entry e (round e / (2m), slot offset e % (2m)) when it belongs to
// U(i) and this is the first round it is met in; -1 otherwise.
__device__ __forceinline__ int csr_entry(const CsrArgs &a, size_t seg0, int i, int vl, int e,
                                         const int *ci, const int *bi) {
    const int r = e / (2 * a.m), t = e - r * 2 * a.m;
    const int s = (ci[r] - 1) * a.m + t;
    if (s < 0 || s >= a.n) return -1;
    const size_t sg = seg0 + (size_t)r * a.n;
    const int j = a.perm[sg + s];
    if (j < 0 || j >= a.n) {
        raise_error(CRS_DEVERR_INDEX);
        return -1;
    }
    if (a.bucket[sg + j] != bi[r]) return -1;
    if (a.causal && j > i) return -1;
    if (a.no_self && j == i) return -1;
    if (j >= vl) return -1;
    for (int rr = 0; rr < r; ++rr) {                 // met in an earlier round?
        const size_t s2 = seg0 + (size_t)rr * a.n;
        if (a.bucket[s2 + j] != bi[rr]) continue;
        const int cj = a.inv_perm[s2 + j] / a.m;
        if (cj == ci[rr] || cj == ci[rr] - 1) return -1;
    }
    return j;
}

// pass 0: counts into row_ptr[row + 1]; pass 1: the sorted keys into col_idx
template <int PASS>
__global__ void __launch_bounds__(kCsrThreads) lsh_csr_kernel(CsrArgs a) {
    __shared__ int ci[kMaxRounds], bi[kMaxRounds];
    __shared__ int keys[kCsrMax];
    __shared__ int cnt;
    const long long row = blockIdx.x;               // (b*h) * n + i
    const int bh = (int)(row / a.n), i = (int)(row - (long long)bh * a.n);
    const size_t seg0 = (size_t)bh * a.rounds * a.n;
    const int vl = a.valid_len ? a.valid_len[bh / a.H] : a.n;
    if (threadIdx.x < a.rounds) {
        const size_t sg = seg0 + (size_t)threadIdx.x * a.n;
        int slot = a.inv_perm[sg + i];
        if (slot < 0 || slot >= a.n) {
            raise_error(CRS_DEVERR_INDEX);
            slot = -2 * a.m;                         // a window with no slot in range
        }
        ci[threadIdx.x] = slot >= 0 ? slot / a.m : slot;
        bi[threadIdx.x] = a.bucket[sg + i];
    }
    if (threadIdx.x == 0) cnt = 0;
    __syncthreads();
    const int total = a.rounds * 2 * a.m;
    int local = 0;
    for (int e = threadIdx.x; e < total; e += kCsrThreads) {
        const int j = csr_entry(a, seg0, i, vl, e, ci, bi);
        if (j >= 0) {
            if (PASS == 0) ++local;
            else keys[atomicAdd(&cnt, 1)] = j;
        }
    }
    if (PASS == 0) {
        local = __reduce_add_sync(0xffffffffu, local);
        if ((threadIdx.x & 31) == 0 && local) atomicAdd(&cnt, local);
        __syncthreads();
        if (threadIdx.x == 0) a.row_ptr[row + 1] = cnt;
        if (row == 0 && threadIdx.x == 0) a.row_ptr[0] = 0;
        return;
    }
    __syncthreads();
    const int c = cnt;
    int len = 32;
    while (len < c) len <<= 1;
    for (int e = c + threadIdx.x; e < len; e += kCsrThreads) keys[e] = 0x7fffffff;
    __syncthreads();
    for (int k = 2; k <= len; k <<= 1) {
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            for (int e = threadIdx.x; e < len; e += kCsrThreads) {
                const int p = e ^ jj;
                if (p > e) {
                    const int x = keys[e], y = keys[p];
                    const bool up = (e & k) == 0;
                    if ((x > y) == up) {
                        keys[e] = y;
                        keys[p] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
    const int64_t base = a.row_ptr[row];
    const int64_t cap = a.row_ptr[row + 1] - base;
    const int room = (int64_t)c < cap ? c : (int)(cap > 0 ? cap : 0);
    for (int e = threadIdx.x; e < room; e += kCsrThreads) a.col_idx[base + e] = keys[e];
}

// Inclusive prefix sum of row_ptr[1..rows] in place (one CTA; row_ptr[0] = 0).
__global__ void __launch_bounds__(1024) lsh_csr_scan_kernel(int64_t *row_ptr, long long rows) {
    __shared__ int64_t part[1024];
    const long long per = (rows + 1023) / 1024;
    const long long b0 = 1 + threadIdx.x * per, b1 = min(rows + 1, b0 + per);
    int64_t s = 0;
    for (long long k = b0; k < b1; ++k) s += row_ptr[k];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {       // Hillis-Steele over the 1024 partials
        const int64_t v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int64_t run = threadIdx.x ? part[threadIdx.x - 1] : 0;
    for (long long k = b0; k < b1; ++k) {
        run += row_ptr[k];
        row_ptr[k] = run;
    }
}

}  // namespace crs

using namespace crs;

extern "C" int crs_lsh_candidates_csr(const crs_lsh_attn_params *a, const int32_t *bucket,
                                      const int32_t *perm, const int32_t *inv_perm,
                                      const int32_t *valid_len, int64_t *row_ptr, int32_t *col_idx,
                                      void *stream) {
    if (!a) return CRS_ERR_INVALID_ARG;
    const crs_lsh_params &p = a->p;
    if (p.B < 1 || p.H < 1 || p.n < 1 || p.n_rounds < 1 || p.n_rounds > kMaxRounds)
        return CRS_ERR_INVALID_ARG;
    if (p.chunk < 1 || p.chunk > 128) return CRS_ERR_INVALID_ARG;
    if (!bucket || !perm || !inv_perm || !row_ptr) return CRS_ERR_INVALID_ARG;
    const long long rows = (long long)p.B * p.H * p.n;
    if (p.n > 65536 || rows > (1LL << 22)) return CRS_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CsrArgs ca{bucket, perm, inv_perm, valid_len, row_ptr, col_idx, p.H, p.n, p.chunk, p.n_rounds,
               a->causal ? 1 : 0, a->no_self ? 1 : 0};
    if (!col_idx) {
        {
            ProfScope _ps(K_LSH_CSR, s);
            lsh_csr_kernel<0><<<(unsigned)rows, kCsrThreads, 0, s>>>(ca);
        }
        CRS_CHECK_LAUNCH();
        {
            ProfScope _ps(K_LSH_CSR, s);
            lsh_csr_scan_kernel<<<1, 1024, 0, s>>>(row_ptr, rows);
        }
        CRS_CHECK_LAUNCH();
        return CRS_OK;
    }
    {
        ProfScope _ps(K_LSH_CSR, s);
        lsh_csr_kernel<1><<<(unsigned)rows, kCsrThreads, 0, s>>>(ca);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}
