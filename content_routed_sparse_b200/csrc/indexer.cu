// Lightning-indexer scores and exact token top-k, sm_100a.
//
// [P2] PaperTrace 2.2 "细粒度索引": §1.1 (score = sum_h w_h ReLU(q_h . k),
// one shared index key), §2.1 Eq.(3)-(4) (Select over r_{t,0:t}; "Select 不等于
// 一次普通 top-k": per-slice candidates merged 2k -> k equal the global top-k,
// the full score matrix is never stored; invalid slots explicit), §3.1 "多卡
// 一致性" (ties broken on (score, index)), "Index K 全扫的字节下界" (decode is a
// contiguous scan of the index-key cache).
//
// Pipeline (both modes): keys of a row are cut into slices of kSlice keys.
//   idx_slice_kernel:  one CTA per (row, slice): scores on CUDA cores into
//                      shared memory as order-preserving uint32 keys, exact
//                      radix select of the slice's top-k, kept in index order;
//                      a row with one slice writes its final answer here.
//   idx_merge_kernel:  one CTA per multi-slice row: exact radix select over
//                      the concatenated slice candidates (index order is kept
//                      by construction), written ascending with -1 padding.
// Ties: a larger key wins; equal keys are taken in increasing position.
#include <math.h>

#include "common.cuh"

namespace crs {

constexpr int kSlice = 16384;          // keys per slice
constexpr int kSelThreads = 512;
constexpr int kMaxIdxHeads = 8;
constexpr int kIdxDim = 64;

// ---------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread (kSelThreads threads).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_excl_scan(int v, int *sh_warp, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sh_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        constexpr int NW = kSelThreads / 32;
        int w = (lane < NW) ? sh_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < NW) sh_warp[lane] = wi - w;       // exclusive warp offsets
        if (lane == NW - 1) sh_warp[32] = wi;        // total
    }
    __syncthreads();
    const int res = sh_warp[warp] + incl - v;
    total = sh_warp[32];
    __syncthreads();
    return res;
}

struct SelScratch {
    int hist[256];
    int warp[33];
    int bcast[4];
};

// Exact selection of the k largest keys among n (key(i), i ascending = index
// order).  Returns the threshold key T and, through need_eq, how many
// elements equal to T are taken (the first ones in index order).
template <typename KeyFn>
__device__ uint32_t block_radix_select(KeyFn key, int n, int k, SelScratch &sc, int &need_eq) {
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = tid; b < 256; b += kSelThreads) sc.hist[b] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kSelThreads) {
            const uint32_t kk = key(i);
            if ((kk & mask) == prefix) atomicAdd(&sc.hist[(kk >> shift) & 255], 1);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns digits [255 - 8l - 7, 255 - 8l], scanned from the top
            int c[8];
            int s = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) { c[u] = sc.hist[255 - (lane * 8 + u)]; s += c[u]; }
            int incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int before = incl - s;   // count in higher digits
            if (before < remaining && remaining <= incl) {
                int acc = before;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (acc < remaining && remaining <= acc + c[u]) {
                        sc.bcast[0] = 255 - (lane * 8 + u);
                        sc.bcast[1] = remaining - acc;
                    }
                    acc += c[u];
                }
            }
        }
        __syncthreads();
        const uint32_t d = (uint32_t)sc.bcast[0];
        remaining = sc.bcast[1];
        prefix |= d << shift;
        mask |= 0xffu << shift;
        __syncthreads();
    }
    need_eq = remaining;
    return prefix;
}

// Writes, in index order, the selected elements: key > T, plus the first
// need_eq elements with key == T.  emit(pos, i, key) is called per element.
template <typename KeyFn, typename EmitFn>
__device__ int block_compact(KeyFn key, int n, uint32_t T, int need_eq, bool take_all,
                             SelScratch &sc, EmitFn emit) {
    int out_base = 0, eq_base = 0;
    for (int t0 = 0; t0 < n; t0 += kSelThreads) {
        const int i = t0 + threadIdx.x;
        uint32_t kk = 0;
        bool gt = false, eq = false;
        if (i < n) {
            kk = key(i);
            gt = take_all || kk > T;
            eq = !take_all && kk == T;
        }
        int eq_tot;
        const int eq_rank = eq_base + block_excl_scan(eq ? 1 : 0, sc.warp, eq_tot);
        const bool take = gt || (eq && eq_rank < need_eq);
        int tk_tot;
        const int pos = out_base + block_excl_scan(take ? 1 : 0, sc.warp, tk_tot);
        if (take) emit(pos, i, kk);
        out_base += tk_tot;
        eq_base += eq_tot;
    }
    return out_base;
}

struct IdxArgs {
    int mode;
    const __nv_bfloat16 *q;       // [rows, H, 64]
    const float *w;               // [rows, H]
    const __nv_bfloat16 *k;       // [keys, 64]
    const int64_t *k_off;         // decode: [rows+1]
    int32_t *out_idx;             // [rows, topk]
    int32_t *out_cnt;             // [rows]
    uint32_t *cand_key;           // [ws_rows, max_slices, topk]
    int32_t *cand_idx;            // [ws_rows, max_slices, topk]
    int32_t *cand_cnt;            // [ws_rows, max_slices]
    int n_rows, H, topk, max_slices;
};

__device__ __forceinline__ void row_range(const IdxArgs &a, int row, int64_t &kb, int &nv) {
    if (a.mode == CRS_IDX_PREFILL) {
        kb = 0;
        nv = row + 1;
    } else {
        kb = a.k_off[row];
        const int64_t e = a.k_off[row + 1];
        nv = (int)(e - kb);
    }
}

// rows whose candidates go through the merge: prefill rows with > kSlice keys
__device__ __forceinline__ int ws_row(const IdxArgs &a, int row) {
    return a.mode == CRS_IDX_PREFILL ? row - kSlice : row;
}

__global__ void __launch_bounds__(kSelThreads) idx_slice_kernel(IdxArgs a) {
    extern __shared__ __align__(16) unsigned char idx_smem[];
    uint32_t *skey = reinterpret_cast<uint32_t *>(idx_smem);          // [kSlice]
    float *sq = reinterpret_cast<float *>(skey + kSlice);             // [H][64]
    float *sw = sq + kMaxIdxHeads * kIdxDim;                          // [H]
    __shared__ SelScratch sc;

    const int slice = blockIdx.x, row = blockIdx.y;
    int64_t kb;
    int nv;
    row_range(a, row, kb, nv);
    if (nv < 0) nv = 0;
    if (nv > a.max_slices * kSlice) {            // longer than the caller's bound
        if (threadIdx.x == 0 && slice == 0) raise_error(CRS_DEVERR_INDEX);
        nv = a.max_slices * kSlice;
    }
    const int n_slices = ceil_div(nv, kSlice);
    if (slice >= max(n_slices, 1)) return;
    const int s0 = slice * kSlice;
    const int ns = min(kSlice, nv - s0);
    const int topk = a.topk;

    if (nv <= topk) {
        // every visible key is selected; no score is needed
        if (slice == 0) {
            int32_t *o = a.out_idx + (size_t)row * topk;
            for (int i = threadIdx.x; i < topk; i += kSelThreads) o[i] = (i < nv) ? i : -1;
            if (threadIdx.x == 0) a.out_cnt[row] = nv;
        }
        return;
    }

    const int H = a.H;
    for (int e = threadIdx.x; e < H * kIdxDim; e += kSelThreads)
        sq[e] = __bfloat162float(a.q[(size_t)row * H * kIdxDim + e]);
    for (int e = threadIdx.x; e < H; e += kSelThreads) sw[e] = a.w[(size_t)row * H + e];
    __syncthreads();

    // ---- scores: one thread per key, 128-byte key rows read as 8 x 16 B
    bool nonfinite = false;
    for (int i = threadIdx.x; i < ns; i += kSelThreads) {
        const uint4 *kr = reinterpret_cast<const uint4 *>(a.k + (size_t)(kb + s0 + i) * kIdxDim);
        float kf[kIdxDim];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint4 v = kr[u];
            const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f = __bfloat1622float2(p2[t]);
                kf[u * 8 + t * 2] = f.x;
                kf[u * 8 + t * 2 + 1] = f.y;
            }
        }
        float s = 0.0f;
        for (int h = 0; h < H; ++h) {
            float dot = 0.0f;
#pragma unroll
            for (int t = 0; t < kIdxDim; ++t) dot = fmaf(sq[h * kIdxDim + t], kf[t], dot);
            // fmaxf(NaN, 0) is 0: test the dot product itself before the ReLU
            if (!isfinite(dot)) nonfinite = true;
            s = fmaf(sw[h], fmaxf(dot, 0.0f), s);
        }
        if (!isfinite(s)) nonfinite = true;
        skey[i] = score_key(s);
    }
    if (__syncthreads_or(nonfinite) && threadIdx.x == 0) raise_error(CRS_DEVERR_NONFINITE);

    auto key = [&](int i) { return skey[i]; };
    int need_eq = 0;
    uint32_t T = 0;
    const bool take_all = ns <= topk;
    if (!take_all) T = block_radix_select(key, ns, topk, sc, need_eq);

    if (n_slices == 1) {
        int32_t *o = a.out_idx + (size_t)row * topk;
        const int cnt = block_compact(key, ns, T, need_eq, take_all, sc,
                                      [&](int pos, int i, uint32_t) { o[pos] = s0 + i; });
        for (int i = cnt + threadIdx.x; i < topk; i += kSelThreads) o[i] = -1;
        if (threadIdx.x == 0) a.out_cnt[row] = cnt;
    } else {
        const size_t base = ((size_t)ws_row(a, row) * a.max_slices + slice) * topk;
        uint32_t *ck = a.cand_key + base;
        int32_t *ci = a.cand_idx + base;
        const int cnt = block_compact(key, ns, T, need_eq, take_all, sc,
                                      [&](int pos, int i, uint32_t kk) {
                                          ck[pos] = kk;
                                          ci[pos] = s0 + i;
                                      });
        if (threadIdx.x == 0) a.cand_cnt[(size_t)ws_row(a, row) * a.max_slices + slice] = cnt;
    }
}

__global__ void __launch_bounds__(kSelThreads) idx_merge_kernel(IdxArgs a, int row0) {
    __shared__ SelScratch sc;
    __shared__ int soff[65];
    const int row = row0 + blockIdx.x;
    int64_t kb;
    int nv;
    row_range(a, row, kb, nv);
    nv = min(max(nv, 0), a.max_slices * kSlice);
    const int n_slices = ceil_div(nv, kSlice);
    if (n_slices <= 1 || nv <= a.topk) return;   // answered by idx_slice_kernel
    const int wr = ws_row(a, row);
    const int topk = a.topk;
    if (threadIdx.x == 0) {
        int s = 0;
        for (int c = 0; c < n_slices; ++c) {
            soff[c] = s;
            s += a.cand_cnt[(size_t)wr * a.max_slices + c];
        }
        soff[n_slices] = s;
    }
    __syncthreads();
    const int N = soff[n_slices];
    const uint32_t *ck = a.cand_key + (size_t)wr * a.max_slices * topk;
    const int32_t *ci = a.cand_idx + (size_t)wr * a.max_slices * topk;
    auto where = [&](int i) {
        int c = 0;
        while (c + 1 < n_slices && soff[c + 1] <= i) ++c;
        return (size_t)c * topk + (i - soff[c]);
    };
    auto key = [&](int i) { return ck[where(i)]; };
    int need_eq = 0;
    uint32_t T = 0;
    const bool take_all = N <= topk;
    if (!take_all) T = block_radix_select(key, N, topk, sc, need_eq);
    int32_t *o = a.out_idx + (size_t)row * topk;
    const int cnt = block_compact(key, N, T, need_eq, take_all, sc,
                                  [&](int pos, int i, uint32_t) { o[pos] = ci[where(i)]; });
    for (int i = cnt + threadIdx.x; i < topk; i += kSelThreads) o[i] = -1;
    if (threadIdx.x == 0) a.out_cnt[row] = cnt;
}

static int idx_validate(const crs_indexer_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->mode != CRS_IDX_PREFILL && p->mode != CRS_IDX_DECODE) return CRS_ERR_INVALID_ARG;
    if (p->n_rows < 1 || p->n_idx_heads < 1 || p->n_idx_heads > kMaxIdxHeads)
        return CRS_ERR_INVALID_ARG;
    if (p->d_idx != kIdxDim) return CRS_ERR_UNSUPPORTED;
    if (p->topk < 1 || p->topk > 4096) return CRS_ERR_INVALID_ARG;
    if (p->mode == CRS_IDX_DECODE && p->max_keys < 0) return CRS_ERR_INVALID_ARG;
    return CRS_OK;
}

static void idx_geometry(const crs_indexer_params *p, int &max_slices, int &ws_rows) {
    if (p->mode == CRS_IDX_PREFILL) {
        max_slices = ceil_div(p->n_rows, kSlice);
        ws_rows = max(0, p->n_rows - kSlice);
    } else {
        max_slices = max(1, ceil_div(p->max_keys, kSlice));
        ws_rows = p->n_rows;
    }
}

}  // namespace crs

using namespace crs;

extern "C" size_t crs_indexer_topk_workspace_size(const crs_indexer_params *p) {
    if (idx_validate(p)) return 0;
    int max_slices, ws_rows;
    idx_geometry(p, max_slices, ws_rows);
    if (max_slices <= 1 || ws_rows == 0) return 0;
    const size_t cand = (size_t)ws_rows * max_slices * p->topk;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    return al(cand * 4) * 2 + al((size_t)ws_rows * max_slices * 4);
}

extern "C" int crs_indexer_topk(const crs_indexer_params *p, const void *q_idx, const float *w,
                                const void *k_idx, const int64_t *k_offsets, int32_t *out_idx,
                                int32_t *out_count, void *ws, size_t ws_bytes, void *stream) {
    int st = idx_validate(p);
    if (st) return st;
    if (!q_idx || !w || !k_idx || !out_idx || !out_count) return CRS_ERR_INVALID_ARG;
    if (p->mode == CRS_IDX_DECODE && !k_offsets) return CRS_ERR_INVALID_ARG;
    const size_t need = crs_indexer_topk_workspace_size(p);
    if (need > 0 && (!ws || ws_bytes < need)) return CRS_ERR_WORKSPACE;
    int max_slices, ws_rows;
    idx_geometry(p, max_slices, ws_rows);
    if (max_slices > 64) return CRS_ERR_UNSUPPORTED;
    IdxArgs a;
    a.mode = p->mode;
    a.q = static_cast<const __nv_bfloat16 *>(q_idx);
    a.w = w;
    a.k = static_cast<const __nv_bfloat16 *>(k_idx);
    a.k_off = k_offsets;
    a.out_idx = out_idx;
    a.out_cnt = out_count;
    a.n_rows = p->n_rows;
    a.H = p->n_idx_heads;
    a.topk = p->topk;
    a.max_slices = max_slices;
    a.cand_key = nullptr;
    a.cand_idx = nullptr;
    a.cand_cnt = nullptr;
    if (need > 0) {
        const size_t cand = (size_t)ws_rows * max_slices * p->topk;
        auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
        char *b = static_cast<char *>(ws);
        a.cand_key = reinterpret_cast<uint32_t *>(b);
        a.cand_idx = reinterpret_cast<int32_t *>(b + al(cand * 4));
        a.cand_cnt = reinterpret_cast<int32_t *>(b + 2 * al(cand * 4));
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t smem = (size_t)kSlice * 4 + (kMaxIdxHeads * kIdxDim + kMaxIdxHeads) * 4;
    CRS_TRY_CUDA(cudaFuncSetAttribute(idx_slice_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem));
    dim3 grid(max_slices, p->n_rows);
    {
        ProfScope _ps(K_IDX_SLICE, s);
        idx_slice_kernel<<<grid, kSelThreads, smem, s>>>(a);
    }
    CRS_CHECK_LAUNCH();
    if (max_slices > 1) {
        const int row0 = (p->mode == CRS_IDX_PREFILL) ? kSlice : 0;
        const int nrows = p->n_rows - row0;
        if (nrows > 0) {
            {
                ProfScope _ps(K_IDX_MERGE, s);
                idx_merge_kernel<<<nrows, kSelThreads, 0, s>>>(a, row0);
            }
            CRS_CHECK_LAUNCH();
        }
    }
    return CRS_OK;
}
