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
// Each thread owns kCompactItems consecutive elements of a tile, so a tile of
// kSelThreads * kCompactItems elements costs two block-wide scans.
constexpr int kCompactItems = 16;

template <typename KeyFn, typename EmitFn>
__device__ int block_compact(KeyFn key, int n, uint32_t T, int need_eq, bool take_all,
                             SelScratch &sc, EmitFn emit) {
    int out_base = 0, eq_base = 0;
    constexpr int kTile = kSelThreads * kCompactItems;
    for (int t0 = 0; t0 < n; t0 += kTile) {
        const int i0 = t0 + threadIdx.x * kCompactItems;
        uint32_t kk[kCompactItems];
        int ce = 0;
#pragma unroll
        for (int u = 0; u < kCompactItems; ++u) {
            const int i = i0 + u;
            kk[u] = (i < n) ? key(i) : 0u;
            ce += (i < n && !take_all && kk[u] == T) ? 1 : 0;
        }
        int eq_tot;
        int eq_rank = eq_base + block_excl_scan(ce, sc.warp, eq_tot);
        bool tk[kCompactItems];
        int ct = 0;
#pragma unroll
        for (int u = 0; u < kCompactItems; ++u) {
            const int i = i0 + u;
            bool take = false;
            if (i < n) {
                if (take_all || kk[u] > T) {
                    take = true;
                } else if (kk[u] == T) {
                    take = eq_rank < need_eq;
                    ++eq_rank;
                }
            }
            tk[u] = take;
            ct += take ? 1 : 0;
        }
        int tk_tot;
        int pos = out_base + block_excl_scan(ct, sc.warp, tk_tot);
#pragma unroll
        for (int u = 0; u < kCompactItems; ++u)
            if (tk[u]) emit(pos++, i0 + u, kk[u]);
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
    const int32_t *row_list;      // optional: rows to process (blockIdx -> row_list[i])
    const int32_t *list_count;    //   and how many entries of row_list are live
    int list_cap;                 //   capacity of row_list
    const uint32_t *keep;         // optional (prefill): kept 64-key blocks per row, a bit each;
    int keep_words;               //   a complete block without its bit is not visible
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

// One (row, slice): wrow is the row's slot in the candidate workspace.
__device__ __forceinline__ void idx_slice_row(const IdxArgs &a, const int slice, const int row,
                                              const int wrow, uint32_t *skey, float *sq, float *sw,
                                              SelScratch &sc) {
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
    const uint32_t *keep_row = a.keep ? a.keep + (size_t)row * a.keep_words : nullptr;
    const int n_full = nv >> 6;                  // complete 64-key blocks of the row
    for (int i = threadIdx.x; i < ns; i += kSelThreads) {
        if (keep_row) {
            const int blk = (s0 + i) >> 6;
            if (blk < n_full && !((keep_row[blk >> 5] >> (blk & 31)) & 1u)) {
                skey[i] = 0u;                    // not a candidate: ranks below every score
                continue;
            }
        }
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
        const size_t base = ((size_t)wrow * a.max_slices + slice) * topk;
        uint32_t *ck = a.cand_key + base;
        int32_t *ci = a.cand_idx + base;
        const int cnt = block_compact(key, ns, T, need_eq, take_all, sc,
                                      [&](int pos, int i, uint32_t kk) {
                                          ck[pos] = kk;
                                          ci[pos] = s0 + i;
                                      });
        if (threadIdx.x == 0) a.cand_cnt[(size_t)wrow * a.max_slices + slice] = cnt;
    }
}

// grid (slice, row); with a row list, grid.y CTAs stride over the list's live entries
__global__ void __launch_bounds__(kSelThreads) idx_slice_kernel(IdxArgs a) {
    extern __shared__ __align__(16) unsigned char idx_smem[];
    uint32_t *skey = reinterpret_cast<uint32_t *>(idx_smem);          // [kSlice]
    float *sq = reinterpret_cast<float *>(skey + kSlice);             // [H][64]
    float *sw = sq + kMaxIdxHeads * kIdxDim;                          // [H]
    __shared__ SelScratch sc;
    if (a.row_list) {
        const int live = min(*a.list_count, a.list_cap);
        for (int i = blockIdx.y; i < live; i += gridDim.y) {
            idx_slice_row(a, blockIdx.x, a.row_list[i], i, skey, sq, sw, sc);
            __syncthreads();
        }
    } else {
        idx_slice_row(a, blockIdx.x, blockIdx.y, ws_row(a, blockIdx.y), skey, sq, sw, sc);
    }
}

__device__ __forceinline__ void idx_merge_row(const IdxArgs &a, const int row, const int wr,
                                              SelScratch &sc, int *soff);

__global__ void __launch_bounds__(kSelThreads) idx_merge_kernel(IdxArgs a, int row0) {
    __shared__ SelScratch sc;
    __shared__ int soff[65];
    if (a.row_list) {
        const int live = min(*a.list_count, a.list_cap);
        for (int i = blockIdx.x; i < live; i += gridDim.x) {
            idx_merge_row(a, a.row_list[i], i, sc, soff);
            __syncthreads();
        }
    } else {
        idx_merge_row(a, row0 + blockIdx.x, ws_row(a, row0 + blockIdx.x), sc, soff);
    }
}

__device__ __forceinline__ void idx_merge_row(const IdxArgs &a, const int row, const int wr,
                                              SelScratch &sc, int *soff) {
    int64_t kb;
    int nv;
    row_range(a, row, kb, nv);
    nv = min(max(nv, 0), a.max_slices * kSlice);
    const int n_slices = ceil_div(nv, kSlice);
    if (n_slices <= 1 || nv <= a.topk) return;   // answered by idx_slice_kernel
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

// ---------------------------------------------------------------------------
// Decode path.  A decode row's scores are O(ctx) (one query per sequence), so
// they are written once as order-preserving keys (4 B per cached key) while
// the index-key cache is streamed; no score matrix exists.
//   idx_decode_score_kernel: grid (tile, row): 4096 keys per CTA, scores ->
//     keys, and a histogram of the keys' top 12 bits added to the row's
//     global histogram;
//   idx_decode_select_kernel: one CTA per row: the histogram locates the
//     12-bit bucket holding the k-th largest key; only that bucket's keys are
//     resolved exactly (radix select on the low bits), then one ordered
//     compaction over the row writes the ascending index list.
// ---------------------------------------------------------------------------
constexpr int kDecTile = 4096;
constexpr int kDecBins = 4096;            // top 12 bits of the key
constexpr int kDecThreads = 256;
constexpr int kDecEqCap = 16384;          // bucket size resolved in shared memory

struct DecArgs {
    const __nv_bfloat16 *q;
    const float *w;
    const __nv_bfloat16 *k;
    const int64_t *k_off;
    uint32_t *keys;                       // [rows][max_words * 32] score keys
    uint32_t *hist;                       // [rows][kDecBins]
    uint32_t *bm_gt, *bm_eq;              // [rows][max_words] position bitmaps
    uint2 *eq_buf;                        // [rows][kDecEqCap] (key, position) of bucket B
    int *eq_cnt;                          // [rows]
    int4 *info;                           // [rows]: bucket B, to take from B, |B|, 0
    int32_t *out_idx;
    int32_t *out_cnt;
    int n_rows, H, topk, max_tiles, max_words;
};

// Scores on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate):
// 16 keys form the M side (A operand, ldmatrix from a swizzled shared tile),
// the index heads (padded to 8) the N side, the 64 dims K.  Thread (g, t4)
// receives the dot products of keys g and g+8 with heads 2 t4 and 2 t4 + 1;
// the weighted ReLU sum over heads 0..3 needs one shuffle.  Each warp streams
// its own 16-key slices of the 4096-key tile through a 2-deep cp.async ring.
__device__ __forceinline__ void ldsm_x4_a(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecSlice = 16;                           // keys per mma slice

__global__ void __launch_bounds__(kDecThreads) idx_decode_score_kernel(DecArgs a) {
    __shared__ __align__(128) unsigned char ktile[kDecWarps][2][kDecSlice * 128];
    __shared__ uint32_t sh[kDecBins];
    const int tile = blockIdx.x, row = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t kb = a.k_off[row];
    int nv = (int)(a.k_off[row + 1] - kb);
    if (nv > a.max_words * 32) {                 // longer than the caller's bound
        if (tile == 0 && threadIdx.x == 0) raise_error(CRS_DEVERR_INDEX);
        nv = a.max_words * 32;
    }
    if (nv <= a.topk) return;                 // every key is selected; no score needed
    const int s0 = tile * kDecTile;
    if (s0 >= nv) return;
    const int ns = min(kDecTile, nv - s0);
    const int H = a.H;
    const int g = lane >> 2, t4 = lane & 3;
    // B fragments: head n = g (zero for n >= H), dims 16 kk + 2 t4 (+8)
    uint32_t bq[4][2];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t v = 0u;
            if (g < H) {
                const __nv_bfloat16 *qp = a.q + ((size_t)row * H + g) * kIdxDim + kk * 16 + hh * 8 + t4 * 2;
                v = *reinterpret_cast<const uint32_t *>(qp);
            }
            bq[kk][hh] = v;
        }
    }
    const float w0 = (2 * t4 < H) ? a.w[(size_t)row * H + 2 * t4] : 0.0f;
    const float w1 = (2 * t4 + 1 < H) ? a.w[(size_t)row * H + 2 * t4 + 1] : 0.0f;
    for (int e = threadIdx.x; e < kDecBins; e += kDecThreads) sh[e] = 0u;
    __syncthreads();

    const int nsl = (ns + kDecSlice - 1) / kDecSlice;     // 16-key slices in the tile
    bool nonfinite = false;
    auto issue = [&](int sl, int buf) {
        // 16 keys x 8 chunks of 16 B: lane handles chunks lane and lane + 32
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = lane + u * 32;
            const int r = e >> 3, c = e & 7;
            const int key = sl * kDecSlice + r;
            const bool ok = key < ns;
            const __nv_bfloat16 *src = a.k + (size_t)(kb + s0 + (ok ? key : 0)) * kIdxDim + c * 8;
            cp_async16_zfill(&ktile[warp][buf][0] + r * 128 + ((c ^ (r & 7)) << 4), src, ok);
        }
        cp_async_commit();
    };
    int sl = warp;
    if (sl < nsl) issue(sl, 0);
    for (int it = 0; sl < nsl; ++it, sl += kDecWarps) {
        const int buf = it & 1;
        const int nxt = sl + kDecWarps;
        if (nxt < nsl) {
            issue(nxt, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t base = smem_u32(&ktile[warp][buf][0]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            // A: rows = keys; matrices (keys 0-7, k lo), (8-15, lo), (0-7, hi), (8-15, hi)
            const int mi = lane >> 3;
            const int r = (lane & 7) + ((mi & 1) << 3);
            const int ch = kk * 2 + (mi >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_a(base + r * 128 + ((ch ^ (r & 7)) << 4), a0, a1, a2, a3);
            mma16816(c, a0, a1, a2, a3, bq[kk][0], bq[kk][1]);
        }
        // c0, c1: key g, heads 2 t4, 2 t4 + 1; c2, c3: key g + 8
        if (!isfinite(c[0]) || !isfinite(c[1]) || !isfinite(c[2]) || !isfinite(c[3])) nonfinite = true;
        float s_lo = fmaf(w0, fmaxf(c[0], 0.0f), w1 * fmaxf(c[1], 0.0f));
        float s_hi = fmaf(w0, fmaxf(c[2], 0.0f), w1 * fmaxf(c[3], 0.0f));
        // heads 2 t4 .. 2 t4 + 1 live in lanes t4 = 0..3 of the quad: sum the quad
        s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
        s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
        s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
        s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
        if (t4 == 0) {
            const int k_lo = sl * kDecSlice + g, k_hi = k_lo + 8;
            if (k_lo < ns) {
                const uint32_t key = score_key(s_lo);
                a.keys[(size_t)row * a.max_words * 32 + s0 + k_lo] = key;
                atomicAdd(&sh[key >> 20], 1u);
            }
            if (k_hi < ns) {
                const uint32_t key = score_key(s_hi);
                a.keys[(size_t)row * a.max_words * 32 + s0 + k_hi] = key;
                atomicAdd(&sh[key >> 20], 1u);
            }
        }
        __syncwarp();
    }
    if (__syncthreads_or(nonfinite) && threadIdx.x == 0) raise_error(CRS_DEVERR_NONFINITE);
    uint32_t *gh = a.hist + (size_t)row * kDecBins;
    for (int e = threadIdx.x; e < kDecBins; e += kDecThreads)
        if (sh[e]) atomicAdd(gh + e, sh[e]);
}

// Per row (one warp): the 12-bit bucket B that holds the topk-th largest key
// (from the top of the histogram), how many keys to take from it, and its size.
__global__ void __launch_bounds__(256) idx_decode_bucket_kernel(DecArgs a) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= a.n_rows) return;
    const uint32_t *gh = a.hist + (size_t)row * kDecBins;
    constexpr int per = kDecBins / 32;             // bins per lane, top-down
    int cnt = 0;
    {
        // lane l owns bins [kDecBins - per (l + 1), kDecBins - per l): 16-byte loads, all in flight
        const uint4 *g4 = reinterpret_cast<const uint4 *>(gh + kDecBins - per * (lane + 1));
        uint4 v[per / 4];
#pragma unroll
        for (int u = 0; u < per / 4; ++u) v[u] = g4[u];
#pragma unroll
        for (int u = 0; u < per / 4; ++u) cnt += (int)(v[u].x + v[u].y + v[u].z + v[u].w);
    }
    int incl = cnt;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o2);
        if (lane >= o2) incl += t;
    }
    const int before = incl - cnt, topk = a.topk;
    if (lane == 0) a.eq_cnt[row] = 0;
    if (lane == 31 && incl < topk) a.info[row] = make_int4(-1, 0, 0, 0);   // every key is taken
    if (before < topk && topk <= incl) {
        int acc = before;
        for (int u = 0; u < per; ++u) {
            const int bin = kDecBins - 1 - (lane * per + u);
            const int c = (int)gh[bin];
            if (acc < topk && topk <= acc + c) a.info[row] = make_int4(bin, topk - acc, c, 0);
            acc += c;
        }
    }
}

// grid (8192-key part, row): one warp per 32 keys writes the bitmap words of
// "bucket above B" (ballot) and clears the tie words; keys of bucket B go to
// the row's (key, position) list when it fits.
constexpr int kDecMarkKeys = 8192;
__global__ void __launch_bounds__(256) idx_decode_mark_kernel(DecArgs a) {
    const int row = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t kb = a.k_off[row];
    const int nv = min((int)(a.k_off[row + 1] - kb), a.max_words * 32);
    if (nv <= a.topk) return;
    const int4 inf = a.info[row];
    const uint32_t B = (uint32_t)inf.x;
    const bool collect = inf.z <= kDecEqCap;
    const uint32_t *keys = a.keys + (size_t)row * a.max_words * 32;
    const int w0 = blockIdx.x * (kDecMarkKeys / 32), w1 = min((nv + 31) / 32, w0 + kDecMarkKeys / 32);
    uint32_t *gt = a.bm_gt + (size_t)row * a.max_words;
    uint32_t *eqm = a.bm_eq + (size_t)row * a.max_words;
    for (int wb = w0 + warp * 4; wb < w1; wb += 32) {
        // four words per warp and iteration: four 128-byte loads in flight
        uint32_t kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = (wb + u) * 32 + lane;
            kv[u] = (wb + u < w1 && i < nv) ? keys[i] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
        const int w = wb + u;
        if (w >= w1) break;
        const int i = w * 32 + lane;
        const uint32_t kk = kv[u];
        const bool in = i < nv;
        const unsigned g = __ballot_sync(0xffffffffu, in && (kk >> 20) > B);
        const unsigned e = __ballot_sync(0xffffffffu, in && (kk >> 20) == B);
        if (lane == 0) {
            gt[w] = g;
            eqm[w] = 0u;
        }
        if (collect && e) {
            int base = 0;
            if (lane == 0) base = atomicAdd(a.eq_cnt + row, __popc(e));
            base = __shfl_sync(0xffffffffu, base, 0);
            if ((e >> lane) & 1u) {
                const int slot = base + __popc(e & ((1u << lane) - 1u));
                if (slot < kDecEqCap) a.eq_buf[(size_t)row * kDecEqCap + slot] = make_uint2(kk, (uint32_t)i);
            }
        }
        }
    }
}

// Per row: exact threshold inside bucket B, ties marked, then one ordered sweep
// over the position bitmaps writes the ascending index list (ties smallest
// position first).  A bucket too large for the list selects over the whole row.
__global__ void __launch_bounds__(kSelThreads) idx_decode_select_kernel(DecArgs a) {
    __shared__ SelScratch sc;
    const int row = blockIdx.x;
    const int64_t kb = a.k_off[row];
    int nv = (int)(a.k_off[row + 1] - kb);
    nv = min(max(nv, 0), a.max_words * 32);
    const int topk = a.topk;
    int32_t *o = a.out_idx + (size_t)row * topk;
    if (nv <= topk) {
        for (int i = threadIdx.x; i < topk; i += kSelThreads) o[i] = (i < nv) ? i : -1;
        if (threadIdx.x == 0) a.out_cnt[row] = nv;
        return;
    }
    const uint32_t *keys = a.keys + (size_t)row * a.max_words * 32;
    const int4 inf = a.info[row];
    int need_eq;
    if (inf.z > kDecEqCap) {
        // a very populated bucket (e.g. many exactly-equal scores): select over the whole row
        const uint32_t T = block_radix_select([&](int i) { return keys[i]; }, nv, topk, sc, need_eq);
        const int cnt = block_compact([&](int i) { return keys[i]; }, nv, T, need_eq, false, sc,
                                      [&](int pos, int i, uint32_t) { o[pos] = i; });
        for (int i = cnt + threadIdx.x; i < topk; i += kSelThreads) o[i] = -1;
        if (threadIdx.x == 0) a.out_cnt[row] = cnt;
        return;
    }
    // 1. exact threshold among bucket B's keys, then mark them
    const uint2 *eb = a.eq_buf + (size_t)row * kDecEqCap;
    const int size_b = min(a.eq_cnt[row], kDecEqCap);
    const uint32_t T = block_radix_select([&](int i) { return eb[i].x; }, size_b, inf.y, sc, need_eq);
    uint32_t *gt = a.bm_gt + (size_t)row * a.max_words;
    uint32_t *eqm = a.bm_eq + (size_t)row * a.max_words;
    for (int i = threadIdx.x; i < size_b; i += kSelThreads) {
        const uint2 v = eb[i];
        if (v.x > T) atomicOr(gt + (v.y >> 5), 1u << (v.y & 31));
        else if (v.x == T) atomicOr(eqm + (v.y >> 5), 1u << (v.y & 31));
    }
    __syncthreads();
    // 2. ordered sweep: thread t owns a contiguous run of words
    const int nwords = (nv + 31) / 32;
    const int per = (nwords + kSelThreads - 1) / kSelThreads;
    const int wa = min(nwords, threadIdx.x * per), wz = min(nwords, wa + per);
    int gtc = 0, eqc = 0;
    for (int w = wa; w < wz; ++w) {
        gtc += __popc(gt[w]);
        eqc += __popc(eqm[w]);
    }
    int tot;
    const int eq_before = block_excl_scan(eqc, sc.warp, tot);
    int allow = min(max(need_eq - eq_before, 0), eqc);   // ties this thread may take
    const int out0 = block_excl_scan(gtc + allow, sc.warp, tot);
    int pos = out0;
    for (int w = wa; w < wz; ++w) {
        uint32_t e = eqm[w];
        const int pe = __popc(e);
        if (pe > allow)
            for (int r = pe - allow; r > 0; --r) e &= ~(0x80000000u >> __clz(e));   // keep the lowest
        allow -= __popc(e);
        for (uint32_t m = gt[w] | e; m; m &= m - 1u) o[pos++] = w * 32 + (__ffs(m) - 1);
    }
    for (int i = tot + threadIdx.x; i < topk; i += kSelThreads) o[i] = -1;
    if (threadIdx.x == 0) a.out_cnt[row] = tot;
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

// tensor-core prefill path (indexer_tc.cu, same translation unit)
namespace crs {
static bool prefill_tc_applicable(const crs_indexer_params *p);
static size_t prefill_tc_workspace(const crs_indexer_params *p);
static int launch_prefill_tc(const crs_indexer_params *p, const void *q_idx, const float *wgt,
                             const void *k_idx, int32_t *out_idx, int32_t *out_count, void *ws,
                             cudaStream_t s, const uint32_t *keep, int keep_words, int top_blocks);
}  // namespace crs

struct DecWs {
    size_t keys, hist, bm, eq_buf, eq_cnt, info, total;   // byte offsets
};
static DecWs dec_ws_layout(const crs_indexer_params *p) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t rows = (size_t)p->n_rows;
    const size_t words = (size_t)ceil_div(max(p->max_keys, 1), 32);
    DecWs w;
    w.keys = 0;
    w.hist = w.keys + al(rows * words * 32 * 4);   // score keys, fixed stride per row
    w.bm = w.hist + al(rows * kDecBins * 4);
    w.eq_buf = w.bm + al(rows * words * 4 * 2);
    w.eq_cnt = w.eq_buf + al(rows * kDecEqCap * 8);
    w.info = w.eq_cnt + al(rows * 4);
    w.total = w.info + al(rows * 16);
    return w;
}

extern "C" size_t crs_indexer_topk_workspace_size(const crs_indexer_params *p) {
    if (idx_validate(p)) return 0;
    if (p->mode == CRS_IDX_DECODE) return dec_ws_layout(p).total;
    if (prefill_tc_applicable(p)) return prefill_tc_workspace(p);
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p->mode == CRS_IDX_DECODE) {
        const DecWs L = dec_ws_layout(p);
        char *wb = static_cast<char *>(ws);
        DecArgs d;
        d.q = static_cast<const __nv_bfloat16 *>(q_idx);
        d.w = w;
        d.k = static_cast<const __nv_bfloat16 *>(k_idx);
        d.k_off = k_offsets;
        d.keys = reinterpret_cast<uint32_t *>(wb + L.keys);
        d.hist = reinterpret_cast<uint32_t *>(wb + L.hist);
        d.max_words = ceil_div(max(p->max_keys, 1), 32);
        d.bm_gt = reinterpret_cast<uint32_t *>(wb + L.bm);
        d.bm_eq = d.bm_gt + (size_t)p->n_rows * d.max_words;
        d.eq_buf = reinterpret_cast<uint2 *>(wb + L.eq_buf);
        d.eq_cnt = reinterpret_cast<int *>(wb + L.eq_cnt);
        d.info = reinterpret_cast<int4 *>(wb + L.info);
        d.out_idx = out_idx;
        d.out_cnt = out_count;
        d.n_rows = p->n_rows;
        d.H = p->n_idx_heads;
        d.topk = p->topk;
        d.max_tiles = max(1, ceil_div(p->max_keys, kDecTile));
        CRS_TRY_CUDA(cudaMemsetAsync(d.hist, 0, (size_t)p->n_rows * kDecBins * 4, s));
        {
            ProfScope _ps(K_IDX_SLICE, s);
            idx_decode_score_kernel<<<dim3(d.max_tiles, p->n_rows), kDecThreads, 0, s>>>(d);
        }
        CRS_CHECK_LAUNCH();
        {
            ProfScope _ps(K_IDX_SELECT, s);
            idx_decode_bucket_kernel<<<ceil_div(p->n_rows, 8), 256, 0, s>>>(d);
        }
        CRS_CHECK_LAUNCH();
        {
            ProfScope _ps(K_IDX_SELECT, s);
            idx_decode_mark_kernel<<<dim3(ceil_div(d.max_tiles * kDecTile, kDecMarkKeys), p->n_rows), 256, 0, s>>>(d);
        }
        CRS_CHECK_LAUNCH();
        {
            ProfScope _ps(K_IDX_SELECT, s);
            idx_decode_select_kernel<<<p->n_rows, kSelThreads, 0, s>>>(d);
        }
        CRS_CHECK_LAUNCH();
        return CRS_OK;
    }
    if (prefill_tc_applicable(p))
        return launch_prefill_tc(p, q_idx, w, k_idx, out_idx, out_count, ws, s, nullptr, 0, 0);
    int max_slices, ws_rows;
    idx_geometry(p, max_slices, ws_rows);
    if (max_slices > 64) return CRS_ERR_UNSUPPORTED;
    IdxArgs a;
    a.row_list = nullptr;
    a.list_count = nullptr;
    a.list_cap = 0;
    a.keep = nullptr;
    a.keep_words = 0;
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
