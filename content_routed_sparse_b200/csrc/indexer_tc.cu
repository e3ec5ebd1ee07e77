// Prefill lightning indexer on the tensor cores (tcgen05 + TMA), exact top-k.
//
// [P2] PaperTrace 2.2 "细粒度索引" §1.1 (r_{t,s} = sum_h w_{t,h} ReLU(q_{t,h} . k_s),
// one shared index key), §2.1 ("Select 不等于一次普通 top-k": the score matrix is
// never stored; slices are filtered and merged), "Index K 全扫的字节下界"
// (prefill index Q and K form a matrix product: "tiled GEMM + streaming top-k").
//
// One CTA per 128-query tile, keys in tiles of 64 (causal: keys <= the tile's
// last row).  Warp roles: warp 0 loads Q (once) and K tiles with TMA into a
// ring of shared buffers; warp 1 issues tcgen05.mma for the 4 index heads
// (M=128, N=64, K=64 each) into one of two TMEM accumulator sets
// (4 heads x 64 columns); warps 4..11 read the accumulators (warp quadrant =
// rows, two warps per quadrant split the 64 keys), form the weighted ReLU sum
// and act on the scores.  Two modes:
//   SAMPLE: every 8th key tile; scores (top 16 bits of the order-preserving
//           key) are written out per row;
//   FILTER: every key tile; a score whose key is >= the row's threshold is
//           appended to that (row, key half)'s candidate list.
// idx_tc_tau_kernel picks each row's threshold from its samples so that about
// 1.25 k scores pass; idx_tc_final_kernel merges a row's two candidate lists by
// position and selects the exact top-k (ties to the smaller position); a row
// whose candidates number fewer than k or overflowed a list is recomputed by
// the exact CUDA-core slice path.  The threshold only decides how much work
// the final selection sees, never the result.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc.cuh"

namespace crs {

constexpr int kIqM = 128;           // query rows per CTA
constexpr int kIkN = 64;            // keys per tile
constexpr int kIH = 4;              // index heads on this path
constexpr int kID = 64;             // index head dim
constexpr int kIStages = 8;         // K-tile ring
constexpr int kISampStride = 8;     // SAMPLE mode: every 8th key tile
constexpr int kICapHalf = 2048;     // candidates per (row, key half)
constexpr int kIFallbackRows = 4096;
constexpr int kIThreads = 384;      // 12 warps
constexpr uint64_t kIWaitNs = 2000000000ull;
constexpr float kIBeta = 1.25f;

struct IdxTcSmem {
    unsigned char q[kIH][kIqM * 128];        // per head: 128 rows x 64 dims, SW128
    unsigned char k[kIStages][kIkN * 128];   // key tiles: 64 keys x 64 dims, SW128
    float w[kIqM][kIH];
    uint32_t tau[kIqM];
    uint64_t qfull;
    uint64_t kfull[kIStages];
    uint64_t kempty[kIStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int fail;
};

struct IdxTcArgs {
    const float *w;           // [n, 4]
    const uint32_t *tau;      // [n] FILTER thresholds (order-preserving keys)
    uint16_t *samples;        // [n, samp_slots] SAMPLE output (0 = no sample)
    uint32_t *cand_key;       // [n, 2, kICapHalf]
    int32_t *cand_idx;        // [n, 2, kICapHalf]
    int32_t *cand_cnt;        // [n, 2]
    int n, samp_slots, n_tiles_rows;
};

template <int MODE>   // 0 = SAMPLE, 1 = FILTER
__global__ void __launch_bounds__(kIThreads, 1)
idx_prefill_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      IdxTcArgs a) {
    extern __shared__ unsigned char idx_tc_raw[];
    const uint32_t mis = smem_u32(idx_tc_raw) & 1023u;
    IdxTcSmem &S = *reinterpret_cast<IdxTcSmem *>(idx_tc_raw + ((1024u - mis) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // heaviest tiles first: row tile i has i+1 times the work of tile 0
    const int tile_i = a.n_tiles_rows - 1 - blockIdx.x;
    const int r0 = tile_i * kIqM;
    const int key_end = min(a.n, r0 + kIqM);                  // causal: keys < key_end
    const int nt_all = (key_end + kIkN - 1) / kIkN;
    const int ntiles = MODE == 0 ? (nt_all + kISampStride - 1) / kISampStride : nt_all;

    if (tid == 0) {
        tc::mbar_init(&S.qfull, 1);
        for (int i = 0; i < kIStages; ++i) {
            tc::mbar_init(&S.kfull[i], 1);
            tc::mbar_init(&S.kempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&S.tfull[i], 1);
            tc::mbar_init(&S.tempty[i], 8);       // one arrival per epilogue warp
        }
        tc::mbar_fence_init();
        S.fail = 0;
    }
    for (int e = tid; e < kIqM * kIH; e += kIThreads) {
        const int r = e / kIH, h = e - r * kIH;
        const int t = r0 + r;
        S.w[r][h] = (t < a.n) ? a.w[(size_t)t * kIH + h] : 0.0f;
    }
    if (MODE == 1)
        for (int r = tid; r < kIqM; r += kIThreads) S.tau[r] = (r0 + r < a.n) ? a.tau[r0 + r] : 0u;
    if (warp == 2) tc::tmem_alloc(&S.tmem_base, 512);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(&S.qfull, kIH * kIqM * 128);
            for (int h = 0; h < kIH; ++h) tc::tma_load_3d(S.q[h], &tq, 0, h, r0, &S.qfull);
            for (int j = 0; j < ntiles; ++j) {
                const int s = j % kIStages, u = j / kIStages;
                if (u > 0 &&
                    !tc::mbar_wait_bounded(&S.kempty[s], (u - 1) & 1, kIWaitNs, K_IDX_PREFILL_TC, 1)) {
                    atomicOr(&S.fail, 1);
                    break;
                }
                const int kt = MODE == 0 ? j * kISampStride : j;
                tc::mbar_arrive_expect_tx(&S.kfull[s], kIkN * 128);
                tc::tma_load_2d(S.k[s], &tk, 0, kt * kIkN, &S.kfull[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16_f32(kIqM, kIkN, 0, 0);
            bool ok = tc::mbar_wait_bounded(&S.qfull, 0, kIWaitNs, K_IDX_PREFILL_TC, 2);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j % kIStages, u = j / kIStages;
                const int b = j & 1, v = j >> 1;
                ok = tc::mbar_wait_bounded(&S.kfull[s], u & 1, kIWaitNs, K_IDX_PREFILL_TC, 3);
                if (ok && v > 0) ok = tc::mbar_wait_bounded(&S.tempty[b], (v - 1) & 1, kIWaitNs, K_IDX_PREFILL_TC, 4);
                if (!ok) break;
                tc::fence_after();
                const uint32_t kbase = smem_u32(S.k[s]);
#pragma unroll
                for (int h = 0; h < kIH; ++h) {
                    const uint32_t qbase = smem_u32(S.q[h]);
#pragma unroll
                    for (int k = 0; k < kID / 16; ++k) {
                        const uint64_t ad = tc::smem_desc(qbase + k * 32, 16, 1024, tc::kLayoutSW128);
                        const uint64_t bd = tc::smem_desc(kbase + k * 32, 16, 1024, tc::kLayoutSW128);
                        tc::mma_bf16(tmem + b * 256 + h * 64, ad, bd, idesc, k > 0 ? 1u : 0u);
                    }
                }
                tc::commit(&S.kempty[s]);
                tc::commit(&S.tfull[b]);
            }
            if (!ok) atomicOr(&S.fail, 1);
        }
    } else if (warp >= 4) {
        // ---------------- epilogue: row = quadrant * 32 + lane, key half hf
        const int quad = warp & 3, hf = (warp - 4) >> 2;
        const int row = quad * 32 + lane;
        const int t = r0 + row;
        const bool row_ok = t < a.n;
        float wr[kIH];
#pragma unroll
        for (int h = 0; h < kIH; ++h) wr[h] = S.w[row][h];
        const uint32_t tau = MODE == 1 ? S.tau[row] : 0u;
        int cnt = 0;
        const size_t cbase = ((size_t)(row_ok ? t : 0) * 2 + hf) * kICapHalf;
        const uint32_t tq_lane = tmem + ((uint32_t)(quad * 32) << 16);
        bool nonfinite = false;
        for (int j = 0; j < ntiles; ++j) {
            const int b = j & 1, v = j >> 1;
            const bool ok = tc::mbar_wait_bounded(&S.tfull[b], v & 1, kIWaitNs, K_IDX_PREFILL_TC, 5);
            if (__any_sync(0xffffffffu, !ok)) {
                if (lane == 0) atomicOr(&S.fail, 1);
                break;
            }
            tc::fence_after();
            float sc[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) sc[i] = 0.0f;
#pragma unroll
            for (int h = 0; h < kIH; ++h) {
                uint32_t d[32];
                tc::tmem_ld32(tq_lane + b * 256 + h * 64 + hf * 32, d);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float x = __uint_as_float(d[i]);
                    nonfinite |= !isfinite(x);
                    sc[i] = fmaf(wr[h], fmaxf(x, 0.0f), sc[i]);
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.tempty[b]);
            const int kt = MODE == 0 ? j * kISampStride : j;
            const int key0 = kt * kIkN + hf * 32;
            if constexpr (MODE == 0) {
                if (row_ok) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        uint32_t lo = 0u, hi = 0u;
                        const int ka = key0 + 2 * i, kb2 = ka + 1;
                        if (ka <= t) lo = score_key(sc[2 * i]) >> 16;
                        if (kb2 <= t) hi = score_key(sc[2 * i + 1]) >> 16;
                        pk[i] = lo | (hi << 16);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(a.samples + (size_t)t * a.samp_slots +
                                                           j * kIkN + hf * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u) dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                }
            } else {
                if (row_ok) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int key = key0 + i;
                        const uint32_t kk = score_key(sc[i]);
                        if (key <= t && kk >= tau) {
                            if (cnt < kICapHalf) {
                                a.cand_key[cbase + cnt] = kk;
                                a.cand_idx[cbase + cnt] = key;
                            }
                            ++cnt;
                        }
                    }
                }
            }
        }
        if (MODE == 1 && row_ok) a.cand_cnt[(size_t)t * 2 + hf] = cnt;
        if (nonfinite) raise_error(CRS_DEVERR_NONFINITE);
    }
    tc::fence_before();
    __syncthreads();
    if (S.fail && tid == 0) raise_error(CRS_DEVERR_TIMEOUT);
    if (warp == 2) tc::tmem_dealloc(tmem, 512);
}


// ---------------------------------------------------------------------------
// Per-row threshold from the samples (one warp per row): with n_valid sampled
// keys out of t+1 visible, keep the R = ceil(1.25 k n_valid / (t+1))-th largest
// sample's top 16 bits; every key at or above it passes the filter (about
// 1.25 k of them).  Rows with t+1 <= k, or too few samples, pass everything.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) idx_tc_tau_kernel(const uint16_t *__restrict__ samples,
                                                         uint32_t *__restrict__ tau, int n,
                                                         int samp_slots, int topk) {
    __shared__ int hist[8][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= n) return;
    int *hw = hist[warp];
    if (t + 1 <= topk) {
        if (lane == 0) tau[t] = 0u;
        return;
    }
    const int key_end = min(n, (t / kIqM) * kIqM + kIqM);
    const int nt_all = (key_end + kIkN - 1) / kIkN;
    const int slots = ((nt_all + kISampStride - 1) / kISampStride) * kIkN;
    const uint16_t *sp = samples + (size_t)t * samp_slots;
    for (int b = lane; b < 256; b += 32) hw[b] = 0;
    __syncwarp();
    int nvalid = 0;
    for (int i = lane; i < slots; i += 32) {
        const uint32_t v = sp[i];
        if (v) {
            ++nvalid;
            atomicAdd(&hw[v >> 8], 1);
        }
    }
    nvalid = warp_sum_int(nvalid);
    __syncwarp();
    const long long R = ((long long)nvalid * topk * 5 + 4LL * (t + 1) - 1) / (4LL * (t + 1));  // ceil(1.25 k nv/(t+1))
    if (R < 1 || R > nvalid) {
        if (lane == 0) tau[t] = 0u;
        return;
    }
    // top-down scan of 256 bins: lane l owns bins [255 - 8l - 7, 255 - 8l]
    auto find = [&](int need, int &bin, int &rem) {
        int c[8], s = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) { c[u] = hw[255 - (lane * 8 + u)]; s += c[u]; }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        const int before = incl - s;
        int fb = -1, fr = 0;
        if (before < need && need <= incl) {
            int acc = before;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (fb < 0 && acc < need && need <= acc + c[u]) { fb = 255 - (lane * 8 + u); fr = need - acc; }
                acc += c[u];
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, fb >= 0);
        const int src = m ? __ffs(m) - 1 : 0;
        bin = __shfl_sync(0xffffffffu, fb, src);
        rem = __shfl_sync(0xffffffffu, fr, src);
    };
    int b1, rem1;
    find((int)R, b1, rem1);
    __syncwarp();
    for (int b = lane; b < 256; b += 32) hw[b] = 0;
    __syncwarp();
    for (int i = lane; i < slots; i += 32) {
        const uint32_t v = sp[i];
        if (v && (int)(v >> 8) == b1) atomicAdd(&hw[v & 255], 1);
    }
    __syncwarp();
    int b2, rem2;
    find(rem1, b2, rem2);
    if (lane == 0) tau[t] = ((uint32_t)b1 << 24) | ((uint32_t)b2 << 16);
}

// ---------------------------------------------------------------------------
// Per row: merge the two candidate lists by position, exact top-k, ascending
// output.  Rows whose lists overflowed, or hold fewer than k candidates, are
// queued for the exact slice path.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSelThreads)
idx_tc_final_kernel(const uint32_t *__restrict__ cand_key, const int32_t *__restrict__ cand_idx,
                    const int32_t *__restrict__ cand_cnt, int32_t *__restrict__ out_idx,
                    int32_t *__restrict__ out_cnt, int32_t *__restrict__ fb_list,
                    int32_t *__restrict__ fb_count, int n, int topk) {
    __shared__ SelScratch sc;
    __shared__ int32_t aidx[kICapHalf], bidx[kICapHalf];
    extern __shared__ uint32_t mrg[];            // [2 * kICapHalf] keys, then [2 * kICapHalf] positions
    const int t = blockIdx.x;
    int32_t *o = out_idx + (size_t)t * topk;
    if (t + 1 <= topk) {
        for (int i = threadIdx.x; i < topk; i += kSelThreads) o[i] = (i <= t) ? i : -1;
        if (threadIdx.x == 0) out_cnt[t] = t + 1;
        return;
    }
    const int c0 = cand_cnt[(size_t)t * 2], c1 = cand_cnt[(size_t)t * 2 + 1];
    if (c0 > kICapHalf || c1 > kICapHalf || c0 + c1 < topk) {
        if (threadIdx.x == 0) {
            const int pos = atomicAdd(fb_count, 1);
            if (pos < kIFallbackRows) fb_list[pos] = t;
            else raise_error(CRS_DEVERR_INDEX);
        }
        return;
    }
    const size_t ba = (size_t)t * 2 * kICapHalf, bb = ba + kICapHalf;
    for (int i = threadIdx.x; i < c0; i += kSelThreads) aidx[i] = cand_idx[ba + i];
    for (int i = threadIdx.x; i < c1; i += kSelThreads) bidx[i] = cand_idx[bb + i];
    __syncthreads();
    uint32_t *mk = mrg;
    int32_t *mi = reinterpret_cast<int32_t *>(mrg + 2 * kICapHalf);
    auto lower = [](const int32_t *arr, int len, int x) {
        int lo = 0, hi = len;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (arr[mid] < x) lo = mid + 1; else hi = mid;
        }
        return lo;
    };
    for (int i = threadIdx.x; i < c0; i += kSelThreads) {
        const int p = i + lower(bidx, c1, aidx[i]);
        mk[p] = cand_key[ba + i];
        mi[p] = aidx[i];
    }
    for (int i = threadIdx.x; i < c1; i += kSelThreads) {
        const int p = i + lower(aidx, c0, bidx[i]);
        mk[p] = cand_key[bb + i];
        mi[p] = bidx[i];
    }
    __syncthreads();
    const int N = c0 + c1;
    int need_eq = 0;
    const uint32_t T = block_radix_select([&](int i) { return mk[i]; }, N, topk, sc, need_eq);
    const int cnt = block_compact([&](int i) { return mk[i]; }, N, T, need_eq, false, sc,
                                  [&](int pos, int i, uint32_t) { o[pos] = mi[i]; });
    for (int i = cnt + threadIdx.x; i < topk; i += kSelThreads) o[i] = -1;
    if (threadIdx.x == 0) out_cnt[t] = cnt;
}

// ----------------------------------------------------------------- host --
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

struct PrefillTcWs {
    uint16_t *samples;
    uint32_t *tau;
    uint32_t *cand_key;
    int32_t *cand_idx;
    int32_t *cand_cnt;
    int32_t *fb_list;
    int32_t *fb_count;
    uint32_t *fb_ckey;
    int32_t *fb_cidx;
    int32_t *fb_ccnt;
    int samp_slots, fb_slices;
    size_t total;
};

static void prefill_tc_layout(int n, int topk, PrefillTcWs &w, char *base) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const int n_key_tiles = (n + kIkN - 1) / kIkN;
    w.samp_slots = ((n_key_tiles + kISampStride - 1) / kISampStride) * kIkN;
    w.fb_slices = max(1, ceil_div(n, kSlice));
    const int fbr = min(n, kIFallbackRows);
    size_t off = 0;
    auto take = [&](size_t bytes) { char *p = base ? base + off : nullptr; off += al(bytes); return p; };
    w.samples = reinterpret_cast<uint16_t *>(take((size_t)n * w.samp_slots * 2));
    w.tau = reinterpret_cast<uint32_t *>(take((size_t)n * 4));
    w.cand_key = reinterpret_cast<uint32_t *>(take((size_t)n * 2 * kICapHalf * 4));
    w.cand_idx = reinterpret_cast<int32_t *>(take((size_t)n * 2 * kICapHalf * 4));
    w.cand_cnt = reinterpret_cast<int32_t *>(take((size_t)n * 2 * 4));
    w.fb_list = reinterpret_cast<int32_t *>(take((size_t)fbr * 4));
    w.fb_count = reinterpret_cast<int32_t *>(take(4));
    w.fb_ckey = reinterpret_cast<uint32_t *>(take((size_t)fbr * w.fb_slices * topk * 4));
    w.fb_cidx = reinterpret_cast<int32_t *>(take((size_t)fbr * w.fb_slices * topk * 4));
    w.fb_ccnt = reinterpret_cast<int32_t *>(take((size_t)fbr * w.fb_slices * 4));
    w.total = off;
}

static bool prefill_tc_applicable(const crs_indexer_params *p) {
    return p->mode == CRS_IDX_PREFILL && p->n_idx_heads == kIH && p->d_idx == kID &&
           p->topk <= kICapHalf && p->n_rows >= 1 && p->n_rows <= 64 * kSlice;
}

static size_t prefill_tc_workspace(const crs_indexer_params *p) {
    PrefillTcWs w;
    prefill_tc_layout(p->n_rows, p->topk, w, nullptr);
    return w.total;
}

static int launch_prefill_tc(const crs_indexer_params *p, const void *q_idx, const float *wgt,
                             const void *k_idx, int32_t *out_idx, int32_t *out_count, void *ws,
                             cudaStream_t s) {
    const int n = p->n_rows, topk = p->topk;
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return CRS_ERR_CUDA;
    if ((reinterpret_cast<uintptr_t>(q_idx) & 15) || (reinterpret_cast<uintptr_t>(k_idx) & 15))
        return CRS_ERR_INVALID_ARG;
    CUtensorMap tq, tk;
    {
        cuuint64_t dims[3] = {(cuuint64_t)kID, (cuuint64_t)kIH, (cuuint64_t)n};
        cuuint64_t strides[2] = {(cuuint64_t)kID * 2, (cuuint64_t)kIH * kID * 2};
        cuuint32_t box[3] = {(cuuint32_t)kID, 1, (cuuint32_t)kIqM};
        cuuint32_t estr[3] = {1, 1, 1};
        if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q_idx), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CRS_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)kID, (cuuint64_t)n};
        cuuint64_t strides[1] = {(cuuint64_t)kID * 2};
        cuuint32_t box[2] = {(cuuint32_t)kID, (cuuint32_t)kIkN};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(k_idx), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CRS_ERR_CUDA;
    }
    PrefillTcWs w;
    prefill_tc_layout(n, topk, w, static_cast<char *>(ws));
    IdxTcArgs a;
    a.w = wgt;
    a.tau = w.tau;
    a.samples = w.samples;
    a.cand_key = w.cand_key;
    a.cand_idx = w.cand_idx;
    a.cand_cnt = w.cand_cnt;
    a.n = n;
    a.samp_slots = w.samp_slots;
    a.n_tiles_rows = ceil_div(n, kIqM);
    const size_t smem = sizeof(IdxTcSmem) + 1024;
    CRS_TRY_CUDA(cudaFuncSetAttribute(idx_prefill_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    CRS_TRY_CUDA(cudaFuncSetAttribute(idx_prefill_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    CRS_TRY_CUDA(cudaMemsetAsync(w.fb_count, 0, 4, s));
    {
        ProfScope _ps(K_IDX_PREFILL_TC, s);
        idx_prefill_tc_kernel<0><<<a.n_tiles_rows, kIThreads, smem, s>>>(tq, tk, a);
    }
    CRS_CHECK_LAUNCH();
    {
        ProfScope _ps(K_IDX_SELECT, s);
        idx_tc_tau_kernel<<<ceil_div(n, 8), 256, 0, s>>>(w.samples, w.tau, n, w.samp_slots, topk);
    }
    CRS_CHECK_LAUNCH();
    {
        ProfScope _ps(K_IDX_PREFILL_TC, s);
        idx_prefill_tc_kernel<1><<<a.n_tiles_rows, kIThreads, smem, s>>>(tq, tk, a);
    }
    CRS_CHECK_LAUNCH();
    const int dsm = 4 * kICapHalf * 4;
    CRS_TRY_CUDA(cudaFuncSetAttribute(idx_tc_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsm));
    {
        ProfScope _ps(K_IDX_SELECT, s);
        idx_tc_final_kernel<<<n, kSelThreads, dsm, s>>>(w.cand_key, w.cand_idx, w.cand_cnt, out_idx,
                                                          out_count, w.fb_list, w.fb_count, n, topk);
    }
    CRS_CHECK_LAUNCH();
    // exact slice path for the queued rows (usually none)
    IdxArgs f;
    f.mode = CRS_IDX_PREFILL;
    f.q = static_cast<const __nv_bfloat16 *>(q_idx);
    f.w = wgt;
    f.k = static_cast<const __nv_bfloat16 *>(k_idx);
    f.k_off = nullptr;
    f.out_idx = out_idx;
    f.out_cnt = out_count;
    f.cand_key = w.fb_ckey;
    f.cand_idx = w.fb_cidx;
    f.cand_cnt = w.fb_ccnt;
    f.n_rows = n;
    f.H = kIH;
    f.topk = topk;
    f.max_slices = w.fb_slices;
    f.row_list = w.fb_list;
    f.list_count = w.fb_count;
    const int fbr = min(n, kIFallbackRows);
    const size_t ssm = (size_t)kSlice * 4 + (kMaxIdxHeads * kIdxDim + kMaxIdxHeads) * 4;
    CRS_TRY_CUDA(cudaFuncSetAttribute(idx_slice_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm));
    {
        ProfScope _ps(K_IDX_SLICE, s);
        idx_slice_kernel<<<dim3(w.fb_slices, fbr), kSelThreads, ssm, s>>>(f);
    }
    CRS_CHECK_LAUNCH();
    if (w.fb_slices > 1) {
        ProfScope _ps(K_IDX_MERGE, s);
        idx_merge_kernel<<<fbr, kSelThreads, 0, s>>>(f, 0);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

}  // namespace crs
