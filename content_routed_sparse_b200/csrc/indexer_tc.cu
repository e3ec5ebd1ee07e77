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
// (4 heads x 64 columns); warp 2 owns the TMEM allocation; warps 4..19 read
// the accumulators (warp % 4 = TMEM lane quadrant = 32 query rows, four warps
// per quadrant take 16 keys each), release them at once, and form the
// weighted ReLU sum with paired fp32 FMAs.  Two modes:
//   SAMPLE: every 8th key tile; scores (top 16 bits of the order-preserving
//           key) are written out per row;
//   FILTER: every key tile; a score whose key is >= the row's threshold is
//           appended to that (row, part)'s candidate list.
// idx_tc_tau_kernel picks each row's threshold from its samples so that about
// 1.25 k scores pass; idx_tc_final_kernel selects the exact top-k over a row's
// four candidate lists (ties to the smaller position, output ascending); a
// row whose candidates number fewer than k or overflowed a list is recomputed
// by the exact CUDA-core slice path.  The threshold only decides how much work
// the final selection sees, never the result.
#include <cuda.h>
#include <float.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc.cuh"

namespace crs {

constexpr int kIqM = 128;           // query rows per CTA
constexpr int kIkN = 64;            // keys per tile
constexpr int kIH = 4;              // index heads on this path
constexpr int kID = 64;             // index head dim
constexpr int kIStages = 3;         // K-tile ring
constexpr int kISampStride = 8;     // SAMPLE mode: every 8th key tile
constexpr int kIParts = 4;          // a key tile is split in 4 parts of 16 keys (one epilogue warp each)
constexpr int kIPartKeys = kIkN / kIParts;
constexpr int kICap = 2048;         // candidates per (row, part) list
constexpr int kIFallbackRows = 4096;
constexpr int kIRing = 24;          // FILTER: staged candidates per row (<= 7 pending + 16 new)
constexpr int kIFlush = 8;          //   written out 8 at a time (one 32-byte run per array)
constexpr int kIEpiWarps = 4 * kIParts;             // 4 TMEM lane quadrants x 4 parts
constexpr int kIThreads = 32 * (4 + kIEpiWarps);    // TMA, MMA, TMEM-alloc, spare + epilogue
constexpr uint64_t kIWaitNs = 2000000000ull;
constexpr uint32_t kISuspendNs = 128;    // pipeline waits: short suspends, prompt wake-up
constexpr float kIBeta = 1.25f;

struct IdxTcSmem {
    unsigned char q[kIH][kIqM * 128];        // per head: 128 rows x 64 dims, SW128
    unsigned char k[kIStages][kIkN * 128];   // key tiles: 64 keys x 64 dims, SW128
    float w[kIqM][kIH];
    uint32_t tau[kIqM];
    uint64_t ring[kIEpiWarps][kIRing][32];   // FILTER: (score bits << 32 | position) per lane (row)
    float stage[kIEpiWarps][kIPartKeys][32]; // FILTER: a tile's 16 scores per lane
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
    uint32_t *cand_key;       // [n, kIParts, kICap]
    int32_t *cand_idx;        // [n, kIParts, kICap]
    int32_t *cand_cnt;        // [n, kIParts]
    const uint32_t *keep;     // optional: [n, keep_words] kept 64-key blocks (one bit each);
    int keep_words;           //   a complete block without its bit is masked for that row
    int n, samp_slots, n_tiles_rows;
};

// One flush round of a FILTER epilogue warp: up to 4 rows (the lowest set bits
// of `rows`, lanes = rows of the warp's quadrant); lanes [8g, 8g + 8) write the
// next (at most 8) staged entries of the g-th row to its candidate list, as one
// 32-byte run per array.  Entries past the list capacity are dropped (the count
// still records them, so the row falls back).  Returns the rows served.
__device__ __forceinline__ unsigned flush_round(const IdxTcArgs &a, const uint64_t *ring,
                                                unsigned rows, int flushed, int cnt, int t_base,
                                                int part) {
    const int lane = threadIdx.x & 31, g = lane >> 3;
    int src[4];
    unsigned m = rows;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        src[u] = m ? __ffs(m) - 1 : -1;
        m &= m - 1u;
    }
    const int mine = g == 0 ? src[0] : g == 1 ? src[1] : g == 2 ? src[2] : src[3];
    const int sl = mine < 0 ? 0 : mine;
    const int f = __shfl_sync(0xffffffffu, flushed, sl);
    const int c = __shfl_sync(0xffffffffu, cnt, sl);
    const int e = f + (lane & 7);
    if (mine >= 0 && e < c && e < kICap) {
        const uint64_t v = ring[(e % kIRing) * 32 + mine];
        const size_t base = ((size_t)(t_base + mine) * kIParts + part) * kICap;
        a.cand_key[base + e] = score_key(__uint_as_float((uint32_t)(v >> 32)));
        a.cand_idx[base + e] = (int32_t)(uint32_t)v;
    }
    return rows & ~m;
}

// 0xffffffff if a >= b (false for NaN), else 0
__device__ __forceinline__ uint32_t set_ge_mask(float a, float b) {
    uint32_t r;
    asm("set.ge.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(a), "f"(b));
    return r;
}

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
    // CTAs start at different key tiles (and wrap), so they do not all read the same
    // tile of K at once; a row's candidate order does not matter to the selection
    const int t_off = ntiles > 0 ? (int)((blockIdx.x * 37u) % (unsigned)ntiles) : 0;

    if (tid == 0) {
        tc::mbar_init(&S.qfull, 1);
        for (int i = 0; i < kIStages; ++i) {
            tc::mbar_init(&S.kfull[i], 1);
            tc::mbar_init(&S.kempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&S.tfull[i], 1);
            tc::mbar_init(&S.tempty[i], kIEpiWarps);   // one arrival per epilogue warp
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
                    !tc::mbar_wait_bounded(&S.kempty[s], (u - 1) & 1, kIWaitNs, K_IDX_PREFILL_TC, 1, kISuspendNs)) {
                    atomicOr(&S.fail, 1);
                    break;
                }
                const int js = j + t_off < ntiles ? j + t_off : j + t_off - ntiles;
                const int kt = MODE == 0 ? js * kISampStride : js;
                tc::mbar_arrive_expect_tx(&S.kfull[s], kIkN * 128);
                tc::tma_load_2d(S.k[s], &tk, 0, kt * kIkN, &S.kfull[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16_f32(kIqM, kIkN, 0, 0);
            bool ok = tc::mbar_wait_bounded(&S.qfull, 0, kIWaitNs, K_IDX_PREFILL_TC, 2, kISuspendNs);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int s = j % kIStages, u = j / kIStages;
                const int b = j & 1, v = j >> 1;
                ok = tc::mbar_wait_bounded(&S.kfull[s], u & 1, kIWaitNs, K_IDX_PREFILL_TC, 3, kISuspendNs);
                if (ok && v > 0) ok = tc::mbar_wait_bounded(&S.tempty[b], (v - 1) & 1, kIWaitNs, K_IDX_PREFILL_TC, 4, kISuspendNs);
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
        // ---------------- epilogue: row = quadrant * 32 + lane, keys [16 part, 16 part + 16)
        const int ew = warp - 4, quad = warp & 3, part = ew >> 2;
        const int row = quad * 32 + lane;
        const int t = r0 + row;
        const bool row_ok = t < a.n;
        uint64_t w2[kIH];                        // (w_h, w_h) for the paired FMA
#pragma unroll
        for (int h = 0; h < kIH; ++h) w2[h] = f32x2_pack(S.w[row][h], S.w[row][h]);
        const uint32_t tau = MODE == 1 ? S.tau[row] : 0u;
        // key >= tau  <=>  score >= key_score(tau) for every non-NaN score
        const float tauf = tau == 0u ? -INFINITY : key_score(tau);
        int cnt = 0, flushed = 0, slot = 0;          // FILTER: appended, written out, ring slot
        uint64_t *ring = &S.ring[ew][0][0];
        const uint32_t tq_lane = tmem + ((uint32_t)(quad * 32) << 16) + part * kIPartKeys;
        uint64_t nanacc = 0ull;                  // score pairs x 0: stays 0 unless a score is NaN/inf
        float *stage = &S.stage[ew][0][0];
        for (int j = 0; j < ntiles; ++j) {
            const int b = j & 1, v = j >> 1;
            const bool ok = tc::mbar_wait_bounded(&S.tfull[b], v & 1, kIWaitNs, K_IDX_PREFILL_TC, 5, kISuspendNs);
            if (__any_sync(0xffffffffu, !ok)) {
                if (lane == 0) atomicOr(&S.fail, 1);
                break;
            }
            tc::fence_after();
            uint32_t d[kIH][kIPartKeys];
#pragma unroll
            for (int h = 0; h < kIH; ++h) tc::tmem_ld16(tq_lane + b * 256 + h * 64, d[h]);
            tc::tmem_ld_wait();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.tempty[b]);     // accumulators free for tile j + 2
            // score = sum_h w_h ReLU(q_h . k); a NaN dot survives the ReLU (max.NaN)
            uint64_t acc[kIPartKeys / 2];
#pragma unroll
            for (int i = 0; i < kIPartKeys / 2; ++i) acc[i] = 0ull;
#pragma unroll
            for (int h = 0; h < kIH; ++h)
#pragma unroll
                for (int i = 0; i < kIPartKeys / 2; ++i)
                    acc[i] = f32x2_fma(w2[h],
                                       f32x2_pack(relu_nan(__uint_as_float(d[h][2 * i])),
                                                  relu_nan(__uint_as_float(d[h][2 * i + 1]))),
                                       acc[i]);
            float sc[kIPartKeys];
#pragma unroll
            for (int i = 0; i < kIPartKeys / 2; ++i) {
                nanacc = f32x2_fma(acc[i], 0ull, nanacc);
                f32x2_unpack(acc[i], sc[2 * i], sc[2 * i + 1]);
            }
            const int js = j + t_off < ntiles ? j + t_off : j + t_off - ntiles;
            const int kt = MODE == 0 ? js * kISampStride : js;
            const int key0 = kt * kIkN + part * kIPartKeys;
            // keys > t (causal) exist only in the CTA's last two tiles
            const int lim = t - key0 + 1;            // keys [key0, key0 + lim) are visible
            uint32_t vis = lim >= kIPartKeys ? 0xffffu : (lim <= 0 ? 0u : ((1u << lim) - 1u));
            // hierarchical mode: a key tile is one 64-key block; a complete block the
            // row did not keep is not visible (the open block and later keys are)
            if (a.keep != nullptr && row_ok && kt < ((t + 1) >> 6) &&
                !((__ldg(a.keep + (size_t)t * a.keep_words + (kt >> 5)) >> (kt & 31)) & 1u))
                vis = 0u;
            if constexpr (MODE == 0) {
                if (row_ok) {
                    uint32_t pk[kIPartKeys / 2];
#pragma unroll
                    for (int i = 0; i < kIPartKeys / 2; ++i) {
                        const uint32_t lo = ((vis >> (2 * i)) & 1u) ? score_key(sc[2 * i]) >> 16 : 0u;
                        const uint32_t hi = ((vis >> (2 * i + 1)) & 1u) ? score_key(sc[2 * i + 1]) >> 16 : 0u;
                        pk[i] = lo | (hi << 16);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(a.samples + (size_t)t * a.samp_slots +
                                                           js * kIkN + part * kIPartKeys);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            } else {
                // pass mask: set.ge gives an all-ones word per passing key, one LOP3 merges it
                uint32_t pm = 0u;
#pragma unroll
                for (int i = 0; i < kIPartKeys; ++i) pm |= set_ge_mask(sc[i], tauf) & (1u << i);
                pm &= row_ok ? vis : 0u;
                if (__any_sync(0xffffffffu, pm != 0u)) {
                    // the scores go through shared memory so that the set bits can
                    // be visited with a dynamic index; each lane stages its row's
                    // passing (score, position) pairs in its ring
#pragma unroll
                    for (int i = 0; i < kIPartKeys; ++i) stage[i * 32 + lane] = sc[i];
                    while (pm) {
                        const int i = __ffs(pm) - 1;
                        pm &= pm - 1u;
                        ring[slot * 32 + lane] =
                            ((uint64_t)__float_as_uint(stage[i * 32 + lane]) << 32) | (uint32_t)(key0 + i);
                        slot = slot + 1 == kIRing ? 0 : slot + 1;
                        ++cnt;
                    }
                    __syncwarp();
                    // until every row has < 8 staged entries: 8 entries of up to 4
                    // rows per round, one 32-byte run per row and array
                    unsigned full;
                    while ((full = __ballot_sync(0xffffffffu, cnt - flushed >= kIFlush)) != 0u) {
                        const unsigned done = flush_round(a, ring, full, flushed, cnt, r0 + quad * 32, part);
                        if ((done >> lane) & 1u) flushed += kIFlush;
                    }
                }
            }
        }
        if (MODE == 1) {
            unsigned left;
            while ((left = __ballot_sync(0xffffffffu, cnt > flushed)) != 0u) {
                const unsigned done = flush_round(a, ring, left, flushed, cnt, r0 + quad * 32, part);
                if ((done >> lane) & 1u) flushed = min(cnt, flushed + kIFlush);
            }
        }
        if (MODE == 1 && row_ok) a.cand_cnt[(size_t)t * kIParts + part] = cnt;
        float n0, n1;
        f32x2_unpack(nanacc, n0, n1);
        if (row_ok && (n0 != 0.0f || n1 != 0.0f)) raise_error(CRS_DEVERR_NONFINITE);
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
                                                         int samp_slots, int topk, int top_blocks) {
    __shared__ int hist[8][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= n) return;
    int *hw = hist[warp];
    // the row's candidate keys: all t + 1, or (hierarchical) the kept blocks + the open block
    long long cand = t + 1;
    const int nbt = (t + 1) >> 6;
    if (top_blocks > 0 && nbt > top_blocks) cand = (long long)top_blocks * 64 + (t + 1 - nbt * 64);
    if (cand <= topk) {
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
    const long long R = ((long long)nvalid * topk * 5 + 4LL * cand - 1) / (4LL * cand);  // ceil(1.25 k nv/cand)
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
// Per row (one warp): exact top-k over the row's candidates, ascending output.
//   1. 4 radix passes of 8 bits over the candidate keys (warp histogram)
//      give the k-th largest key T and how many keys equal to T are taken;
//   2. positions with key > T are set in a bitmap over [0, t], positions with
//      key == T in a second one;
//   3. one ordered sweep over the bitmap words emits the positions ascending,
//      taking the tied positions smallest first.
// Rows whose lists overflowed, or hold fewer than k candidates, are queued
// for the exact slice path.
// ---------------------------------------------------------------------------
constexpr int kFinWarps = 8;

__host__ __device__ __forceinline__ size_t fin_warp_words(int n) { return 256 + 2 * (size_t)((n + 31) / 32); }

// Finds, from the top bin down, the bin holding the need-th largest count; need
// is then replaced by its rank inside that bin.  Warp-collective.
__device__ __forceinline__ int warp_top_bin(const uint32_t *hist, int &need) {
    const int lane = threadIdx.x & 31;
    int c[8], s = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) { c[u] = (int)hist[255 - (lane * 8 + u)]; s += c[u]; }
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
    need = __shfl_sync(0xffffffffu, fr, src);
    return __shfl_sync(0xffffffffu, fb, src);
}

__global__ void __launch_bounds__(kFinWarps * 32)
idx_tc_final_kernel(const uint32_t *__restrict__ cand_key, const int32_t *__restrict__ cand_idx,
                    const int32_t *__restrict__ cand_cnt, int32_t *__restrict__ out_idx,
                    int32_t *__restrict__ out_cnt, int32_t *__restrict__ fb_list,
                    int32_t *__restrict__ fb_count, int n, int topk) {
    extern __shared__ uint32_t fin_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= n) return;                                   // warp-uniform; no block barriers below
    uint32_t *hist = fin_smem + (size_t)warp * fin_warp_words(n);
    const int nwords = (t + 1 + 31) >> 5;                 // bitmap words over positions [0, t]
    uint32_t *bm_gt = hist + 256;
    uint32_t *bm_eq = bm_gt + (n + 31) / 32;
    int32_t *o = out_idx + (size_t)t * topk;
    if (t + 1 <= topk) {
        for (int i = lane; i < topk; i += 32) o[i] = (i <= t) ? i : -1;
        if (lane == 0) out_cnt[t] = t + 1;
        return;
    }
    int c[kIParts], N = 0;
    bool over = false;
#pragma unroll
    for (int q = 0; q < kIParts; ++q) {
        c[q] = cand_cnt[(size_t)t * kIParts + q];
        over |= c[q] > kICap;
        N += c[q];
    }
    if (over || N < topk) {
        if (lane == 0) {
            const int pos = atomicAdd(fb_count, 1);
            if (pos < kIFallbackRows) fb_list[pos] = t;
            else raise_error(CRS_DEVERR_INDEX);
        }
        return;
    }
    const uint32_t *ck = cand_key + (size_t)t * kIParts * kICap;
    const int32_t *ci = cand_idx + (size_t)t * kIParts * kICap;
    // 1. radix select
    uint32_t prefix = 0u, mask = 0u;
    int need = topk;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
#pragma unroll
        for (int u = 0; u < 8; ++u) hist[lane * 8 + u] = 0u;
        __syncwarp();
        // eight keys per lane in flight per step (the passes are bound by load latency)
#pragma unroll
        for (int q = 0; q < kIParts; ++q)
            for (int i0 = lane; i0 < c[q]; i0 += 8 * 32) {
                uint32_t kk[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + u * 32;
                    kk[u] = i < c[q] ? __ldg(ck + q * kICap + i) : 0u;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (i0 + u * 32 < c[q] && (kk[u] & mask) == prefix) atomicAdd(&hist[(kk[u] >> shift) & 255u], 1u);
            }
        __syncwarp();
        const int bin = warp_top_bin(hist, need);
        prefix |= (uint32_t)bin << shift;
        mask |= 0xffu << shift;
        __syncwarp();
    }
    const uint32_t T = prefix;                            // the k-th largest key; take `need` ties
    // 2. bitmaps
    for (int w = lane; w < nwords; w += 32) { bm_gt[w] = 0u; bm_eq[w] = 0u; }
    __syncwarp();
#pragma unroll
    for (int q = 0; q < kIParts; ++q)
        for (int i0 = lane; i0 < c[q]; i0 += 8 * 32) {
            uint32_t kk[8];
            int pos[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * 32;
                const bool in = i < c[q];
                kk[u] = in ? __ldg(ck + q * kICap + i) : 0u;
                pos[u] = in ? __ldg(ci + q * kICap + i) : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u * 32 < c[q] && kk[u] >= T)
                    atomicOr(kk[u] > T ? &bm_gt[pos[u] >> 5] : &bm_eq[pos[u] >> 5], 1u << (pos[u] & 31));
        }
    __syncwarp();
    // 3. ordered sweep: word w = round * 32 + lane
    int eq_base = 0, out_base = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
        const int w = w0 + lane;
        uint32_t g = 0u, e = 0u;
        if (w < nwords) { g = bm_gt[w]; e = bm_eq[w]; }
        const int pe = __popc(e);
        int incl = pe;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += x;
        }
        const int allow = need - (eq_base + incl - pe);   // ties this word may still take
        if (allow <= 0) e = 0u;
        else
            for (int r = pe - allow; r > 0; --r) e &= ~(0x80000000u >> __clz(e));   // keep the lowest `allow`
        const uint32_t sel = g | e;
        const int ps = __popc(sel);
        int oin = ps;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, oin, off);
            if (lane >= off) oin += x;
        }
        int dst = out_base + oin - ps;
        for (uint32_t m = sel; m; m &= m - 1u) o[dst++] = w * 32 + (__ffs(m) - 1);
        eq_base += __shfl_sync(0xffffffffu, incl, 31);
        out_base += __shfl_sync(0xffffffffu, oin, 31);
    }
    for (int i = out_base + lane; i < topk; i += 32) o[i] = -1;
    if (lane == 0) out_cnt[t] = out_base;
}

// ----------------------------------------------------------------- host --

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
    w.cand_key = reinterpret_cast<uint32_t *>(take((size_t)n * kIParts * kICap * 4));
    w.cand_idx = reinterpret_cast<int32_t *>(take((size_t)n * kIParts * kICap * 4));
    w.cand_cnt = reinterpret_cast<int32_t *>(take((size_t)n * kIParts * 4));
    w.fb_list = reinterpret_cast<int32_t *>(take((size_t)fbr * 4));
    w.fb_count = reinterpret_cast<int32_t *>(take(4));
    w.fb_ckey = reinterpret_cast<uint32_t *>(take((size_t)fbr * w.fb_slices * topk * 4));
    w.fb_cidx = reinterpret_cast<int32_t *>(take((size_t)fbr * w.fb_slices * topk * 4));
    w.fb_ccnt = reinterpret_cast<int32_t *>(take((size_t)fbr * w.fb_slices * 4));
    w.total = off;
}

static bool prefill_tc_applicable(const crs_indexer_params *p) {
    return p->mode == CRS_IDX_PREFILL && p->n_idx_heads == kIH && p->d_idx == kID &&
           p->topk <= 2048 && p->n_rows >= 1 && p->n_rows <= (1 << 19);
}

static size_t prefill_tc_workspace(const crs_indexer_params *p) {
    PrefillTcWs w;
    prefill_tc_layout(p->n_rows, p->topk, w, nullptr);
    return w.total;
}

static int launch_prefill_tc(const crs_indexer_params *p, const void *q_idx, const float *wgt,
                             const void *k_idx, int32_t *out_idx, int32_t *out_count, void *ws,
                             cudaStream_t s, const uint32_t *keep, int keep_words, int top_blocks) {
    const int n = p->n_rows, topk = p->topk;
    PFN_cuTensorMapEncodeTiled_v12000 enc = tc::tensor_map_encoder();
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
    a.keep = keep;
    a.keep_words = keep_words;
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
        idx_tc_tau_kernel<<<ceil_div(n, 8), 256, 0, s>>>(w.samples, w.tau, n, w.samp_slots, topk, top_blocks);
    }
    CRS_CHECK_LAUNCH();
    {
        ProfScope _ps(K_IDX_PREFILL_TC, s);
        idx_prefill_tc_kernel<1><<<a.n_tiles_rows, kIThreads, smem, s>>>(tq, tk, a);
    }
    CRS_CHECK_LAUNCH();
    const size_t per_warp = fin_warp_words(n) * 4;
    const int fin_warps = (int)min((size_t)kFinWarps, ((size_t)200 << 10) / per_warp);
    if (fin_warps < 1) return CRS_ERR_UNSUPPORTED;
    const int dsm = (int)(per_warp * fin_warps);
    CRS_TRY_CUDA(cudaFuncSetAttribute(idx_tc_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dsm));
    {
        ProfScope _ps(K_IDX_SELECT, s);
        idx_tc_final_kernel<<<ceil_div(n, fin_warps), fin_warps * 32, dsm, s>>>(
            w.cand_key, w.cand_idx, w.cand_cnt, out_idx, out_count, w.fb_list, w.fb_count, n, topk);
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
    f.keep = keep;
    f.keep_words = keep_words;
    const int fbr = min(n, kIFallbackRows);
    f.list_cap = fbr;
    const int fb_grid = min(fbr, 2 * 148);      // CTAs stride over the live list entries
    const size_t ssm = (size_t)kSlice * 4 + (kMaxIdxHeads * kIdxDim + kMaxIdxHeads) * 4;
    CRS_TRY_CUDA(cudaFuncSetAttribute(idx_slice_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm));
    {
        ProfScope _ps(K_IDX_SLICE, s);
        idx_slice_kernel<<<dim3(w.fb_slices, fb_grid), kSelThreads, ssm, s>>>(f);
    }
    CRS_CHECK_LAUNCH();
    if (w.fb_slices > 1) {
        ProfScope _ps(K_IDX_MERGE, s);
        idx_merge_kernel<<<fb_grid, kSelThreads, 0, s>>>(f, 0);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

}  // namespace crs
