// Block-mass selector (COBS-style): block descriptors and block selection, sm_100a.
//
// [P5] "COBS 阅读笔记": Eq.(11) (block mean, population covariance), Eq.(16)
// (rank-r factor xi_i = sqrt(lambda_i) u_i), Eq.(20) and Algorithm 2 (Gram
// route: eigen-decompose G = Kt Kt^T / L, xi_i = Kt^T w_i / sqrt(L)), Eq.(14)
// and (19) (second-order log-mass score), Eq.(15)/(6) (GQA group score = sum
// over the group of each head's softmax over blocks), "可缓存性约束" (the
// descriptor is computed once, when the block is full).
#include <math.h>

#include "common.cuh"
#include "tc.cuh"

namespace crs {

// ---------------------------------------------------------------------------
// K8: one warp per block.  Keys (bf16) are staged in shared memory; the mean
// and the Gram matrix are formed in fp32; the L x L symmetric eigenproblem is
// solved by the cyclic Jacobi method in the parallel "round-robin" ordering
// (Brent & Luk, 1985): each round applies L/2 disjoint plane rotations, one
// sweep is L-1 rounds, sweeps repeat until the off-diagonal mass is below
// 1e-12 of the total (at most 15 sweeps).  Lane k owns row/column k.
// ---------------------------------------------------------------------------
constexpr int kBdWarps = 4;
constexpr int kBdMaxL = 32;
constexpr int kBdD = 128;

struct BdWarpSmem {
    __nv_bfloat16 k[kBdMaxL][kBdD];
    float mu[kBdD];
    float g[kBdMaxL][kBdMaxL + 1];
    float v[kBdMaxL][kBdMaxL + 1];
    float rc[kBdMaxL], rs[kBdMaxL];
    int partner[kBdMaxL];
};
// subspace descriptors ([P5] Eq.(17)): the projected centred keys Y = Kt U (L x sd)
struct BdWarpSmemSS {
    float y[kBdMaxL][kBdD + 1];
};

// SS: the eigenvectors are those of U^T Sigma U, taken by the same Gram route on
// Y = Kt U (U [D, sd] staged once per CTA in shared memory, after the warps'
// areas); xi then has sd entries per vector.
template <bool SS>
__global__ void __launch_bounds__(kBdWarps * 32)
block_describe_kernel(const __nv_bfloat16 *__restrict__ K, float *__restrict__ mu_out,
                      float *__restrict__ xi_out, int n_kv, int T, int L, int rank, int blk_begin,
                      int n_blk, int n_full, const float *__restrict__ U, int sd) {
    extern __shared__ __align__(16) unsigned char bd_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    BdWarpSmem &S = reinterpret_cast<BdWarpSmem *>(bd_smem)[warp];
    BdWarpSmemSS *SY = reinterpret_cast<BdWarpSmemSS *>(bd_smem + kBdWarps * sizeof(BdWarpSmem));
    float *sU = reinterpret_cast<float *>(bd_smem + kBdWarps * (sizeof(BdWarpSmem) + sizeof(BdWarpSmemSS)));
    if constexpr (SS) {
        for (int e = threadIdx.x; e < kBdD * sd; e += kBdWarps * 32) sU[e] = U[e];
        __syncthreads();
    }
    const long long item = (long long)blockIdx.x * kBdWarps + warp;
    const int sh = blockIdx.y;                 // seq * n_kv + h
    if (item >= n_blk) return;
    const int blk = blk_begin + (int)item;
    const int seq = sh / n_kv, h = sh - seq * n_kv;
    const size_t tok0 = (size_t)seq * T + (size_t)blk * L;

    // stage the block's keys: L rows x 256 B
    for (int e = lane; e < L * 16; e += 32) {
        const int r = e >> 4, c = e & 15;
        const uint4 v = *reinterpret_cast<const uint4 *>(K + ((tok0 + r) * n_kv + h) * kBdD + c * 8);
        *reinterpret_cast<uint4 *>(&S.k[r][c * 8]) = v;
    }
    __syncwarp();
    const float invL = 1.0f / (float)L;
    for (int d = lane; d < kBdD; d += 32) {
        float acc = 0.0f;
        for (int r = 0; r < L; ++r) acc += __bfloat162float(S.k[r][d]);
        S.mu[d] = acc * invL;
    }
    __syncwarp();
    if constexpr (SS) {
        // Y[r][j] = sum_d Kt[r][d] U[d][j]; lane owns columns j = lane, lane + 32, ...
        for (int j = lane; j < sd; j += 32)
            for (int r = 0; r < L; ++r) {
                float acc = 0.0f;
                for (int d = 0; d < kBdD; ++d)
                    acc = fmaf(__bfloat162float(S.k[r][d]) - S.mu[d], sU[d * sd + j], acc);
                SY[warp].y[r][j] = acc;
            }
        __syncwarp();
    }
    // Gram row `lane`: G[i][j] = (1/L) sum_d Kt[i][d] Kt[j][d]  (SS: over Y's sd columns)
    if (lane < L) {
        float grow[kBdMaxL];
#pragma unroll
        for (int j = 0; j < kBdMaxL; ++j) grow[j] = 0.0f;
        if constexpr (SS) {
            for (int t = 0; t < sd; ++t) {
                const float yi = SY[warp].y[lane][t];
#pragma unroll
                for (int j = 0; j < kBdMaxL; ++j)
                    if (j < L) grow[j] = fmaf(yi, SY[warp].y[j][t], grow[j]);
            }
        } else {
            for (int d = 0; d < kBdD; ++d) {
                const float md = S.mu[d];
                const float ki = __bfloat162float(S.k[lane][d]) - md;
#pragma unroll
                for (int j = 0; j < kBdMaxL; ++j)
                    if (j < L) grow[j] = fmaf(ki, __bfloat162float(S.k[j][d]) - md, grow[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kBdMaxL; ++j)
            if (j < L) {
                S.g[lane][j] = grow[j] * invL;
                S.v[lane][j] = (lane == j) ? 1.0f : 0.0f;
            }
    }
    __syncwarp();

    // ---- parallel cyclic Jacobi
    const int nm1 = L - 1;                    // L even: players 0..L-1, player L-1 fixed
    for (int sweep = 0; sweep < 15; ++sweep) {
        float off = 0.0f, tot = 0.0f;
        if (lane < L)
            for (int j = 0; j < L; ++j) {
                const float x = S.g[lane][j];
                tot += x * x;
                if (j != lane) off += x * x;
            }
        off = warp_sum(off);
        tot = warp_sum(tot);
        if (off <= 1e-12f * tot || off == 0.0f) break;
        for (int t = 0; t < nm1; ++t) {
            if (lane < L) {
                int q;
                if (lane == nm1) {
                    // the p with 2p = t (mod L-1)
                    q = 0;
                    for (int p = 0; p < nm1; ++p)
                        if ((2 * p) % nm1 == t % nm1) q = p;
                } else {
                    q = ((t - lane) % nm1 + nm1) % nm1;
                    if (q == lane) q = nm1;
                }
                S.partner[lane] = q;
                if (lane < q) {
                    const float app = S.g[lane][lane], aqq = S.g[q][q], apq = S.g[lane][q];
                    float c = 1.0f, s = 0.0f;
                    if (apq != 0.0f && fabsf(apq) > 1e-30f * (fabsf(app) + fabsf(aqq))) {
                        const float theta = (aqq - app) / (2.0f * apq);
                        float tt;
                        if (fabsf(theta) > 1e18f)
                            tt = 0.5f / theta;
                        else
                            tt = copysignf(1.0f, theta) / (fabsf(theta) + sqrtf(theta * theta + 1.0f));
                        c = rsqrtf(tt * tt + 1.0f);
                        s = tt * c;
                    }
                    S.rc[lane] = c;
                    S.rs[lane] = s;
                }
            }
            __syncwarp();
            // columns: A <- A J, V <- V J (lane = row k)
            if (lane < L) {
                for (int p = 0; p < L; ++p) {
                    const int q = S.partner[p];
                    if (p < q) {
                        const float c = S.rc[p], s = S.rs[p];
                        const float akp = S.g[lane][p], akq = S.g[lane][q];
                        S.g[lane][p] = c * akp - s * akq;
                        S.g[lane][q] = s * akp + c * akq;
                        const float vkp = S.v[lane][p], vkq = S.v[lane][q];
                        S.v[lane][p] = c * vkp - s * vkq;
                        S.v[lane][q] = s * vkp + c * vkq;
                    }
                }
            }
            __syncwarp();
            // rows: A <- J^T A (lane = column k)
            if (lane < L) {
                for (int p = 0; p < L; ++p) {
                    const int q = S.partner[p];
                    if (p < q) {
                        const float c = S.rc[p], s = S.rs[p];
                        const float apk = S.g[p][lane], aqk = S.g[q][lane];
                        S.g[p][lane] = c * apk - s * aqk;
                        S.g[q][lane] = s * apk + c * aqk;
                    }
                }
            }
            __syncwarp();
        }
    }

    // ---- the `rank` largest eigenvalues (ties: lower index), xi = Kt^T w / sqrt(L)
    float lam = (lane < L) ? S.g[lane][lane] : -INFINITY;
    bool taken = false;
    const float rs_L = rsqrtf((float)L);
    const size_t dbase = ((size_t)sh * n_full + blk);
    for (int e = 0; e < rank; ++e) {
        float best = taken ? -INFINITY : lam;
        int bi = taken ? 0x7fffffff : lane;
        if (lane >= L) { best = -INFINITY; bi = 0x7fffffff; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
        }
        if (lane == bi) taken = true;
        const int xd = SS ? sd : kBdD;
        float *xo = xi_out + (dbase * rank + e) * xd;
        if (e >= L || bi >= L) {
            for (int d = lane; d < xd; d += 32) xo[d] = 0.0f;
            continue;
        }
        for (int d = lane; d < xd; d += 32) {
            float acc = 0.0f;
            if constexpr (SS) {
                for (int r = 0; r < L; ++r) acc = fmaf(SY[warp].y[r][d], S.v[r][bi], acc);
            } else {
                const float md = S.mu[d];
                for (int r = 0; r < L; ++r) acc = fmaf(__bfloat162float(S.k[r][d]) - md, S.v[r][bi], acc);
            }
            xo[d] = acc * rs_L;
        }
    }
    for (int d = lane; d < kBdD; d += 32) mu_out[dbase * kBdD + d] = S.mu[d];
}

// ---------------------------------------------------------------------------
// K9a: second-order scores s_{g,b}.  One thread per (block, query head) of a
// tile of blocks; descriptors and the scaled queries are staged in shared
// memory (rows padded by one float against bank conflicts).
// ---------------------------------------------------------------------------
constexpr int kBsThreads = 128;
constexpr int kBsMaxTile = 32;              // blocks per CTA at most (G = 1 would stage 128)
__host__ __device__ inline int bs_tile(int G) { return min(kBsThreads / G, kBsMaxTile); }

// xdim: entries per eigenvector (D, or the subspace size with qx != nullptr:
// the queries projected and scaled, [n_seq * n_q][xdim], [P5] Eq.(18)).
__global__ void __launch_bounds__(kBsThreads)
block_score_kernel(const __nv_bfloat16 *__restrict__ Q, const float *__restrict__ mu,
                   const float *__restrict__ xi, float *__restrict__ sc_out, int n_kv, int n_q,
                   int G, int rank, int n_full, float scale, int xdim, const float *__restrict__ qx) {
    extern __shared__ float bs_smem[];
    const int nbt = bs_tile(G);                 // blocks per CTA
    const int DP = kBdD + 1;
    float *sq = bs_smem;                        // [G][DP]
    float *sqx = sq + G * DP;                   // [G][DP] projected queries (subspace)
    float *sd = sqx + G * DP;                   // [nbt][(1+rank)][DP]
    const int sh = blockIdx.y, seq = sh / n_kv, h = sh - seq * n_kv;
    const int b0 = blockIdx.x * nbt;
    const int nb = min(nbt, n_full - b0);
    for (int e = threadIdx.x; e < G * kBdD; e += kBsThreads) {
        const int g = e / kBdD, d = e - g * kBdD;
        const size_t row = (size_t)seq * n_q + h * G + g;
        sq[g * DP + d] = scale * __bfloat162float(Q[row * kBdD + d]);
        if (qx && d < xdim) sqx[g * DP + d] = qx[row * xdim + d];
    }
    const int rows = 1 + rank;
    {   // every descriptor row of the tile in flight at once (4-byte async copies
        // into the padded rows); warp w copies rows w, w + 4, ...
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        for (int row = warp; row < nb * rows; row += kBsThreads / 32) {
            const int bl = row / rows, rr = row - bl * rows;
            const size_t blk = (size_t)sh * n_full + b0 + bl;
            const float *src = rr == 0 ? mu + blk * kBdD : xi + (blk * rank + (rr - 1)) * xdim;
            const int len = rr == 0 ? kBdD : xdim;
            for (int d = lane; d < len; d += 32) cp_async4(&sd[row * DP + d], src + d);
        }
        cp_async_commit();
        cp_async_wait<0>();
    }
    __syncthreads();
    const int bl = threadIdx.x / G, g = threadIdx.x - bl * G;
    if (bl >= nb) return;
    const float *q = sq + g * DP;
    const float *qq = qx ? sqx + g * DP : q;
    const float *dsc = sd + bl * rows * DP;
    float lin = 0.0f;
    for (int d = 0; d < kBdD; ++d) lin = fmaf(q[d], dsc[d], lin);
    float quad = 0.0f;
    for (int e = 0; e < rank; ++e) {
        float p = 0.0f;
        const float *x = dsc + (1 + e) * DP;
        for (int d = 0; d < xdim; ++d) p = fmaf(qq[d], x[d], p);
        quad = fmaf(p, p, quad);
    }
    sc_out[((size_t)sh * G + g) * n_full + b0 + bl] = fmaf(0.5f, quad, lin);
}

// Copies n floats global -> shared with 16-byte loads when both are 16-byte aligned
// (every load of a thread is issued before the stores that use it).
__device__ __forceinline__ void stage_floats(float *dst, const float *__restrict__ src, int n) {
    if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0) {
        const int n4 = n >> 2;
        const float4 *s4 = reinterpret_cast<const float4 *>(src);
        float4 *d4 = reinterpret_cast<float4 *>(dst);
        for (int e0 = threadIdx.x; e0 < n4; e0 += 4 * blockDim.x) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * blockDim.x;
                v[u] = e < n4 ? __ldg(s4 + e) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * blockDim.x;
                if (e < n4) d4[e] = v[u];
            }
        }
        for (int e = (n4 << 2) + threadIdx.x; e < n; e += blockDim.x) dst[e] = __ldg(src + e);
    } else {
        for (int e = threadIdx.x; e < n; e += blockDim.x) dst[e] = __ldg(src + e);
    }
}

// qx[row][j] = sum_d U[d][j] scale q[row][d].
__global__ void __launch_bounds__(256)
query_project_kernel(const __nv_bfloat16 *__restrict__ Q, const float *__restrict__ U,
                     float *__restrict__ qx, int n_rows, int sd, float scale) {
    // 16 query rows per CTA; U (D x sd) and the rows staged in shared memory, then
    // thread (row, j) forms qx[row][j] = sum_d U[d][j] scale q[d] as one FMA chain in d order
    extern __shared__ float qp_smem[];
    float *Us = qp_smem;                         // [D][sd]
    float *qs = Us + (size_t)kBdD * sd;          // [16][D]
    const int r0 = blockIdx.x * 16;
    stage_floats(Us, U, kBdD * sd);
    for (int e = threadIdx.x; e < 16 * kBdD; e += blockDim.x) {
        const int r = e / kBdD, dd = e - r * kBdD;
        qs[e] = r0 + r < n_rows ? scale * __bfloat162float(Q[(size_t)(r0 + r) * kBdD + dd]) : 0.0f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * sd; e += blockDim.x) {
        const int r = e / sd, j = e - r * sd;
        if (r0 + r >= n_rows) continue;
        float acc = 0.0f;
#pragma unroll 8
        for (int dd = 0; dd < kBdD; ++dd) acc = fmaf(Us[dd * sd + j], qs[r * kBdD + dd], acc);
        qx[(size_t)(r0 + r) * sd + j] = acc;
    }
}

// K9a specialised for G query heads and rank R, streaming the descriptors
// through shared memory.  The work is the list of chunks of 16 blocks of every
// (sequence, KV head) (mu 8 KB + xi 32 KB, contiguous in HBM; the last chunk of
// a (sequence, KV head) may be short); a CTA owns a contiguous range of that list
// (two CTAs per SM, equal ranges, so no partial last wave), reloading its scaled
// queries when the range crosses into the next (sequence, KV head).  Chunks
// arrive by two bulk copies each into a 2-stage ring, so one chunk is in flight
// while the previous is scored.  Eight lanes share a block: lane s reads
// 16-byte chunks s, s + 8, s + 16, s + 24 of each 512-byte row (a group's
// reads are 128 contiguous bytes: no bank conflicts), forms its G x (1 + R)
// partial dot products with the scaled queries (read the same way), and the
// group sums them with three shuffle steps.
constexpr int kBsChunk = 16;                        // blocks per chunk
constexpr int kBsThreadsT = 8 * kBsChunk;          // 8 lanes per block
constexpr int kBsStages = 2;
constexpr uint64_t kBsWaitNs = 1000000000ull;

template <int G, int R>
struct BsSmem {
    float mu[kBsStages][kBsChunk][kBdD];
    float xi[kBsStages][kBsChunk][R][kBdD];
    float sq[G][kBdD];
    uint64_t full[kBsStages];
};

template <int G, int R>
__global__ void __launch_bounds__(kBsThreadsT, 2)
block_score_tma_kernel(const __nv_bfloat16 *__restrict__ Q, const float *__restrict__ mu,
                       const float *__restrict__ xi, float *__restrict__ sc_out, int n_kv, int n_q,
                       int n_full, int total_chunks, int chunks_per_cta, float scale) {
    extern __shared__ __align__(128) unsigned char bs_raw[];
    BsSmem<G, R> &S = *reinterpret_cast<BsSmem<G, R> *>(bs_raw);
    const int cps = ceil_div(n_full, kBsChunk);    // chunks per (sequence, KV head)
    const int c_lo = blockIdx.x * chunks_per_cta;
    const int n_chunks = min(total_chunks, c_lo + chunks_per_cta) - c_lo;
    if (n_chunks <= 0) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto issue = [&](int c) {                      // one thread
        const int st = c % kBsStages;
        const int gc = c_lo + c, sh = gc / cps, b0 = (gc - sh * cps) * kBsChunk;
        const int nb = min(kBsChunk, n_full - b0);
        const uint32_t mb = (uint32_t)nb * kBdD * 4, xb = mb * R;
        tc::mbar_arrive_expect_tx(&S.full[st], mb + xb);
        tc::bulk_load(&S.mu[st][0][0], mu + ((size_t)sh * n_full + b0) * kBdD, mb, &S.full[st]);
        tc::bulk_load(&S.xi[st][0][0][0], xi + ((size_t)sh * n_full + b0) * R * kBdD, xb, &S.full[st]);
    };
    if (tid == 0) {
        for (int st = 0; st < kBsStages; ++st) tc::mbar_init(&S.full[st], 1);
        tc::mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0)
        for (int c = 0; c < min(kBsStages, n_chunks); ++c) issue(c);
    const int sub = lane & 7, grp = warp * 4 + (lane >> 3);     // block of the chunk
    const float4 *q4 = reinterpret_cast<const float4 *>(&S.sq[0][0]);
    bool ok = true;
    int cur_sh = -1;
    for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kBsStages;
        const int gc = c_lo + c, sh = gc / cps, b_hi = n_full;
        const int b = (gc - sh * cps) * kBsChunk + grp;
        if (sh != cur_sh) {                        // uniform: the scaled queries of this (sequence, KV head)
            __syncthreads();                       // the previous ones are no longer read
            const int seq = sh / n_kv, h = sh - seq * n_kv;
            for (int e = tid; e < G * kBdD; e += blockDim.x) {
                const int g = e / kBdD, d = e - g * kBdD;
                S.sq[g][d] = scale * __bfloat162float(Q[((size_t)seq * n_q + h * G + g) * kBdD + d]);
            }
            cur_sh = sh;
        }
        ok = ok && tc::mbar_wait_bounded(&S.full[st], (c / kBsStages) & 1, kBsWaitNs, K_BLK_SCORE, 1);
        if (__syncthreads_or(!ok)) break;
        {   // every lane computes (the group shuffles need all 32); invalid blocks only skip the store
            const float4 *m4 = reinterpret_cast<const float4 *>(&S.mu[st][grp][0]);
            const float4 *x4 = reinterpret_cast<const float4 *>(&S.xi[st][grp][0][0]);
            float lin[G], pr[G][R];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                lin[g] = 0.0f;
#pragma unroll
                for (int e = 0; e < R; ++e) pr[g][e] = 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int f = u * 8 + sub;                 // 16-byte chunk of the row
                const float4 mv = m4[f];
                float4 xv[R];
#pragma unroll
                for (int e = 0; e < R; ++e) xv[e] = x4[e * (kBdD / 4) + f];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 qv = q4[g * (kBdD / 4) + f];
                    lin[g] = fmaf(qv.x, mv.x, lin[g]);
                    lin[g] = fmaf(qv.y, mv.y, lin[g]);
                    lin[g] = fmaf(qv.z, mv.z, lin[g]);
                    lin[g] = fmaf(qv.w, mv.w, lin[g]);
#pragma unroll
                    for (int e = 0; e < R; ++e) {
                        pr[g][e] = fmaf(qv.x, xv[e].x, pr[g][e]);
                        pr[g][e] = fmaf(qv.y, xv[e].y, pr[g][e]);
                        pr[g][e] = fmaf(qv.z, xv[e].z, pr[g][e]);
                        pr[g][e] = fmaf(qv.w, xv[e].w, pr[g][e]);
                    }
                }
            }
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    lin[g] += __shfl_xor_sync(0xffffffffu, lin[g], off);
#pragma unroll
                    for (int e = 0; e < R; ++e) pr[g][e] += __shfl_xor_sync(0xffffffffu, pr[g][e], off);
                }
            }
            if (sub == 0 && b < b_hi) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float quad = 0.0f;
#pragma unroll
                    for (int e = 0; e < R; ++e) quad = fmaf(pr[g][e], pr[g][e], quad);
                    sc_out[((size_t)sh * G + g) * n_full + b] = fmaf(0.5f, quad, lin[g]);
                }
            }
        }
        __syncthreads();                                  // stage st is read: refill it
        if (tid == 0 && c + kBsStages < n_chunks) issue(c + kBsStages);
    }
}

// ---------------------------------------------------------------------------
// K9b: group softmax sum, top blocks, token list.  One CTA per (seq, KV head).
// ---------------------------------------------------------------------------
constexpr int kPickT = 1024;

__host__ __device__ inline size_t pick_smem_bytes(int G, int n_full, int top) {
    return (size_t)G * n_full * 4 + (size_t)top * 8;
}

// Exclusive prefix sums over the CTA of two per-thread counts (thread order).
__device__ __forceinline__ void cta_exscan2(int a, int b, int &ea, int &eb, int &ta, int &tb, int2 *wtot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int xa = __shfl_up_sync(0xffffffffu, ia, o), xb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
            ia += xa;
            ib += xb;
        }
    }
    if (lane == 31) wtot[warp] = make_int2(ia, ib);
    __syncthreads();
    if (warp == 0) {
        int2 v = lane < kPickT / 32 ? wtot[lane] : make_int2(0, 0);
        int sa = v.x, sb = v.y;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int xa = __shfl_up_sync(0xffffffffu, sa, o), xb = __shfl_up_sync(0xffffffffu, sb, o);
            if (lane >= o) {
                sa += xa;
                sb += xb;
            }
        }
        if (lane < kPickT / 32) wtot[lane] = make_int2(sa - v.x, sb - v.y);   // exclusive per warp
        if (lane == 31) wtot[kPickT / 32] = make_int2(sa, sb);                 // totals
    }
    __syncthreads();
    const int2 base = wtot[warp], tot = wtot[kPickT / 32];
    ea = base.x + ia - a;
    eb = base.y + ib - b;
    ta = tot.x;
    tb = tot.y;
    __syncthreads();                                    // wtot is reused by the next scan
}

// One CTA per (sequence, KV head), thread t owning blocks [t KPT, t KPT + KPT).
// The 32 / G warps of query head g form its softmax over blocks (max and sum
// by shuffles, combined across the warps in a fixed order; exponentials kept
// in shared memory); the group sum of the heads' probabilities is formed per
// block in head order.  The k-th largest block key is built bit by bit from
// the top (32 CTA-wide counts), ties at it go to the smaller blocks, and the
// kept blocks are listed in block order by CTA-wide prefix sums.
template <int KPT>
__global__ void __launch_bounds__(kPickT)
block_pick_kernel(const float *__restrict__ sc, int32_t *__restrict__ tok, int32_t *__restrict__ cnt,
                  int G, int n_full, int L, int T, int top, int window, int cap) {
    extern __shared__ __align__(16) unsigned char bp_smem[];
    float *ex = reinterpret_cast<float *>(bp_smem);                       // [G][n_full]
    int *sel = reinterpret_cast<int *>(ex + (size_t)G * n_full);         // [top] kept blocks
    int *tstart = sel + top;                                              // [top] output offsets
    __shared__ float iz[16];
    __shared__ float part_red[kPickT / 32];
    __shared__ int2 wtot[kPickT / 32 + 1];
    const int sh = blockIdx.x, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    {   // G divides 16, so the 32 warps split evenly over the heads
        const int wph = (kPickT / 32) / G, g = warp / wph, part = warp - g * wph;
        const float *s = sc + ((size_t)sh * G + g) * n_full;
        float *e = ex + (size_t)g * n_full;
        float m = -INFINITY;
        for (int b0 = part * 32; b0 < n_full; b0 += 8 * wph * 32) {    // 8 loads in flight per lane
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int b = b0 + u * wph * 32 + lane;
                v[u] = b < n_full ? s[b] : -INFINITY;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int b = b0 + u * wph * 32 + lane;
                if (b < n_full) e[b] = v[u];
                m = fmaxf(m, v[u]);
            }
        }
        m = warp_max(m);
        if (lane == 0) part_red[warp] = m;
        __syncthreads();
        m = -INFINITY;
        for (int q = 0; q < wph; ++q) m = fmaxf(m, part_red[g * wph + q]);
        __syncthreads();
        float z = 0.0f;
        for (int b = part * 32 + lane; b < n_full; b += wph * 32) {
            const float x = __expf(e[b] - m);
            e[b] = x;
            z += x;
        }
        z = warp_sum(z);
        if (lane == 0) part_red[warp] = z;
        __syncthreads();
        if (part == 0 && lane == 0) {
            float zt = 0.0f;
            for (int q = 0; q < wph; ++q) zt += part_red[g * wph + q];
            iz[g] = 1.0f / zt;
        }
    }
    __syncthreads();
    const int bt0 = tid * KPT;
    uint32_t key[KPT];
    bool valid[KPT];
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        const int b = bt0 + u;
        valid[u] = b < n_full;
        key[u] = 0u;
        if (valid[u]) {
            float acc = 0.0f;
            for (int g = 0; g < G; ++g) acc += __fmul_rn(ex[(size_t)g * n_full + b], iz[g]);
            key[u] = score_key(acc);
        }
    }
    int ph = 0;
    auto count_ge = [&](uint32_t c) -> int {
        int local = 0;
#pragma unroll
        for (int u = 0; u < KPT; ++u) local += (valid[u] && key[u] >= c) ? 1 : 0;
        if (KPT == 1) return __syncthreads_count(local);       // one barrier already
        return cta_count(local, ph);
    };
    // exact top k by (key desc, block asc): Tk = the largest key with >= k keys at or above it
    const int k = min(top, n_full);
    uint32_t Tk = 0u;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t c = Tk | (1u << bit);
        if (count_ge(c) >= k) Tk = c;
    }
    const int need = k - (Tk == 0xffffffffu ? 0 : count_ge(Tk + 1u));   // ties at Tk to keep
    int n_eq = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) n_eq += (valid[u] && key[u] == Tk) ? 1 : 0;
    int eq_before, dummy, t0, t1;
    cta_exscan2(n_eq, 0, eq_before, dummy, t0, t1, wtot);
    const int wstart = max(0, T - window);
    bool take[KPT];
    int n_take = 0, n_tok = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        const int b = bt0 + u;
        const bool eq = valid[u] && key[u] == Tk;
        take[u] = (valid[u] && key[u] > Tk) || (eq && eq_before < need);
        eq_before += eq ? 1 : 0;
        n_take += take[u] ? 1 : 0;
        n_tok += take[u] ? min(L, max(0, wstart - b * L)) : 0;   // tokens of b before the window
    }
    int slot, tpos, n_sel, nblk_tok;
    cta_exscan2(n_take, n_tok, slot, tpos, n_sel, nblk_tok, wtot);
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        if (!take[u]) continue;
        const int b = bt0 + u;
        sel[slot] = b;
        tstart[slot] = tpos;
        ++slot;
        tpos += min(L, max(0, wstart - b * L));
    }
    __syncthreads();
    // token list: kept blocks' positions before the window (blocks ascending),
    // then the window [wstart, T)
    int32_t *to = tok + (size_t)sh * cap;
    for (int e = tid; e < n_sel * L; e += kPickT) {
        const int i = e / L, r = e - i * L;
        const int b = sel[i];
        if (b * L + r < wstart) to[tstart[i] + r] = b * L + r;
    }
    const int nwin = T - wstart;
    for (int i = tid; i < nwin; i += kPickT) to[nblk_tok + i] = wstart + i;
    const int total = nblk_tok + nwin;
    for (int i = total + tid; i < cap; i += kPickT) to[i] = -1;
    if (tid == 0) cnt[sh] = total;
}

// Host: the instantiation for n_full blocks (KPT = blocks per thread).
template <typename... A>
static void launch_pick(int n_full, int grid, size_t smem, cudaStream_t s, A... args) {
    if (n_full <= kPickT) block_pick_kernel<1><<<grid, kPickT, smem, s>>>(args...);
    else if (n_full <= 2 * kPickT) block_pick_kernel<2><<<grid, kPickT, smem, s>>>(args...);
    else if (n_full <= 4 * kPickT) block_pick_kernel<4><<<grid, kPickT, smem, s>>>(args...);
    else block_pick_kernel<8><<<grid, kPickT, smem, s>>>(args...);
}
static cudaError_t pick_prepare(int n_full, size_t smem) {
    const void *f = n_full <= kPickT ? (const void *)block_pick_kernel<1>
                    : n_full <= 2 * kPickT ? (const void *)block_pick_kernel<2>
                    : n_full <= 4 * kPickT ? (const void *)block_pick_kernel<4>
                                           : (const void *)block_pick_kernel<8>;
    return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

// ---------------------------------------------------------------------------
// First-order and box selectors ([P5] Table 1): per-block summaries that are
// scored without a quadratic term.
//   Quest ([P5] Eq.(23)-(24)): kmin, kmax = element-wise key minimum and
//     maximum of the block (bf16, exact: they are key values); score
//     sum_t max(q_t kmin_t, q_t kmax_t) = sum_t q_t (q_t > 0 ? kmax_t : kmin_t).
//   Mean-pool: the block mean (fp32), score q . mu (crs_block_select, rank 0).
// ---------------------------------------------------------------------------
constexpr int kQdWarps = 8;

// One warp per block: lane l takes dims [4l, 4l + 4) of each of the L keys.
__global__ void __launch_bounds__(kQdWarps * 32)
quest_describe_kernel(const __nv_bfloat16 *__restrict__ K, __nv_bfloat16 *__restrict__ kmin,
                      __nv_bfloat16 *__restrict__ kmax, int T, int n_kv, int L, int n_full, int blk_begin,
                      int n_blk) {
    const int sh = blockIdx.y, seq = sh / n_kv, h = sh - seq * n_kv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * kQdWarps + warp;
    if (i >= n_blk) return;
    const int blk = blk_begin + i;
    float lo[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
    float hi[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    const __nv_bfloat16 *k0 = K + (((size_t)seq * T + (size_t)blk * L) * n_kv + h) * kBdD + 4 * lane;
    const size_t row = (size_t)n_kv * kBdD;
#pragma unroll 8
    for (int r = 0; r < L; ++r) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(k0 + r * row));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
        const float v[4] = {a.x, a.y, b.x, b.y};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            lo[t] = fminf(lo[t], v[t]);
            hi[t] = fmaxf(hi[t], v[t]);
        }
    }
    const size_t o = ((size_t)sh * n_full + blk) * kBdD + 4 * lane;
    __nv_bfloat162 l0 = __floats2bfloat162_rn(lo[0], lo[1]), l1 = __floats2bfloat162_rn(lo[2], lo[3]);
    __nv_bfloat162 h0 = __floats2bfloat162_rn(hi[0], hi[1]), h1 = __floats2bfloat162_rn(hi[2], hi[3]);
    *reinterpret_cast<uint2 *>(kmin + o) = make_uint2(*reinterpret_cast<uint32_t *>(&l0), *reinterpret_cast<uint32_t *>(&l1));
    *reinterpret_cast<uint2 *>(kmax + o) = make_uint2(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1));
}

// K9a for these selectors.  One warp scores 32 / G blocks at a time: lane l
// holds dims [4l, 4l + 4) of the G scaled queries (registers) and of each
// block's summary, forms the 32 partial sums (block j, head g) -> index
// j G + g, and a five-step butterfly reduce-scatter leaves lane v with the
// total of index v.
constexpr int kWsWarps = 8;
constexpr int kWsGroups = 2;              // block groups per warp
enum { kWsQuest = 0, kWsMean = 1 };

template <int G, int MODE>
__global__ void __launch_bounds__(kWsWarps * 32)
block_score_warp_kernel(const __nv_bfloat16 *__restrict__ Q, const void *__restrict__ A,
                        const void *__restrict__ B, float *__restrict__ sc_out, int n_kv, int n_q,
                        int n_full, float scale) {
    constexpr int BPW = 32 / G;
    const int sh = blockIdx.y, seq = sh / n_kv, h = sh - seq * n_kv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float q[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(Q + ((size_t)seq * n_q + h * G + g) * kBdD + 4 * lane));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
        q[g][0] = scale * a.x;
        q[g][1] = scale * a.y;
        q[g][2] = scale * b.x;
        q[g][3] = scale * b.y;
    }
    const int n_groups = ceil_div(n_full, BPW);
    const int grp0 = (blockIdx.x * kWsWarps + warp) * kWsGroups;
    for (int gi = 0; gi < kWsGroups; ++gi) {
        const int b0 = (grp0 + gi) * BPW;
        if (grp0 + gi >= n_groups) break;                 // warp-uniform
        float v[32];
#pragma unroll
        for (int j = 0; j < BPW; ++j) {
            const int b = b0 + j;
            const size_t o = ((size_t)sh * n_full + b) * kBdD + 4 * lane;
            float lo[4] = {0.0f, 0.0f, 0.0f, 0.0f}, hi[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            if (b < n_full) {
                if constexpr (MODE == kWsQuest) {
                    const uint2 rl = __ldcs(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(A) + o));
                    const uint2 rh = __ldcs(reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(B) + o));
                    const float2 l0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&rl.x));
                    const float2 l1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&rl.y));
                    const float2 h0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&rh.x));
                    const float2 h1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&rh.y));
                    lo[0] = l0.x; lo[1] = l0.y; lo[2] = l1.x; lo[3] = l1.y;
                    hi[0] = h0.x; hi[1] = h0.y; hi[2] = h1.x; hi[3] = h1.y;
                } else {
                    const float4 m = __ldcs(reinterpret_cast<const float4 *>(static_cast<const float *>(A) + o));
                    lo[0] = m.x; lo[1] = m.y; lo[2] = m.z; lo[3] = m.w;
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float acc = 0.0f;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if constexpr (MODE == kWsQuest) acc = fmaf(q[g][t], q[g][t] > 0.0f ? hi[t] : lo[t], acc);
                    else acc = fmaf(q[g][t], lo[t], acc);
                }
                v[j * G + g] = acc;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < o; ++i) {
                const float send = up ? v[i] : v[i + o];
                const float keep = up ? v[i + o] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        const int j = lane / G, g = lane - j * G, b = b0 + j;
        if (b < n_full) sc_out[((size_t)sh * G + g) * n_full + b] = v[0];
    }
}

template <int MODE>
static cudaError_t launch_score_warp(int G, dim3 grid, cudaStream_t s, const void *Q, const void *A,
                                     const void *B, float *sc, int n_kv, int n_q, int n_full, float scale) {
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(Q);
    switch (G) {
    case 1: block_score_warp_kernel<1, MODE><<<grid, kWsWarps * 32, 0, s>>>(q, A, B, sc, n_kv, n_q, n_full, scale); break;
    case 2: block_score_warp_kernel<2, MODE><<<grid, kWsWarps * 32, 0, s>>>(q, A, B, sc, n_kv, n_q, n_full, scale); break;
    case 4: block_score_warp_kernel<4, MODE><<<grid, kWsWarps * 32, 0, s>>>(q, A, B, sc, n_kv, n_q, n_full, scale); break;
    case 8: block_score_warp_kernel<8, MODE><<<grid, kWsWarps * 32, 0, s>>>(q, A, B, sc, n_kv, n_q, n_full, scale); break;
    case 16: block_score_warp_kernel<16, MODE><<<grid, kWsWarps * 32, 0, s>>>(q, A, B, sc, n_kv, n_q, n_full, scale); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

static dim3 score_warp_grid(int G, int n_full, int n_sh) {
    const int n_groups = ceil_div(n_full, 32 / G);
    return dim3(ceil_div(n_groups, kWsWarps * kWsGroups), n_sh);
}

// ---------------------------------------------------------------------------
// Deployed descriptor compression ([P5] §5.5): the block mean in bf16 and each
// scaled eigenvector in E2M1 FP4 with one fp32 scale (absmax / 6).  One warp
// per vector, four elements per lane; codes: bit 3 sign, bits 0-2 index into
// {0, 0.5, 1, 1.5, 2, 3, 4, 6}, nearest value, ties to the zero-mantissa code
// (decided in fp32 on the quotient x / scale).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e2m1_code(float x, float s) {
    if (!(s > 0.0f)) return 0u;
    const float y = x / s;
    const float a = fabsf(y);
    const uint32_t idx = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                         (a >= 3.5f) + (a > 5.0f);
    return ((y < 0.0f && idx != 0u) ? 8u : 0u) | idx;
}

// grid (vectors / 8, 1): warps 0..7 take vectors; vector v < n_mu is a mean
// (bf16), the rest are scaled eigenvectors (FP4 + scale)
__global__ void __launch_bounds__(256) block_quantize_kernel(const float *__restrict__ mu,
                                                             const float *__restrict__ xi,
                                                             __nv_bfloat16 *__restrict__ mu16,
                                                             uint8_t *__restrict__ xi4,
                                                             float *__restrict__ xi_scale,
                                                             long long n_mu, long long n_xi) {
    const long long v = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (v < n_mu) {
        const float4 x = reinterpret_cast<const float4 *>(mu + v * kBdD)[lane];
        __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t *>(&a);
        o.y = *reinterpret_cast<uint32_t *>(&b);
        reinterpret_cast<uint2 *>(mu16 + v * kBdD)[lane] = o;
        return;
    }
    const long long w = v - n_mu;
    if (w >= n_xi) return;
    const float4 x = reinterpret_cast<const float4 *>(xi + w * kBdD)[lane];
    const float amax = warp_max(fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
    const float sc = amax / 6.0f;
    const uint32_t c = e2m1_code(x.x, sc) | (e2m1_code(x.y, sc) << 4) | (e2m1_code(x.z, sc) << 8) |
                       (e2m1_code(x.w, sc) << 12);
    reinterpret_cast<uint16_t *>(xi4 + w * (kBdD / 2))[lane] = (uint16_t)c;
    if (lane == 0) xi_scale[w] = sc;
}

// bf16 bit patterns of the eight E2M1 magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6},
// split into high and low bytes so that one byte permute looks up four codes.
constexpr uint32_t kE2m1HiLo = 0x3F3F3F00u, kE2m1HiHi = 0x40404040u;
constexpr uint32_t kE2m1LoLo = 0xC0800000u, kE2m1LoHi = 0xC0804000u;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Eight E2M1 codes (element j in bits [4j, 4j+4): magnitude index in the low
// three bits, sign in the fourth) -> eight bf16, two per word, element 2k in
// the low half of word k.  Every E2M1 value is exact in bf16.  The high and
// low bytes of each magnitude come from the byte tables above (one permute
// looks up four codes); a code's sign is the top bit of its byte in w (odd
// elements) or in w << 4 (even elements), replicated by the permute's sign
// mode into the high byte before the two bytes are interleaved.
__device__ __forceinline__ uint4 e2m1x8_to_bf16(uint32_t w) {
    const uint32_t m = w & 0x77777777u, mh = m >> 16, w4 = w << 4;
    const uint32_t hiA = prmt(kE2m1HiLo, kE2m1HiHi, m) | (prmt(w4, w, 0xD9C8u) & 0x80808080u);
    const uint32_t hiB = prmt(kE2m1HiLo, kE2m1HiHi, mh) | (prmt(w4, w, 0xFBEAu) & 0x80808080u);
    const uint32_t loA = prmt(kE2m1LoLo, kE2m1LoHi, m), loB = prmt(kE2m1LoLo, kE2m1LoHi, mh);
    uint4 o;
    o.x = prmt(loA, hiA, 0x5140u);
    o.y = prmt(loA, hiA, 0x7362u);
    o.z = prmt(loB, hiB, 0x5140u);
    o.w = prmt(loB, hiB, 0x7362u);
    return o;
}

// K9a on compressed descriptors, on the tensor cores.  A tile is 128
// consecutive blocks of one (sequence, KV head); per tile the CTA forms
//   lin_g   = Q_g . mu_b                  (A = the bf16 means, TMA, 128B swizzle)
//   p_{e,g} = Q_g . code(xi_{b,e})        (A = the codes widened to bf16)
// as M=128 (blocks) x N=16 (query heads, zero-padded) x K=128 products with
// fp32 accumulators in TMEM; Q is the raw bf16 query (every product of two
// bf16 is exact in fp32, so nothing is split), and the softmax scale and the
// per-vector FP4 scale are applied in the epilogue:
//   score_g = s lin_g + 1/2 sum_e (s sigma_e p_{e,g})^2.
// Warp roles: 0 loads the mean tile and query rows (TMA, two stages); 1
// owns TMEM and issues the MMAs; 4..7 read the accumulators (warp % 4 = lane
// quadrant = 32 blocks); 8..15 read the codes of the next tile into registers while widening the
// current one, one eigenvector at a time, into a four-buffer ring of bf16
// operand tiles.  Persistent: each CTA walks a contiguous range of tiles.
constexpr int kFtM = 128;                     // blocks per tile
constexpr int kFtN = 16;                      // query-head columns (G <= 16)
constexpr int kFtMaxR = 4;
constexpr int kFtStages = 2;                  // mean + query tiles
constexpr int kFtDecBufs = 4;                 // widened eigenvector tiles
constexpr int kFtDecWarps = 8;
constexpr int kFtThreads = 32 * (8 + kFtDecWarps);
constexpr uint32_t kFtSuspendNs = 256;

struct FtSmem {
    unsigned char mu[kFtStages][2][kFtM * 128];    // [stage][K half]: 128 blocks x 64 dims, SW128
    unsigned char dec[kFtDecBufs][2][kFtM * 128];  // [buffer][K half]: one eigenvector as bf16
    unsigned char q[kFtStages][2][kFtN * 128];     // [stage][K half]: 16 rows x 64 dims, rows >= G zero
    unsigned char p[kFtStages][2][kFtN * 128];     // subspace form: projected query, value row g, residual 8 + g
    uint64_t full[kFtStages], raw_empty[kFtStages], dec_full[kFtDecBufs], dec_empty[kFtDecBufs];
    uint64_t tm_full[2], tm_empty[2];
    uint32_t tmem_base;
    int fail;
};

struct FtArgs {
    const __nv_bfloat16 *mu16;
    const uint8_t *xi4;
    const float *xi_scale;
    float *sc_out;
    int n_kv, n_q, G, R, n_full, tiles_per_sh, total_tiles, tiles_per_cta;
    int code_bytes;     // bytes of codes per eigenvector: 64 (D = 128) or 48 (subspace, <= 96 dims)
    int split;          // 1: the code products take the projected query (bf16 value + residual)
    float scale;
};

__global__ void __launch_bounds__(kFtThreads, 1)
block_score_fp4_tc_kernel(const __grid_constant__ CUtensorMap tmu, const __grid_constant__ CUtensorMap tq,
                          const __grid_constant__ CUtensorMap tp, FtArgs a) {
    extern __shared__ unsigned char ft_raw[];
    const uint32_t mis = smem_u32(ft_raw) & 1023u;
    FtSmem &S = *reinterpret_cast<FtSmem *>(ft_raw + ((1024u - mis) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t_lo = blockIdx.x * a.tiles_per_cta;
    const int nt = min(a.total_tiles, t_lo + a.tiles_per_cta) - t_lo;
    if (nt <= 0) return;
    const int R = a.R;
    if (tid == 0) {
        for (int i = 0; i < kFtStages; ++i) {
            tc::mbar_init(&S.full[i], 1);
            tc::mbar_init(&S.raw_empty[i], 1);
        }
        for (int i = 0; i < kFtDecBufs; ++i) {
            tc::mbar_init(&S.dec_full[i], kFtDecWarps);
            tc::mbar_init(&S.dec_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&S.tm_full[i], 1);
            tc::mbar_init(&S.tm_empty[i], 4);
        }
        tc::mbar_fence_init();
        S.fail = 0;
    }
    {   // query rows G..15 of every stage stay zero (the TMA box writes rows 0..G-1)
        uint4 *qz = reinterpret_cast<uint4 *>(&S.q[0][0][0]);
        for (int i = tid; i < (int)(sizeof(S.q) / 16); i += kFtThreads) qz[i] = make_uint4(0, 0, 0, 0);
    }
    tc::fence_proxy_async();
    if (warp == 1) tc::tmem_alloc(&S.tmem_base, 256);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = S.tmem_base;
    auto tile_of = [&](int i, int &sh, int &b0, int &nb) {
        const int t = t_lo + i;
        sh = t / a.tiles_per_sh;
        b0 = (t - sh * a.tiles_per_sh) * kFtM;
        nb = min(kFtM, a.n_full - b0);
    };

    if (warp == 0) {
        // ---------------- loads
        if (lane == 0) {
            for (int i = 0; i < nt; ++i) {
                const int s = i % kFtStages, u = i / kFtStages;
                if (u > 0 && !tc::mbar_wait_bounded(&S.raw_empty[s], (u - 1) & 1, kBsWaitNs, K_BLK_SCORE, 10,
                                                    kFtSuspendNs)) {
                    atomicOr(&S.fail, 1);
                    break;
                }
                int sh, b0, nb;
                tile_of(i, sh, b0, nb);
                const int seq = sh / a.n_kv, h = sh - seq * a.n_kv;
                tc::mbar_arrive_expect_tx(&S.full[s], 2 * kFtM * 128 + 2 * a.G * 128 + (a.split ? 2 * kFtN * 128 : 0));
                const int row = sh * a.n_full + b0;
                tc::tma_load_2d(S.mu[s][0], &tmu, 0, row, &S.full[s]);
                tc::tma_load_2d(S.mu[s][1], &tmu, 64, row, &S.full[s]);
                const int qrow = seq * a.n_q + h * a.G;
                tc::tma_load_2d(S.q[s][0], &tq, 0, qrow, &S.full[s]);
                tc::tma_load_2d(S.q[s][1], &tq, 64, qrow, &S.full[s]);
                if (a.split) {           // this (sequence, KV head)'s 16 projected rows
                    tc::tma_load_2d(S.p[s][0], &tp, 0, sh * kFtN, &S.full[s]);
                    tc::tma_load_2d(S.p[s][1], &tp, 64, sh * kFtN, &S.full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16_f32(kFtM, kFtN, 0, 0);
            bool ok = true;
            int j = 0;                                   // eigenvector tiles consumed so far
            for (int i = 0; ok && i < nt; ++i) {
                const int s = i % kFtStages, u = i / kFtStages, acc = i & 1, w = i >> 1;
                ok = tc::mbar_wait_bounded(&S.full[s], u & 1, kBsWaitNs, K_BLK_SCORE, 11, kFtSuspendNs);
                if (ok && w > 0)
                    ok = tc::mbar_wait_bounded(&S.tm_empty[acc], (w - 1) & 1, kBsWaitNs, K_BLK_SCORE, 12,
                                               kFtSuspendNs);
                if (!ok) break;
                tc::fence_after();
                const uint32_t d0 = tmem + acc * 128;
                auto mma_tile = [&](unsigned char (*A)[kFtM * 128], unsigned char (*B)[kFtN * 128], uint32_t d) {
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t ad = tc::smem_desc(smem_u32(A[kh]) + k * 32, 16, 1024, tc::kLayoutSW128);
                            const uint64_t bd = tc::smem_desc(smem_u32(B[kh]) + k * 32, 16, 1024,
                                                              tc::kLayoutSW128);
                            tc::mma_bf16(d, ad, bd, idesc, (kh | k) ? 1u : 0u);
                        }
                };
                mma_tile(S.mu[s], S.q[s], d0);
                for (int e = 0; e < R; ++e, ++j) {
                    const int b = j % kFtDecBufs, v = j / kFtDecBufs;
                    ok = tc::mbar_wait_bounded(&S.dec_full[b], v & 1, kBsWaitNs, K_BLK_SCORE, 13, kFtSuspendNs);
                    if (!ok) break;
                    tc::fence_after();
                    mma_tile(S.dec[b], a.split ? S.p[s] : S.q[s], d0 + 16 * (1 + e));
                    tc::commit(&S.dec_empty[b]);
                }
                if (!ok) break;
                tc::commit(&S.raw_empty[s]);
                tc::commit(&S.tm_full[acc]);
            }
            if (!ok) atomicOr(&S.fail, 1);
        }
    } else if (warp >= 8) {
        // ---------------- widen the codes.  A thread owns, per eigenvector e and
        // K half kh, words [c0, c0 + 4) of block r: dims [64 kh + 8 c, +8) for
        // c in that range, which become 16-byte chunks c of row r.  A quarter
        // warp covers 4 consecutive rows x both c0, so its swizzled 16-byte
        // stores hit 8 distinct bank groups.  The codes of tile i+1 are read
        // (16-byte loads) into registers while tile i is widened.
        const int dw = warp - 8;
        const int r = dw * 16 + (lane >> 3) * 4 + ((lane & 7) >> 1), c0 = (lane & 1) * 4;
        uint4 cur[kFtMaxR][2], nxt[kFtMaxR][2];
        auto fetch = [&](int i, uint4 (&dst)[kFtMaxR][2]) {
            int sh, b0, nb;
            tile_of(i, sh, b0, nb);
            const uint8_t *src = a.xi4 + ((size_t)sh * a.n_full + b0 + r) * R * a.code_bytes + c0 * 4;
#pragma unroll
            for (int e = 0; e < kFtMaxR; ++e)
#pragma unroll
                for (int kh = 0; kh < 2; ++kh)     // codes past code_bytes (dims the vector lacks) are zero
                    dst[e][kh] = (e < R && r < nb && kh * 32 + c0 * 4 < a.code_bytes)
                                     ? __ldg(reinterpret_cast<const uint4 *>(src + e * a.code_bytes + kh * 32))
                                     : make_uint4(0, 0, 0, 0);
        };
        fetch(0, cur);
        int j = 0;
        bool ok = true;
        for (int i = 0; ok && i < nt; ++i) {
            if (i + 1 < nt) fetch(i + 1, nxt);
#pragma unroll
            for (int e = 0; e < kFtMaxR; ++e) {
                if (e >= R) break;
                const int b = j % kFtDecBufs, v = j / kFtDecBufs;
                ++j;
                if (v > 0) {
                    ok = tc::mbar_wait_bounded(&S.dec_empty[b], (v - 1) & 1, kBsWaitNs, K_BLK_SCORE, 15,
                                               kFtSuspendNs);
                    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                }
#pragma unroll
                for (int kh = 0; kh < 2; ++kh) {
                    const uint32_t wv[4] = {cur[e][kh].x, cur[e][kh].y, cur[e][kh].z, cur[e][kh].w};
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        *reinterpret_cast<uint4 *>(S.dec[b][kh] + tc::sw128(r, c0 + k)) = e2m1x8_to_bf16(wv[k]);
                }
                tc::fence_proxy_async();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&S.dec_full[b]);
            }
#pragma unroll
            for (int e = 0; e < kFtMaxR; ++e)
#pragma unroll
                for (int kh = 0; kh < 2; ++kh) cur[e][kh] = nxt[e][kh];
        }
        if (!ok && lane == 0) atomicOr(&S.fail, 1);
    } else if (warp >= 4) {
        // ---------------- epilogue: thread = TMEM lane = block b0 + row
        const int quad = warp & 3, row = quad * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        // this block's FP4 scales, read kFtScaleAhead tiles ahead so that no
        // global-load latency sits between two accumulator hand-offs
        constexpr int kFtScaleAhead = 3;
        float sring[kFtScaleAhead + 1][kFtMaxR];
        auto load_sig = [&](int i, float (&dst)[kFtMaxR]) {
            int sh, b0, nb;
            tile_of(i, sh, b0, nb);
            const bool valid = i < nt && row < nb;
            const size_t blk = (size_t)sh * a.n_full + b0 + row;
#pragma unroll
            for (int e = 0; e < kFtMaxR; ++e)
                dst[e] = (valid && e < R) ? __ldg(a.xi_scale + blk * R + e) : 0.0f;
        };
#pragma unroll
        for (int k = 0; k < kFtScaleAhead; ++k) load_sig(k, sring[k]);
        for (int i = 0; i < nt; ++i) {
            const int acc = i & 1, w = i >> 1;
            int sh, b0, nb;
            tile_of(i, sh, b0, nb);
            const bool valid = row < nb;
            load_sig(i + kFtScaleAhead, sring[kFtScaleAhead]);
            float sig[kFtMaxR];
#pragma unroll
            for (int e = 0; e < kFtMaxR; ++e) sig[e] = a.scale * sring[0][e];
#pragma unroll
            for (int k = 0; k < kFtScaleAhead; ++k)
#pragma unroll
                for (int e = 0; e < kFtMaxR; ++e) sring[k][e] = sring[k + 1][e];
            const bool ok = tc::mbar_wait_bounded(&S.tm_full[acc], w & 1, kBsWaitNs, K_BLK_SCORE, 16, kFtSuspendNs);
            if (__any_sync(0xffffffffu, !ok)) {
                if (lane == 0) atomicOr(&S.fail, 1);
                break;
            }
            tc::fence_after();
            uint32_t d[1 + kFtMaxR][16];
            tc::tmem_ld16(tl + acc * 128, d[0]);
#pragma unroll
            for (int e = 0; e < kFtMaxR; ++e)
                if (e < R) tc::tmem_ld16(tl + acc * 128 + 16 * (1 + e), d[1 + e]);
            tc::tmem_ld_wait();
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.tm_empty[acc]);
            if (valid) {
#pragma unroll
                for (int g = 0; g < kFtN; ++g) {
                    if (g >= a.G) break;
                    float quad2 = 0.0f;
#pragma unroll
                    for (int e = 0; e < kFtMaxR; ++e) {      // sig[e] = 0 for e >= R
                        float dot = __uint_as_float(e < R ? d[1 + e][g] : 0u);
                        // + the residual column (rows 8 + g of the split query: a fixed index)
                        if (a.split && g < kFtN / 2) dot += __uint_as_float(e < R ? d[1 + e][kFtN / 2 + g] : 0u);
                        const float pe = sig[e] * dot;
                        quad2 = fmaf(pe, pe, quad2);
                    }
                    a.sc_out[((size_t)sh * a.G + g) * a.n_full + b0 + row] =
                        fmaf(0.5f, quad2, a.scale * __uint_as_float(d[0][g]));
                }
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (S.fail && tid == 0) raise_error(CRS_DEVERR_TIMEOUT);
    if (warp == 1) tc::tmem_dealloc(tmem, 256);
}

static int bd_validate(const crs_block_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->n_seq < 1 || p->n_kv < 1 || p->T < 1) return CRS_ERR_INVALID_ARG;
    if (p->D != kBdD) return CRS_ERR_UNSUPPORTED;
    if (p->L < 2 || p->L > kBdMaxL || (p->L & 1)) return CRS_ERR_UNSUPPORTED;
    if (p->rank < 1 || p->rank > 8 || p->rank > p->L) return CRS_ERR_INVALID_ARG;
    return CRS_OK;
}

}  // namespace crs

using namespace crs;

extern "C" int crs_block_describe(const crs_block_params *p, const void *K, float *mu, float *xi,
                                  void *stream) {
    int st = bd_validate(p);
    if (st) return st;
    if (!K || !mu || !xi) return CRS_ERR_INVALID_ARG;
    const int n_full = p->T / p->L;
    if (p->blk_begin < 0 || p->blk_end > n_full || p->blk_begin > p->blk_end)
        return CRS_ERR_INVALID_ARG;
    const int n_blk = p->blk_end - p->blk_begin;
    if (n_blk == 0) return CRS_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t smem = sizeof(BdWarpSmem) * kBdWarps;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_describe_kernel<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    dim3 grid(ceil_div(n_blk, kBdWarps), p->n_seq * p->n_kv);
    {
        ProfScope _ps(K_BLK_DESCRIBE, s);
        block_describe_kernel<false><<<grid, kBdWarps * 32, smem, s>>>(
            static_cast<const __nv_bfloat16 *>(K), mu, xi, p->n_kv, p->T, p->L, p->rank, p->blk_begin,
            n_blk, n_full, nullptr, 0);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

extern "C" int crs_block_describe_ss(const crs_block_params *p, const void *K, const float *U, int sd,
                                     float *mu, float *xi_ss, void *stream) {
    int st = bd_validate(p);
    if (st) return st;
    if (!K || !U || !mu || !xi_ss) return CRS_ERR_INVALID_ARG;
    if (sd < 1 || sd > kBdD) return CRS_ERR_INVALID_ARG;
    const int n_full = p->T / p->L;
    if (p->blk_begin < 0 || p->blk_end > n_full || p->blk_begin > p->blk_end)
        return CRS_ERR_INVALID_ARG;
    const int n_blk = p->blk_end - p->blk_begin;
    if (n_blk == 0) return CRS_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t smem = (sizeof(BdWarpSmem) + sizeof(BdWarpSmemSS)) * kBdWarps + (size_t)kBdD * sd * 4;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_describe_kernel<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    dim3 grid(ceil_div(n_blk, kBdWarps), p->n_seq * p->n_kv);
    {
        ProfScope _ps(K_BLK_DESCRIBE, s);
        block_describe_kernel<true><<<grid, kBdWarps * 32, smem, s>>>(
            static_cast<const __nv_bfloat16 *>(K), mu, xi_ss, p->n_kv, p->T, p->L, p->rank, p->blk_begin,
            n_blk, n_full, U, sd);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

static int bs_validate(const crs_block_sel_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->b.rank < 0) return CRS_ERR_INVALID_ARG;
    crs_block_params b = p->b;
    b.blk_begin = 0;
    b.blk_end = 0;
    b.rank = max(1, b.rank);                 // rank 0: the first-order (mean-pool) score
    int st = bd_validate(&b);
    if (st) return st;
    if (p->n_q < 1 || p->n_q % p->b.n_kv) return CRS_ERR_INVALID_ARG;
    const int G = p->n_q / p->b.n_kv;
    if (G > 16 || (16 % G) != 0) return CRS_ERR_UNSUPPORTED;
    const int n_full = p->b.T / p->b.L;
    if (n_full < 1 || n_full > 8192) return CRS_ERR_UNSUPPORTED;
    if (p->top_blocks < 1 || p->top_blocks > n_full) return CRS_ERR_INVALID_ARG;
    if (p->window < 0 || p->window > p->b.T) return CRS_ERR_INVALID_ARG;
    return CRS_OK;
}

// K9b launch shared by every selector: scores sc [n_seq * n_kv][G][n_full] -> token lists.
static int launch_block_pick(const crs_block_sel_params *p, const float *sc, int32_t *tok_idx,
                             int32_t *tok_count, cudaStream_t s) {
    const int G = p->n_q / p->b.n_kv, n_full = p->b.T / p->b.L;
    const int cap = p->top_blocks * p->b.L + p->window;
    const size_t smem_b = pick_smem_bytes(G, n_full, p->top_blocks);
    if (smem_b > 200 * 1024) return CRS_ERR_UNSUPPORTED;
    CRS_TRY_CUDA(pick_prepare(n_full, smem_b));
    {
        ProfScope _ps(K_BLK_PICK, s);
        launch_pick(n_full, p->b.n_seq * p->b.n_kv, smem_b, s, sc, tok_idx, tok_count, G, n_full, p->b.L,
                    p->b.T, p->top_blocks, p->window, cap);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

extern "C" size_t crs_block_select_workspace_size(const crs_block_sel_params *p) {
    if (bs_validate(p)) return 0;
    const size_t n_full = p->b.T / p->b.L;
    return (size_t)p->b.n_seq * p->n_q * n_full * sizeof(float);
}

extern "C" int crs_block_select(const crs_block_sel_params *p, const void *Q, const float *mu,
                                const float *xi, int32_t *tok_idx, int32_t *tok_count, void *ws,
                                size_t ws_bytes, void *stream) {
    int st = bs_validate(p);
    if (st) return st;
    if (!Q || !mu || (!xi && p->b.rank > 0) || !tok_idx || !tok_count) return CRS_ERR_INVALID_ARG;
    const size_t need = crs_block_select_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int G = p->n_q / p->b.n_kv;
    const int n_full = p->b.T / p->b.L;
    if (p->b.rank == 0) {                    // mean-pool: q . mu only
        if ((reinterpret_cast<uintptr_t>(Q) & 7) || (reinterpret_cast<uintptr_t>(mu) & 15))
            return CRS_ERR_INVALID_ARG;
        float *sc = static_cast<float *>(ws);
        {
            ProfScope _ps(K_BLK_SCORE, s);
            CRS_TRY_CUDA(launch_score_warp<kWsMean>(G, score_warp_grid(G, n_full, p->b.n_seq * p->b.n_kv), s,
                                                    Q, mu, nullptr, sc, p->b.n_kv, p->n_q, n_full, p->scale));
        }
        return launch_block_pick(p, sc, tok_idx, tok_count, s);
    }
    const int nbt = bs_tile(G);
    const size_t smem_a = ((size_t)2 * G * (kBdD + 1) + (size_t)nbt * (1 + p->b.rank) * (kBdD + 1)) * 4;
    if (smem_a > 227 * 1024) return CRS_ERR_UNSUPPORTED;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a));
    float *sc = static_cast<float *>(ws);
    if (G == 8 && p->b.rank == 4) {
        const long long n_sh = (long long)p->b.n_seq * p->b.n_kv;
        const long long total = n_sh * ceil_div(n_full, kBsChunk);
        if (total > 0x7fffffffLL) return CRS_ERR_UNSUPPORTED;
        int dev = 0, sms = 148;
        CRS_TRY_CUDA(cudaGetDevice(&dev));
        CRS_TRY_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
        const int grid = (int)min(total, (long long)2 * sms);          // two CTAs per SM, one wave
        const int cpc = (int)ceil_div_ll(total, grid);
        const size_t smem_s = sizeof(BsSmem<8, 4>);
        CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_tma_kernel<8, 4>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s));
        ProfScope _ps(K_BLK_SCORE, s);
        block_score_tma_kernel<8, 4><<<(unsigned)ceil_div_ll(total, cpc), kBsThreadsT, smem_s, s>>>(
            static_cast<const __nv_bfloat16 *>(Q), mu, xi, sc, p->b.n_kv, p->n_q, n_full, (int)total, cpc, p->scale);
    } else {
    dim3 ga(ceil_div(n_full, nbt), p->b.n_seq * p->b.n_kv);
    {
        ProfScope _ps(K_BLK_SCORE, s);
        block_score_kernel<<<ga, kBsThreads, smem_a, s>>>(static_cast<const __nv_bfloat16 *>(Q), mu, xi,
                                                          sc, p->b.n_kv, p->n_q, G, p->b.rank, n_full,
                                                          p->scale, kBdD, nullptr);
    }
    }
    CRS_CHECK_LAUNCH();
    return launch_block_pick(p, sc, tok_idx, tok_count, s);
}

extern "C" int crs_block_quantize(const crs_block_params *p, const float *mu, const float *xi,
                                  void *mu16, uint8_t *xi4, float *xi_scale, void *stream) {
    if (!p) return CRS_ERR_INVALID_ARG;
    crs_block_params b = *p;
    b.blk_begin = 0;
    b.blk_end = 0;
    int st = bd_validate(&b);
    if (st) return st;
    if (!mu || !xi || !mu16 || !xi4 || !xi_scale) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mu) | reinterpret_cast<uintptr_t>(xi) |
         reinterpret_cast<uintptr_t>(mu16) | reinterpret_cast<uintptr_t>(xi4)) & 15)
        return CRS_ERR_INVALID_ARG;
    const long long n_mu = (long long)p->n_seq * p->n_kv * (p->T / p->L);
    const long long n_xi = n_mu * p->rank;
    if (n_mu == 0) return CRS_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        ProfScope _ps(K_BLK_QUANTIZE, s);
        block_quantize_kernel<<<(unsigned)ceil_div_ll(n_mu + n_xi, 8), 256, 0, s>>>(
            mu, xi, static_cast<__nv_bfloat16 *>(mu16), xi4, xi_scale, n_mu, n_xi);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

extern "C" int crs_block_select_fp4(const crs_block_sel_params *p, const void *Q, const void *mu16,
                                    const uint8_t *xi4, const float *xi_scale, int32_t *tok_idx,
                                    int32_t *tok_count, void *ws, size_t ws_bytes, void *stream) {
    int st = bs_validate(p);
    if (st) return st;
    if (!Q || !mu16 || !xi4 || !xi_scale || !tok_idx || !tok_count) return CRS_ERR_INVALID_ARG;
    const int G = p->n_q / p->b.n_kv, R = p->b.rank;
    if (R < 1) return CRS_ERR_INVALID_ARG;
    if (R > kFtMaxR) return CRS_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(mu16) |
         reinterpret_cast<uintptr_t>(xi4)) & 15)
        return CRS_ERR_INVALID_ARG;
    const size_t need = crs_block_select_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int n_full = p->b.T / p->b.L;
    float *sc = static_cast<float *>(ws);
    const int n_sh = p->b.n_seq * p->b.n_kv;
    PFN_cuTensorMapEncodeTiled_v12000 enc = tc::tensor_map_encoder();
    if (!enc) return CRS_ERR_CUDA;
    CUtensorMap tmu, tq;
    {   // means: [n_sh * n_full rows, 128 dims] bf16; a box is 128 blocks x 64 dims
        cuuint64_t dims[2] = {(cuuint64_t)kBdD, (cuuint64_t)n_sh * n_full};
        cuuint64_t strides[1] = {(cuuint64_t)kBdD * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)kFtM};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&tmu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(mu16), dims, strides, box,
                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CRS_ERR_CUDA;
    }
    {   // queries: [n_seq * n_q rows, 128 dims] bf16; a box is one KV head's G rows x 64 dims
        cuuint64_t dims[2] = {(cuuint64_t)kBdD, (cuuint64_t)p->b.n_seq * p->n_q};
        cuuint64_t strides[1] = {(cuuint64_t)kBdD * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)G};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(Q), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CRS_ERR_CUDA;
    }
    FtArgs fa;
    fa.mu16 = static_cast<const __nv_bfloat16 *>(mu16);
    fa.xi4 = xi4;
    fa.xi_scale = xi_scale;
    fa.sc_out = sc;
    fa.n_kv = p->b.n_kv;
    fa.n_q = p->n_q;
    fa.G = G;
    fa.R = R;
    fa.n_full = n_full;
    fa.tiles_per_sh = ceil_div(n_full, kFtM);
    fa.total_tiles = n_sh * fa.tiles_per_sh;
    fa.scale = p->scale;
    fa.code_bytes = kBdD / 2;
    fa.split = 0;
    int dev = 0, sms = 148;
    CRS_TRY_CUDA(cudaGetDevice(&dev));
    CRS_TRY_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    fa.tiles_per_cta = ceil_div(fa.total_tiles, max(1, sms));     // one CTA per SM
    const int grid = ceil_div(fa.total_tiles, fa.tiles_per_cta);
    const size_t smem_s = sizeof(FtSmem) + 1024;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_fp4_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s));
    {
        ProfScope _ps(K_BLK_SCORE, s);
        block_score_fp4_tc_kernel<<<grid, kFtThreads, smem_s, s>>>(tmu, tq, tq, fa);
    }
    CRS_CHECK_LAUNCH();
    return launch_block_pick(p, sc, tok_idx, tok_count, s);
}

extern "C" int crs_block_quest_describe(const crs_block_params *p, const void *K, void *kmin, void *kmax,
                                        void *stream) {
    if (!p) return CRS_ERR_INVALID_ARG;
    crs_block_params b = *p;
    b.rank = 1;                              // no eigenvectors here
    int st = bd_validate(&b);
    if (st) return st;
    if (!K || !kmin || !kmax) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(kmin) | reinterpret_cast<uintptr_t>(kmax)) & 7)
        return CRS_ERR_INVALID_ARG;
    const int n_full = p->T / p->L;
    if (p->blk_begin < 0 || p->blk_end > n_full || p->blk_begin > p->blk_end) return CRS_ERR_INVALID_ARG;
    const int n_blk = p->blk_end - p->blk_begin;
    if (n_blk == 0) return CRS_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        ProfScope _ps(K_BLK_DESCRIBE, s);
        quest_describe_kernel<<<dim3(ceil_div(n_blk, kQdWarps), p->n_seq * p->n_kv), kQdWarps * 32, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(K), static_cast<__nv_bfloat16 *>(kmin),
            static_cast<__nv_bfloat16 *>(kmax), p->T, p->n_kv, p->L, n_full, p->blk_begin, n_blk);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

extern "C" int crs_block_select_quest(const crs_block_sel_params *p, const void *Q, const void *kmin,
                                      const void *kmax, int32_t *tok_idx, int32_t *tok_count, void *ws,
                                      size_t ws_bytes, void *stream) {
    int st = bs_validate(p);
    if (st) return st;
    if (!Q || !kmin || !kmax || !tok_idx || !tok_count) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(kmin) | reinterpret_cast<uintptr_t>(kmax)) & 7)
        return CRS_ERR_INVALID_ARG;
    const size_t need = crs_block_select_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int G = p->n_q / p->b.n_kv, n_full = p->b.T / p->b.L;
    float *sc = static_cast<float *>(ws);
    {
        ProfScope _ps(K_BLK_SCORE, s);
        CRS_TRY_CUDA(launch_score_warp<kWsQuest>(G, score_warp_grid(G, n_full, p->b.n_seq * p->b.n_kv), s, Q,
                                                 kmin, kmax, sc, p->b.n_kv, p->n_q, n_full, p->scale));
    }
    return launch_block_pick(p, sc, tok_idx, tok_count, s);
}

extern "C" size_t crs_block_select_ss_workspace_size(const crs_block_sel_params *p, int sd) {
    const size_t sc = crs_block_select_workspace_size(p);
    if (sc == 0 || sd < 1 || sd > kBdD) return 0;
    return ((sc + 255) & ~size_t(255)) + (size_t)p->b.n_seq * p->n_q * sd * sizeof(float);
}

extern "C" int crs_block_select_ss(const crs_block_sel_params *p, const void *Q, const float *U, int sd,
                                   const float *mu, const float *xi_ss, int32_t *tok_idx, int32_t *tok_count,
                                   void *ws, size_t ws_bytes, void *stream) {
    int st = bs_validate(p);
    if (st) return st;
    if (p->b.rank < 1) return CRS_ERR_INVALID_ARG;
    if (!Q || !U || !mu || !xi_ss || !tok_idx || !tok_count) return CRS_ERR_INVALID_ARG;
    if (sd < 1 || sd > kBdD) return CRS_ERR_INVALID_ARG;
    const size_t need = crs_block_select_ss_workspace_size(p, sd);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int G = p->n_q / p->b.n_kv, n_full = p->b.T / p->b.L;
    float *sc = static_cast<float *>(ws);
    float *qx = reinterpret_cast<float *>(static_cast<char *>(ws) +
                                          ((crs_block_select_workspace_size(p) + 255) & ~size_t(255)));
    const int n_rows = p->b.n_seq * p->n_q;
    const int nbt = bs_tile(G);
    const size_t smem_a = ((size_t)2 * G * (kBdD + 1) + (size_t)nbt * (1 + p->b.rank) * (kBdD + 1)) * 4;
    if (smem_a > 227 * 1024) return CRS_ERR_UNSUPPORTED;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem_a));
    {
        ProfScope _ps(K_BLK_SCORE, s);
        _ps.more(1);                              // projection + scorer
        const size_t psm = ((size_t)kBdD * sd + 16 * kBdD) * 4;
        CRS_TRY_CUDA(cudaFuncSetAttribute(query_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)psm));
        query_project_kernel<<<ceil_div(n_rows, 16), 256, psm, s>>>(
            static_cast<const __nv_bfloat16 *>(Q), U, qx,
                                                                  n_rows, sd, p->scale);
        block_score_kernel<<<dim3(ceil_div(n_full, nbt), p->b.n_seq * p->b.n_kv), kBsThreads, smem_a, s>>>(
            static_cast<const __nv_bfloat16 *>(Q), mu, xi_ss, sc, p->b.n_kv, p->n_q, G, p->b.rank, n_full,
            p->scale, sd, qx);
    }
    CRS_CHECK_LAUNCH();
    return launch_block_pick(p, sc, tok_idx, tok_count, s);
}

// ---------------------------------------------------------------------------
// The pages' deployed descriptor ([P5] "子空间方法" Eq.(17)-(18) with "量化",
// Table 3's delivered row): the bf16 block mean in the full space and the r
// scaled eigenvectors of the query-subspace covariance U^T Sigma U (sd <= 96
// dims) in E2M1 FP4, one fp32 scale each.  Codes are stored 48 bytes per
// vector (96 dims, those past sd zero) so that every vector starts on a
// 16-byte boundary.
// ---------------------------------------------------------------------------
namespace crs {
constexpr int kSsPad = 96;                  // stored subspace dims
constexpr int kSsCodeBytes = kSsPad / 2;

// one warp per vector: vectors v < n_mu are means (bf16), the rest subspace
// eigenvectors; lane l < 24 takes dims [4l, 4l + 4)
__global__ void __launch_bounds__(256) block_quantize_ss_kernel(const float *__restrict__ mu,
                                                                const float *__restrict__ xi,
                                                                __nv_bfloat16 *__restrict__ mu16,
                                                                uint8_t *__restrict__ xi4,
                                                                float *__restrict__ xi_scale, long long n_mu,
                                                                long long n_xi, int sd) {
    const long long v = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (v < n_mu) {
        const float4 x = reinterpret_cast<const float4 *>(mu + v * kBdD)[lane];
        __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t *>(&a);
        o.y = *reinterpret_cast<uint32_t *>(&b);
        reinterpret_cast<uint2 *>(mu16 + v * kBdD)[lane] = o;
        return;
    }
    const long long w = v - n_mu;
    if (w >= n_xi) return;
    float x[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int dd = 4 * lane + t;
        x[t] = dd < sd ? xi[w * sd + dd] : 0.0f;
    }
    const float amax = warp_max(fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))));
    const float sc = amax / 6.0f;
    const uint32_t c = e2m1_code(x[0], sc) | (e2m1_code(x[1], sc) << 4) | (e2m1_code(x[2], sc) << 8) |
                       (e2m1_code(x[3], sc) << 12);
    if (lane < kSsPad / 4) reinterpret_cast<uint16_t *>(xi4 + w * kSsCodeBytes)[lane] = (uint16_t)c;
    if (lane == 0) xi_scale[w] = sc;
}

// P[sh][row][j]: per (sequence, KV head) the G projected queries p_g = U^T q_g
// (fp32, one FMA per term in dim order) as a bf16 value (row g) and the bf16
// residual p_g - value (row 8 + g); dims past sd and the other rows zero.
// One CTA per (sequence, KV head): U and the G query rows staged in shared memory.
__global__ void __launch_bounds__(256) query_project_split_kernel(const __nv_bfloat16 *__restrict__ Q,
                                                                  const float *__restrict__ U,
                                                                  __nv_bfloat16 *__restrict__ P, int n_sh,
                                                                  int n_kv, int n_q, int G, int sd) {
    extern __shared__ float qs_smem[];
    float *Us = qs_smem;                          // [D][sd]
    float *qs = Us + (size_t)kBdD * sd;           // [G][D]
    const int sh = blockIdx.x, seq = sh / n_kv, h = sh - seq * n_kv;
    stage_floats(Us, U, kBdD * sd);
    for (int e = threadIdx.x; e < G * kBdD; e += blockDim.x)
        qs[e] = __bfloat162float(Q[((size_t)seq * n_q + h * G) * kBdD + e]);
    __syncthreads();
    __nv_bfloat16 *out = P + (size_t)sh * kFtN * kBdD;
    constexpr int kHalf = kFtN / 2;               // value rows 0..7, residual rows 8..15
    for (int e = threadIdx.x; e < kHalf * kBdD; e += blockDim.x) {
        const int r = e / kBdD, j = e - r * kBdD;
        float acc = 0.0f;
        if (r < G && j < sd) {
#pragma unroll 8
            for (int dd = 0; dd < kBdD; ++dd) acc = fmaf(Us[dd * sd + j], qs[r * kBdD + dd], acc);
        }
        const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
        out[e] = hi;
        out[(size_t)(kHalf + r) * kBdD + j] = __float2bfloat16_rn(acc - __bfloat162float(hi));
    }
}

}  // namespace crs

using namespace crs;

extern "C" int crs_block_quantize_ss(const crs_block_params *p, const float *mu, const float *xi_ss, int sd,
                                     void *mu16, uint8_t *xi4, float *xi_scale, void *stream) {
    if (!p) return CRS_ERR_INVALID_ARG;
    crs_block_params b = *p;
    b.blk_begin = 0;
    b.blk_end = 0;
    int st = bd_validate(&b);
    if (st) return st;
    if (sd < 1 || sd > kBdD) return CRS_ERR_INVALID_ARG;
    if (sd > kSsPad) return CRS_ERR_UNSUPPORTED;
    if (!mu || !xi_ss || !mu16 || !xi4 || !xi_scale) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mu) | reinterpret_cast<uintptr_t>(mu16) | reinterpret_cast<uintptr_t>(xi4)) &
        15)
        return CRS_ERR_INVALID_ARG;
    const long long n_mu = (long long)p->n_seq * p->n_kv * (p->T / p->L);
    const long long n_xi = n_mu * p->rank;
    if (n_mu == 0) return CRS_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        ProfScope _ps(K_BLK_QUANTIZE, s);
        block_quantize_ss_kernel<<<(unsigned)ceil_div_ll(n_mu + n_xi, 8), 256, 0, s>>>(
            mu, xi_ss, static_cast<__nv_bfloat16 *>(mu16), xi4, xi_scale, n_mu, n_xi, sd);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

extern "C" size_t crs_block_select_fp4_ss_workspace_size(const crs_block_sel_params *p, int sd) {
    const size_t sc = crs_block_select_workspace_size(p);
    if (sc == 0 || sd < 1 || sd > kSsPad) return 0;
    return ((sc + 255) & ~size_t(255)) + (size_t)p->b.n_seq * p->b.n_kv * kFtN * kBdD * 2;
}

extern "C" int crs_block_select_fp4_ss(const crs_block_sel_params *p, const void *Q, const float *U, int sd,
                                       const void *mu16, const uint8_t *xi4, const float *xi_scale,
                                       int32_t *tok_idx, int32_t *tok_count, void *ws, size_t ws_bytes,
                                       void *stream) {
    int st = bs_validate(p);
    if (st) return st;
    if (!Q || !U || !mu16 || !xi4 || !xi_scale || !tok_idx || !tok_count) return CRS_ERR_INVALID_ARG;
    const int G = p->n_q / p->b.n_kv, R = p->b.rank;
    if (R < 1 || sd < 1 || sd > kBdD) return CRS_ERR_INVALID_ARG;
    if (R > kFtMaxR || sd > kSsPad || 2 * G > kFtN) return CRS_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(mu16) | reinterpret_cast<uintptr_t>(xi4)) &
        15)
        return CRS_ERR_INVALID_ARG;
    const size_t need = crs_block_select_fp4_ss_workspace_size(p, sd);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int n_full = p->b.T / p->b.L;
    float *sc = static_cast<float *>(ws);
    __nv_bfloat16 *P = reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) +
                                                         ((crs_block_select_workspace_size(p) + 255) & ~size_t(255)));
    const int n_sh = p->b.n_seq * p->b.n_kv;
    PFN_cuTensorMapEncodeTiled_v12000 enc = tc::tensor_map_encoder();
    if (!enc) return CRS_ERR_CUDA;
    CUtensorMap tmu, tq, tp;
    auto encode = [&](CUtensorMap *m, const void *base, cuuint64_t rows, cuuint32_t box_rows) {
        cuuint64_t dims[2] = {(cuuint64_t)kBdD, rows};
        cuuint64_t strides[1] = {(cuuint64_t)kBdD * 2};
        cuuint32_t box[2] = {64, box_rows};
        cuuint32_t estr[2] = {1, 1};
        return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    if (!encode(&tmu, mu16, (cuuint64_t)n_sh * n_full, kFtM) ||
        !encode(&tq, Q, (cuuint64_t)p->b.n_seq * p->n_q, (cuuint32_t)G) ||
        !encode(&tp, P, (cuuint64_t)n_sh * kFtN, kFtN))
        return CRS_ERR_CUDA;
    FtArgs fa;
    fa.mu16 = static_cast<const __nv_bfloat16 *>(mu16);
    fa.xi4 = xi4;
    fa.xi_scale = xi_scale;
    fa.sc_out = sc;
    fa.n_kv = p->b.n_kv;
    fa.n_q = p->n_q;
    fa.G = G;
    fa.R = R;
    fa.n_full = n_full;
    fa.tiles_per_sh = ceil_div(n_full, kFtM);
    fa.total_tiles = n_sh * fa.tiles_per_sh;
    fa.scale = p->scale;
    fa.code_bytes = kSsCodeBytes;
    fa.split = 1;
    int dev = 0, sms = 148;
    CRS_TRY_CUDA(cudaGetDevice(&dev));
    CRS_TRY_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    fa.tiles_per_cta = ceil_div(fa.total_tiles, max(1, sms));
    const int grid = ceil_div(fa.total_tiles, fa.tiles_per_cta);
    const size_t smem_s = sizeof(FtSmem) + 1024;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_fp4_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s));
    const size_t psm = ((size_t)kBdD * sd + (size_t)G * kBdD) * 4;
    CRS_TRY_CUDA(cudaFuncSetAttribute(query_project_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)psm));
    {
        ProfScope _ps(K_BLK_SCORE, s);
        _ps.more(1);                              // projection + scorer
        query_project_split_kernel<<<n_sh, 256, psm, s>>>(static_cast<const __nv_bfloat16 *>(Q), U, P, n_sh,
                                                         p->b.n_kv, p->n_q, G, sd);
        block_score_fp4_tc_kernel<<<grid, kFtThreads, smem_s, s>>>(tmu, tq, tp, fa);
    }
    CRS_CHECK_LAUNCH();
    return launch_block_pick(p, sc, tok_idx, tok_count, s);
}
