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

__global__ void __launch_bounds__(kBdWarps * 32)
block_describe_kernel(const __nv_bfloat16 *__restrict__ K, float *__restrict__ mu_out,
                      float *__restrict__ xi_out, int n_kv, int T, int L, int rank, int blk_begin,
                      int n_blk, int n_full) {
    extern __shared__ __align__(16) unsigned char bd_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    BdWarpSmem &S = reinterpret_cast<BdWarpSmem *>(bd_smem)[warp];
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
    // Gram row `lane`: G[i][j] = (1/L) sum_d Kt[i][d] Kt[j][d]
    if (lane < L) {
        float grow[kBdMaxL];
#pragma unroll
        for (int j = 0; j < kBdMaxL; ++j) grow[j] = 0.0f;
        for (int d = 0; d < kBdD; ++d) {
            const float md = S.mu[d];
            const float ki = __bfloat162float(S.k[lane][d]) - md;
#pragma unroll
            for (int j = 0; j < kBdMaxL; ++j)
                if (j < L) grow[j] = fmaf(ki, __bfloat162float(S.k[j][d]) - md, grow[j]);
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
        float *xo = xi_out + (dbase * rank + e) * kBdD;
        if (e >= L || bi >= L) {
            for (int d = lane; d < kBdD; d += 32) xo[d] = 0.0f;
            continue;
        }
        for (int d = lane; d < kBdD; d += 32) {
            const float md = S.mu[d];
            float acc = 0.0f;
            for (int r = 0; r < L; ++r) acc = fmaf(__bfloat162float(S.k[r][d]) - md, S.v[r][bi], acc);
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

__global__ void __launch_bounds__(kBsThreads)
block_score_kernel(const __nv_bfloat16 *__restrict__ Q, const float *__restrict__ mu,
                   const float *__restrict__ xi, float *__restrict__ sc_out, int n_kv, int n_q,
                   int G, int rank, int n_full, float scale) {
    extern __shared__ float bs_smem[];
    const int nbt = kBsThreads / G;             // blocks per CTA
    const int DP = kBdD + 1;
    float *sq = bs_smem;                        // [G][DP]
    float *sd = sq + G * DP;                    // [nbt][(1+rank)][DP]
    const int sh = blockIdx.y, seq = sh / n_kv, h = sh - seq * n_kv;
    const int b0 = blockIdx.x * nbt;
    const int nb = min(nbt, n_full - b0);
    for (int e = threadIdx.x; e < G * kBdD; e += kBsThreads) {
        const int g = e / kBdD, d = e - g * kBdD;
        sq[g * DP + d] = scale * __bfloat162float(Q[((size_t)seq * n_q + h * G + g) * kBdD + d]);
    }
    const int rows = 1 + rank;
    for (int e = threadIdx.x; e < nb * rows * kBdD; e += kBsThreads) {
        const int bl = e / (rows * kBdD), rem = e - bl * rows * kBdD;
        const int rr = rem / kBdD, d = rem - rr * kBdD;
        const size_t blk = (size_t)sh * n_full + b0 + bl;
        sd[(bl * rows + rr) * DP + d] =
            (rr == 0) ? mu[blk * kBdD + d] : xi[(blk * rank + (rr - 1)) * kBdD + d];
    }
    __syncthreads();
    const int bl = threadIdx.x / G, g = threadIdx.x - bl * G;
    if (bl >= nb) return;
    const float *q = sq + g * DP;
    const float *dsc = sd + bl * rows * DP;
    float lin = 0.0f;
    for (int d = 0; d < kBdD; ++d) lin = fmaf(q[d], dsc[d], lin);
    float quad = 0.0f;
    for (int e = 0; e < rank; ++e) {
        float p = 0.0f;
        const float *x = dsc + (1 + e) * DP;
        for (int d = 0; d < kBdD; ++d) p = fmaf(q[d], x[d], p);
        quad = fmaf(p, p, quad);
    }
    sc_out[((size_t)sh * G + g) * n_full + b0 + bl] = fmaf(0.5f, quad, lin);
}

// K9a specialised for G query heads and rank R, streaming the descriptors
// through shared memory.  A CTA owns a contiguous range of blocks of one
// (sequence, KV head); chunks of 16 blocks (mu 8 KB + xi 32 KB, contiguous in
// HBM) arrive by two bulk copies each into a 2-stage ring, so one chunk is in
// flight while the previous is scored (two CTAs per SM).  Eight lanes share a block: lane s reads
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
                       int n_full, int blocks_per_cta, float scale) {
    extern __shared__ __align__(128) unsigned char bs_raw[];
    BsSmem<G, R> &S = *reinterpret_cast<BsSmem<G, R> *>(bs_raw);
    const int sh = blockIdx.y, seq = sh / n_kv, h = sh - seq * n_kv;
    const int b_lo = blockIdx.x * blocks_per_cta;
    const int b_hi = min(n_full, b_lo + blocks_per_cta);
    if (b_lo >= b_hi) return;
    const int n_chunks = ceil_div(b_hi - b_lo, kBsChunk);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *mu_sh = mu + (size_t)sh * n_full * kBdD;
    const float *xi_sh = xi + (size_t)sh * n_full * R * kBdD;
    auto issue = [&](int c) {                      // one thread
        const int st = c % kBsStages;
        const int b0 = b_lo + c * kBsChunk;
        const int nb = min(kBsChunk, b_hi - b0);
        const uint32_t mb = (uint32_t)nb * kBdD * 4, xb = mb * R;
        tc::mbar_arrive_expect_tx(&S.full[st], mb + xb);
        tc::bulk_load(&S.mu[st][0][0], mu_sh + (size_t)b0 * kBdD, mb, &S.full[st]);
        tc::bulk_load(&S.xi[st][0][0][0], xi_sh + (size_t)b0 * R * kBdD, xb, &S.full[st]);
    };
    if (tid == 0) {
        for (int st = 0; st < kBsStages; ++st) tc::mbar_init(&S.full[st], 1);
        tc::mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0)
        for (int c = 0; c < min(kBsStages, n_chunks); ++c) issue(c);
    for (int e = tid; e < G * kBdD; e += blockDim.x) {
        const int g = e / kBdD, d = e - g * kBdD;
        S.sq[g][d] = scale * __bfloat162float(Q[((size_t)seq * n_q + h * G + g) * kBdD + d]);
    }
    __syncthreads();
    const int sub = lane & 7, grp = warp * 4 + (lane >> 3);     // block of the chunk
    const float4 *q4 = reinterpret_cast<const float4 *>(&S.sq[0][0]);
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kBsStages;
        ok = ok && tc::mbar_wait_bounded(&S.full[st], (c / kBsStages) & 1, kBsWaitNs, K_BLK_SCORE, 1);
        if (__syncthreads_or(!ok)) break;
        const int b = b_lo + c * kBsChunk + grp;
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
constexpr int kPickT = 256;

// One CTA per (sequence, KV head).  Warp g takes query heads g, g + 8, ...:
// the head's softmax over blocks (max and sum by shuffles) goes to its own
// shared row, so the group sum is formed in a fixed order; warp 0 then selects
// the top blocks exactly (4 radix passes over order-preserving keys, no block
// barriers) and lists them in block order (ties: smaller block first).
__global__ void __launch_bounds__(kPickT)
block_pick_kernel(const float *__restrict__ sc, int32_t *__restrict__ tok, int32_t *__restrict__ cnt,
                  int G, int n_full, int L, int T, int top, int window, int cap) {
    extern __shared__ __align__(16) unsigned char bp_smem[];
    float *prob = reinterpret_cast<float *>(bp_smem);                  // [G][n_full]
    uint32_t *keyv = reinterpret_cast<uint32_t *>(prob + (size_t)G * n_full);   // [n_full]
    int *sel = reinterpret_cast<int *>(keyv + n_full);                  // [top] kept blocks
    int *tstart = sel + top;                                            // [top] output offsets
    __shared__ uint32_t hist[256];
    __shared__ int bc[2];
    const int sh = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int g = warp; g < G; g += kPickT / 32) {
        const float *s = sc + ((size_t)sh * G + g) * n_full;
        float *pr = prob + (size_t)g * n_full;
        float m = -INFINITY;
        for (int b = lane; b < n_full; b += 32) m = fmaxf(m, s[b]);
        m = warp_max(m);
        float z = 0.0f;
        for (int b = lane; b < n_full; b += 32) {
            const float e = __expf(s[b] - m);
            pr[b] = e;
            z += e;
        }
        z = warp_sum(z);
        const float iz = 1.0f / z;
        for (int b = lane; b < n_full; b += 32) pr[b] *= iz;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < n_full; b += kPickT) {
        float acc = 0.0f;
        for (int g = 0; g < G; ++g) acc += prob[(size_t)g * n_full + b];
        keyv[b] = score_key(acc);
    }
    __syncthreads();
    const int wstart = max(0, T - window);
    if (warp == 0) {
        // exact top `top` by (score desc, block asc)
        const int k = min(top, n_full);
        uint32_t prefix = 0u, mask = 0u;
        int need = k;
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
#pragma unroll
            for (int u = 0; u < 8; ++u) hist[lane * 8 + u] = 0u;
            __syncwarp();
            for (int b = lane; b < n_full; b += 32) {
                const uint32_t kk = keyv[b];
                if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & 255u], 1u);
            }
            __syncwarp();
            const int bin = warp_top_bin(hist, need);
            prefix |= (uint32_t)bin << shift;
            mask |= 0xffu << shift;
            __syncwarp();
        }
        const uint32_t Tk = prefix;
        // compaction in block order: block b = j * 32 + lane
        int out = 0, eq_seen = 0, tok_pos = 0;
        for (int j0 = 0; j0 < n_full; j0 += 32) {
            const int b = j0 + lane;
            const uint32_t kk = b < n_full ? keyv[b] : 0u;
            const bool eq = b < n_full && kk == Tk;
            const unsigned be = __ballot_sync(0xffffffffu, eq);
            const bool take = (b < n_full && kk > Tk) ||
                              (eq && eq_seen + __popc(be & ((1u << lane) - 1u)) < need);
            const unsigned bt = __ballot_sync(0xffffffffu, take);
            // tokens of block b that lie before the window
            const int nt = take ? min(L, max(0, wstart - b * L)) : 0;
            int incl = nt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += x;
            }
            if (take) {
                const int slot = out + __popc(bt & ((1u << lane) - 1u));
                sel[slot] = b;
                tstart[slot] = tok_pos + incl - nt;
            }
            out += __popc(bt);
            eq_seen += __popc(be);
            tok_pos += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            bc[0] = out;
            bc[1] = tok_pos;
        }
    }
    __syncthreads();
    // token list: kept blocks' positions before the window (blocks ascending),
    // then the window [wstart, T)
    const int n_sel = bc[0], nblk_tok = bc[1];
    int32_t *to = tok + (size_t)sh * cap;
    for (int e = threadIdx.x; e < n_sel * L; e += kPickT) {
        const int i = e / L, r = e - i * L;
        const int b = sel[i];
        if (b * L + r < wstart) to[tstart[i] + r] = b * L + r;
    }
    const int nwin = T - wstart;
    for (int i = threadIdx.x; i < nwin; i += kPickT) to[nblk_tok + i] = wstart + i;
    const int total = nblk_tok + nwin;
    for (int i = total + threadIdx.x; i < cap; i += kPickT) to[i] = -1;
    if (threadIdx.x == 0) cnt[sh] = total;
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

// E2M1 code (4 bits) -> float: index 0/1 -> 0/0.5, else (1 + m/2) 2^(e-1)
__device__ __forceinline__ float e2m1_value(uint32_t c) {
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    const uint32_t mag = e ? (((126u + e) << 23) | (m << 22)) : (m ? 0x3f000000u : 0u);
    return __uint_as_float(mag | ((c & 8u) << 28));
}

// K9a on compressed descriptors: the FP4 counterpart of block_score_tma_kernel.
// A chunk of 16 blocks is 4 KB of bf16 means, 4 KB of FP4 codes and 256 B of
// scales (three bulk copies); lane s of a block's 8-lane group covers dims
// [8s, 8s + 8) and [64 + 8s, 64 + 8s + 8).  Projections are formed on the code
// values and scaled once per vector.
constexpr int kBqChunk = 16;
template <int G, int R>
struct BqSmem {
    __nv_bfloat16 mu[kBsStages][kBqChunk][kBdD];
    uint8_t xi[kBsStages][kBqChunk][R][kBdD / 2];
    float scale[kBsStages][kBqChunk][R];
    float sq[G][kBdD];
    uint64_t full[kBsStages];
};

template <int G, int R>
__global__ void __launch_bounds__(8 * kBqChunk)
block_score_fp4_kernel(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ mu16,
                       const uint8_t *__restrict__ xi4, const float *__restrict__ xi_scale,
                       float *__restrict__ sc_out, int n_kv, int n_q, int n_full, int blocks_per_cta,
                       float scale) {
    extern __shared__ __align__(128) unsigned char bq_raw[];
    BqSmem<G, R> &S = *reinterpret_cast<BqSmem<G, R> *>(bq_raw);
    const int sh = blockIdx.y, seq = sh / n_kv, h = sh - seq * n_kv;
    const int b_lo = blockIdx.x * blocks_per_cta;
    const int b_hi = min(n_full, b_lo + blocks_per_cta);
    if (b_lo >= b_hi) return;
    const int n_chunks = ceil_div(b_hi - b_lo, kBqChunk);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t blk0 = (size_t)sh * n_full;
    auto issue = [&](int c) {                      // one thread
        const int st = c % kBsStages;
        const size_t b0 = blk0 + b_lo + (size_t)c * kBqChunk;
        const int nb = min(kBqChunk, b_hi - (b_lo + c * kBqChunk));
        const uint32_t mb = (uint32_t)nb * kBdD * 2, xb = (uint32_t)nb * R * (kBdD / 2);
        const uint32_t sb = (uint32_t)((nb * R * 4 + 15) & ~15);
        tc::mbar_arrive_expect_tx(&S.full[st], mb + xb + sb);
        tc::bulk_load(&S.mu[st][0][0], mu16 + b0 * kBdD, mb, &S.full[st]);
        tc::bulk_load(&S.xi[st][0][0][0], xi4 + b0 * R * (kBdD / 2), xb, &S.full[st]);
        tc::bulk_load(&S.scale[st][0][0], xi_scale + b0 * R, sb, &S.full[st]);
    };
    if (tid == 0) {
        for (int st = 0; st < kBsStages; ++st) tc::mbar_init(&S.full[st], 1);
        tc::mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0)
        for (int c = 0; c < min(kBsStages, n_chunks); ++c) issue(c);
    for (int e = tid; e < G * kBdD; e += blockDim.x) {
        const int g = e / kBdD, d = e - g * kBdD;
        S.sq[g][d] = scale * __bfloat162float(Q[((size_t)seq * n_q + h * G + g) * kBdD + d]);
    }
    __syncthreads();
    const int sub = lane & 7, grp = warp * 4 + (lane >> 3);
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kBsStages;
        ok = ok && tc::mbar_wait_bounded(&S.full[st], (c / kBsStages) & 1, kBsWaitNs, K_BLK_SCORE, 2);
        if (__syncthreads_or(!ok)) break;
        const int b = b_lo + c * kBqChunk + grp;
        {   // every lane computes (the group shuffles need all 32); invalid blocks only skip the store
            float lin[G], pr[G][R];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                lin[g] = 0.0f;
#pragma unroll
                for (int e = 0; e < R; ++e) pr[g][e] = 0.0f;
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int d0 = half * 64 + sub * 8;              // 8 dims of this lane
                const uint4 mraw = *reinterpret_cast<const uint4 *>(&S.mu[st][grp][d0]);
                const __nv_bfloat162 *m2 = reinterpret_cast<const __nv_bfloat162 *>(&mraw);
                float mv[8];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 f = __bfloat1622float2(m2[t]);
                    mv[2 * t] = f.x;
                    mv[2 * t + 1] = f.y;
                }
                float cv[R][8];
#pragma unroll
                for (int e = 0; e < R; ++e) {
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(&S.xi[st][grp][e][d0 / 2]);
#pragma unroll
                    for (int t = 0; t < 8; ++t) cv[e][t] = e2m1_value((w >> (4 * t)) & 15u);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 q0 = *reinterpret_cast<const float4 *>(&S.sq[g][d0]);
                    const float4 q1 = *reinterpret_cast<const float4 *>(&S.sq[g][d0 + 4]);
                    const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        lin[g] = fmaf(qv[t], mv[t], lin[g]);
#pragma unroll
                        for (int e = 0; e < R; ++e) pr[g][e] = fmaf(qv[t], cv[e][t], pr[g][e]);
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
                    for (int e = 0; e < R; ++e) {
                        const float pe = pr[g][e] * S.scale[st][grp][e];
                        quad = fmaf(pe, pe, quad);
                    }
                    sc_out[((size_t)sh * G + g) * n_full + b] = fmaf(0.5f, quad, lin[g]);
                }
            }
        }
        __syncthreads();                                  // stage st is read: refill it
        if (tid == 0 && c + kBsStages < n_chunks) issue(c + kBsStages);
    }
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
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_describe_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    dim3 grid(ceil_div(n_blk, kBdWarps), p->n_seq * p->n_kv);
    {
        ProfScope _ps(K_BLK_DESCRIBE, s);
        block_describe_kernel<<<grid, kBdWarps * 32, smem, s>>>(
            static_cast<const __nv_bfloat16 *>(K), mu, xi, p->n_kv, p->T, p->L, p->rank, p->blk_begin,
            n_blk, n_full);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

static int bs_validate(const crs_block_sel_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    crs_block_params b = p->b;
    b.blk_begin = 0;
    b.blk_end = 0;
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
    if (!Q || !mu || !xi || !tok_idx || !tok_count) return CRS_ERR_INVALID_ARG;
    const size_t need = crs_block_select_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int G = p->n_q / p->b.n_kv;
    const int n_full = p->b.T / p->b.L;
    const int nbt = kBsThreads / G;
    const size_t smem_a = ((size_t)G * (kBdD + 1) + (size_t)nbt * (1 + p->b.rank) * (kBdD + 1)) * 4;
    if (smem_a > 227 * 1024) return CRS_ERR_UNSUPPORTED;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a));
    float *sc = static_cast<float *>(ws);
    if (G == 8 && p->b.rank == 4) {
        const int n_sh = p->b.n_seq * p->b.n_kv;
        const int per_sh = max(1, min(ceil_div(n_full, kBsChunk), ceil_div(148 * 4, n_sh)));
        const int bpc = ceil_div(ceil_div(n_full, per_sh), kBsChunk) * kBsChunk;
        const size_t smem_s = sizeof(BsSmem<8, 4>);
        CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_tma_kernel<8, 4>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s));
        dim3 gf(ceil_div(n_full, bpc), n_sh);
        ProfScope _ps(K_BLK_SCORE, s);
        block_score_tma_kernel<8, 4><<<gf, kBsThreadsT, smem_s, s>>>(static_cast<const __nv_bfloat16 *>(Q), mu, xi,
                                                            sc, p->b.n_kv, p->n_q, n_full, bpc, p->scale);
    } else {
    dim3 ga(ceil_div(n_full, nbt), p->b.n_seq * p->b.n_kv);
    {
        ProfScope _ps(K_BLK_SCORE, s);
        block_score_kernel<<<ga, kBsThreads, smem_a, s>>>(static_cast<const __nv_bfloat16 *>(Q), mu, xi,
                                                          sc, p->b.n_kv, p->n_q, G, p->b.rank, n_full,
                                                          p->scale);
    }
    }
    CRS_CHECK_LAUNCH();
    const int cap = p->top_blocks * p->b.L + p->window;
    const size_t smem_b = ((size_t)G + 1) * n_full * 4 + (size_t)p->top_blocks * 8;
    if (smem_b > 200 * 1024) return CRS_ERR_UNSUPPORTED;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_pick_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b));
    {
        ProfScope _ps(K_BLK_PICK, s);
        block_pick_kernel<<<p->b.n_seq * p->b.n_kv, kPickT, smem_b, s>>>(
            sc, tok_idx, tok_count, G, n_full, p->b.L, p->b.T, p->top_blocks, p->window, cap);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
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
    const int G = p->n_q / p->b.n_kv;
    if (G != 8 || p->b.rank != 4) return CRS_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(mu16) | reinterpret_cast<uintptr_t>(xi4) |
         reinterpret_cast<uintptr_t>(xi_scale)) & 15)
        return CRS_ERR_INVALID_ARG;
    const size_t need = crs_block_select_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int n_full = p->b.T / p->b.L;
    float *sc = static_cast<float *>(ws);
    const int n_sh = p->b.n_seq * p->b.n_kv;
    // every block's slice of the three arrays (256 B, 256 B, 16 B) starts on a
    // 16-byte boundary, as the bulk copies require
    const int per_sh = max(1, min(ceil_div(n_full, kBqChunk), ceil_div(148 * 4, n_sh)));
    const int bpc = ceil_div(ceil_div(n_full, per_sh), kBqChunk) * kBqChunk;
    const size_t smem_s = sizeof(BqSmem<8, 4>);
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_score_fp4_kernel<8, 4>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_s));
    {
        ProfScope _ps(K_BLK_SCORE, s);
        block_score_fp4_kernel<8, 4><<<dim3(ceil_div(n_full, bpc), n_sh), 8 * kBqChunk, smem_s, s>>>(
            static_cast<const __nv_bfloat16 *>(Q), static_cast<const __nv_bfloat16 *>(mu16), xi4,
            xi_scale, sc, p->b.n_kv, p->n_q, n_full, bpc, p->scale);
    }
    CRS_CHECK_LAUNCH();
    const int cap = p->top_blocks * p->b.L + p->window;
    const size_t smem_b = ((size_t)G + 1) * n_full * 4 + (size_t)p->top_blocks * 8;
    if (smem_b > 200 * 1024) return CRS_ERR_UNSUPPORTED;
    CRS_TRY_CUDA(cudaFuncSetAttribute(block_pick_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b));
    {
        ProfScope _ps(K_BLK_PICK, s);
        block_pick_kernel<<<n_sh, kPickT, smem_b, s>>>(sc, tok_idx, tok_count, G, n_full, p->b.L,
                                                       p->b.T, p->top_blocks, p->window, cap);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}
