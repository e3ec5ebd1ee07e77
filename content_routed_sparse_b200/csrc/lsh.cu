// LSH routing and chunked LSH attention (Reformer-style), sm_100a.
//
// [P1] PaperTrace 2.1.1 "哈希与聚类" §2.1 Eq.(4) (bucket = argmax [xR; -xR]),
// §2.1-2.2 (stable sort on (bucket, position) -> pi, pi^-1; chunks of m slots
// attend to themselves and the previous chunk; causal and padding masks on
// original positions), "重复候选和归一化" (a pair counts once, in its first
// round; rounds merge by log-sum-exp weights).
#include <math.h>

#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace crs {

// --------------------------------------------------------------------------
// K1: hash.  One thread per (token, round).  R_{h,r} and a tile of 128 token
// rows are staged in shared memory; every u_k is a chain of fp32 FMAs over
// the head dim in increasing index order (bit-reproducible bucket ids).
// --------------------------------------------------------------------------
constexpr int kHashTok = 128;

template <typename T>
__global__ void __launch_bounds__(kHashTok) lsh_hash_kernel(const T *__restrict__ X,
                                                            const float *__restrict__ R,
                                                            int32_t *__restrict__ bucket, int H,
                                                            int n, int d, int nb, int rounds) {
    extern __shared__ float sm[];
    const int half = nb / 2;
    const int bh = blockIdx.z, r = blockIdx.y, h = bh % H;
    float *Rs = sm;               // [d][half]
    float *Xs = sm + d * half;    // [kHashTok][d+1]
    const float *Rg = R + ((size_t)h * rounds + r) * (size_t)d * half;
    for (int e = threadIdx.x; e < d * half; e += blockDim.x) Rs[e] = Rg[e];
    const int i0 = blockIdx.x * kHashTok;
    for (int e = threadIdx.x; e < kHashTok * d; e += blockDim.x) {
        const int t = e / d, k = e - t * d, i = i0 + t;
        Xs[t * (d + 1) + k] = (i < n) ? to_f32(X[((size_t)bh * n + i) * d + k]) : 0.0f;
    }
    __syncthreads();
    const int i = i0 + threadIdx.x;
    if (i >= n) return;
    const float *x = Xs + threadIdx.x * (d + 1);
    float bp = 0.0f, bn = 0.0f;
    int ap = 0, an = 0;
    for (int k0 = 0; k0 < half; k0 += 32) {
        float u[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) u[j] = 0.0f;
        for (int t = 0; t < d; ++t) {
            const float xv = x[t];
            const float *rr = Rs + t * half + k0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (k0 + j < half) u[j] = __fmaf_rn(xv, rr[j], u[j]);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int k = k0 + j;
            if (k < half) {
                if (k == 0 || u[j] > bp) { bp = u[j]; ap = k; }
                const float nu = -u[j];
                if (k == 0 || nu > bn) { bn = nu; an = k; }
            }
        }
    }
    // first maximum of [u ; -u] in index order: the +u group precedes the -u group
    const int arg = (bp >= bn) ? ap : half + an;
    bucket[((size_t)bh * rounds + r) * n + i] = arg;
}

// K1 specialised for a compile-time head dim D and half-width HALF: the token
// row lives in registers, R_{h,r} is read from shared memory as broadcast
// float4s; the FMA chain of every u_k is the same as above (index order from
// 0), so the bucket ids are identical.
template <typename T, int D, int HALF>
__global__ void __launch_bounds__(kHashTok) lsh_hash_fixed_kernel(const T *__restrict__ X,
                                                                  const float *__restrict__ R,
                                                                  int32_t *__restrict__ bucket,
                                                                  int H, int n, int rounds) {
    __shared__ __align__(16) float Rs[D * HALF];
    const int bh = blockIdx.z, h = bh % H;
    const int i = blockIdx.x * kHashTok + threadIdx.x;
    float x[D];
    if (i < n) {
        const T *xr = X + ((size_t)bh * n + i) * D;
#pragma unroll
        for (int t = 0; t < D; ++t) x[t] = to_f32(xr[t]);
    }
    for (int r = blockIdx.y; r < rounds; r += gridDim.y) {
        __syncthreads();
        const float4 *Rg = reinterpret_cast<const float4 *>(R + ((size_t)h * rounds + r) * D * HALF);
        for (int e = threadIdx.x; e < D * HALF / 4; e += kHashTok)
            reinterpret_cast<float4 *>(Rs)[e] = Rg[e];
        __syncthreads();
        if (i >= n) continue;
        float bp = 0.0f, bn = 0.0f;
        int ap = 0, an = 0;
#pragma unroll
        for (int k0 = 0; k0 < HALF; k0 += 32) {
            constexpr int W = HALF < 32 ? HALF : 32;
            // u_k pairs (k, k + 1) advance together with one paired fused multiply-add:
            // each lane rounds exactly like __fmaf_rn, in the same index order
            uint64_t u2[W / 2];
#pragma unroll
            for (int j = 0; j < W / 2; ++j) u2[j] = 0ull;
#pragma unroll
            for (int t = 0; t < D; ++t) {
                const uint64_t xx = f32x2_pack(x[t], x[t]);
                const ulonglong2 *rr = reinterpret_cast<const ulonglong2 *>(Rs + t * HALF + k0);
#pragma unroll
                for (int j4 = 0; j4 < W / 4; ++j4) {
                    const ulonglong2 rv = rr[j4];
                    u2[2 * j4] = f32x2_fma(xx, rv.x, u2[2 * j4]);
                    u2[2 * j4 + 1] = f32x2_fma(xx, rv.y, u2[2 * j4 + 1]);
                }
            }
            float u[W];
#pragma unroll
            for (int j = 0; j < W / 2; ++j) f32x2_unpack(u2[j], u[2 * j], u[2 * j + 1]);
#pragma unroll
            for (int j = 0; j < W; ++j) {
                const int k = k0 + j;
                if (k == 0 || u[j] > bp) { bp = u[j]; ap = k; }
                const float nu = -u[j];
                if (k == 0 || nu > bn) { bn = nu; an = k; }
            }
        }
        bucket[((size_t)bh * rounds + r) * n + i] = (bp >= bn) ? ap : HALF + an;
    }
}

// K1 for bf16 rows, two tokens per thread (i and i + 128 of a 256-token tile):
// each R value read from shared memory feeds both tokens, halving the
// shared-memory loads per FMA (the limit of the one-token kernel).  Rows stay
// packed as bf16 pairs in registers and are upcast exactly when used; the FMA
// chain of every u_k is unchanged (index order from 0, one rounding per step),
// so the bucket ids are identical.
constexpr int kHash2Tok = 2 * kHashTok;

template <int D, int HALF>
__global__ void __launch_bounds__(kHashTok) lsh_hash_bf16x2_kernel(const __nv_bfloat16 *__restrict__ X,
                                                                   const float *__restrict__ R,
                                                                   int32_t *__restrict__ bucket,
                                                                   int H, int n, int rounds) {
    __shared__ __align__(16) float Rs[D * HALF];
    const int bh = blockIdx.z, h = bh % H;
    const int i0 = blockIdx.x * kHash2Tok + threadIdx.x, i1 = i0 + kHashTok;
    uint32_t xa[D / 2], xb[D / 2];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
        uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
        if (i0 < n) va = reinterpret_cast<const uint4 *>(X + ((size_t)bh * n + i0) * D)[c];
        if (i1 < n) vb = reinterpret_cast<const uint4 *>(X + ((size_t)bh * n + i1) * D)[c];
        xa[4 * c] = va.x; xa[4 * c + 1] = va.y; xa[4 * c + 2] = va.z; xa[4 * c + 3] = va.w;
        xb[4 * c] = vb.x; xb[4 * c + 1] = vb.y; xb[4 * c + 2] = vb.z; xb[4 * c + 3] = vb.w;
    }
    for (int r = 0; r < rounds; ++r) {
        __syncthreads();
        const float4 *Rg = reinterpret_cast<const float4 *>(R + ((size_t)h * rounds + r) * D * HALF);
        for (int e = threadIdx.x; e < D * HALF / 4; e += kHashTok)
            reinterpret_cast<float4 *>(Rs)[e] = Rg[e];
        __syncthreads();
        float bp[2] = {0.0f, 0.0f}, bn[2] = {0.0f, 0.0f};
        int ap[2] = {0, 0}, an[2] = {0, 0};
#pragma unroll 1
        for (int k0 = 0; k0 < HALF; k0 += 16) {
            constexpr int W = HALF < 16 ? HALF : 16;
            uint64_t ua[W / 2], ub[W / 2];
#pragma unroll
            for (int j = 0; j < W / 2; ++j) ua[j] = ub[j] = 0ull;
#pragma unroll
            for (int t = 0; t < D; ++t) {
                // exact bf16 -> fp32: the 16 bits become the high half of the float
                const uint32_t wa = xa[t >> 1], wb = xb[t >> 1];
                const float fa = __uint_as_float((t & 1) ? (wa & 0xffff0000u) : (wa << 16));
                const float fb = __uint_as_float((t & 1) ? (wb & 0xffff0000u) : (wb << 16));
                const uint64_t pa = f32x2_pack(fa, fa), pb = f32x2_pack(fb, fb);
                const ulonglong2 *rr = reinterpret_cast<const ulonglong2 *>(Rs + t * HALF + k0);
#pragma unroll
                for (int j4 = 0; j4 < W / 4; ++j4) {
                    const ulonglong2 rv = rr[j4];
                    ua[2 * j4] = f32x2_fma(pa, rv.x, ua[2 * j4]);
                    ua[2 * j4 + 1] = f32x2_fma(pa, rv.y, ua[2 * j4 + 1]);
                    ub[2 * j4] = f32x2_fma(pb, rv.x, ub[2 * j4]);
                    ub[2 * j4 + 1] = f32x2_fma(pb, rv.y, ub[2 * j4 + 1]);
                }
            }
#pragma unroll
            for (int j = 0; j < W / 2; ++j) {
                float u[2][2];
                f32x2_unpack(ua[j], u[0][0], u[0][1]);
                f32x2_unpack(ub[j], u[1][0], u[1][1]);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int k = k0 + 2 * j + e;
#pragma unroll
                    for (int z = 0; z < 2; ++z) {
                        if (k == 0 || u[z][e] > bp[z]) { bp[z] = u[z][e]; ap[z] = k; }
                        const float nu = -u[z][e];
                        if (k == 0 || nu > bn[z]) { bn[z] = nu; an[z] = k; }
                    }
                }
            }
        }
        int32_t *bo = bucket + ((size_t)bh * rounds + r) * n;
        if (i0 < n) bo[i0] = (bp[0] >= bn[0]) ? ap[0] : HALF + an[0];
        if (i1 < n) bo[i1] = (bp[1] >= bn[1]) ? ap[1] : HALF + an[1];
    }
}

// --------------------------------------------------------------------------
// K2: stable counting sort of one (b, h, round) segment per 8-CTA cluster.
// Histogram -> exclusive scan (bucket bases) -> tiles of blockDim positions
// in increasing order; inside a tile, the rank of a position among equal
// buckets comes from __match_any_sync within the warp plus the counts of
// earlier warps, so equal buckets keep position order (the (bucket, pos) key).
// --------------------------------------------------------------------------
constexpr int kSortThreads = 512;

// The 8 CTAs of a cluster split one segment into 8
// contiguous position ranges.  Each counts its range's buckets in shared
// memory; after a cluster barrier every CTA reads the other CTAs' counts
// through distributed shared memory, so the slot of the first position of
// bucket b in range p is (positions in buckets < b) + (positions of bucket b
// in ranges < p).  No global scratch is needed.
constexpr int kSortCluster = 8;

__global__ void __cluster_dims__(kSortCluster, 1, 1) __launch_bounds__(kSortThreads)
lsh_sort_cluster_kernel(const int32_t *__restrict__ bucket, int32_t *__restrict__ perm,
                        int32_t *__restrict__ inv_perm, int n, int nb) {
    extern __shared__ int smc[];
    constexpr int NW = kSortThreads / 32;
    int *hist = smc;               // [nb] counts of this range (read by the cluster)
    int *base = hist + nb;         // [nb]
    int *running = base + nb;      // [nb]
    int *wcnt = running + nb;      // [NW][nb]
    __shared__ int scan_w[NW + 1];
    cg::cluster_group cluster = cg::this_cluster();
    const int part = (int)cluster.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t seg = blockIdx.y;
    const int len = (n + kSortCluster - 1) / kSortCluster;
    const int p0 = min(n, part * len), p1 = min(n, p0 + len);
    const int32_t *bk = bucket + seg * n;
    int32_t *pm = perm + seg * n;
    int32_t *ip = inv_perm + seg * n;
    for (int e = tid; e < nb; e += kSortThreads) { hist[e] = 0; running[e] = 0; }
    for (int e = tid; e < NW * nb; e += kSortThreads) wcnt[e] = 0;
    __syncthreads();
    for (int i = p0 + tid; i < p1; i += kSortThreads) {
        const int b = bk[i];
        if (b >= 0 && b < nb) atomicAdd(&hist[b], 1);
        else raise_error(CRS_DEVERR_INDEX);
    }
    cluster.sync();
    // base[b] = sum over ranges of buckets < b, plus bucket b in earlier ranges
    for (int b0 = 0; b0 < nb; b0 += kSortThreads) {
        const int b = b0 + tid;
        int tot = 0, before = 0;
        if (b < nb) {
            for (int q = 0; q < kSortCluster; ++q) {
                const int c = *cluster.map_shared_rank(hist + b, q);
                tot += c;
                if (q < part) before += c;
            }
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) scan_w[warp] = incl;
        __syncthreads();
        if (tid == 0) {
            int acc = b0 == 0 ? 0 : scan_w[NW];
            for (int w = 0; w < NW; ++w) { const int c = scan_w[w]; scan_w[w] = acc; acc += c; }
            scan_w[NW] = acc;
        }
        __syncthreads();
        if (b < nb) base[b] = scan_w[warp] + incl - tot + before;
        __syncthreads();
    }
    cluster.sync();                // every CTA has read the counts it needs
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int t0 = p0; t0 < p1; t0 += kSortThreads) {
        const int i = t0 + tid;
        int b = (i < p1) ? bk[i] : -1;
        if (b >= nb) b = -1;
        const bool valid = b >= 0;
        const unsigned active = __ballot_sync(0xffffffffu, valid);
        int rank = 0, cnt = 0;
        if (valid) {
            const unsigned peers = __match_any_sync(active, b);
            rank = __popc(peers & lt_mask);
            cnt = __popc(peers);
            if (rank == 0) wcnt[warp * nb + b] = cnt;
        }
        __syncthreads();
        if (valid) {
            int off = 0;
            for (int w = 0; w < warp; ++w) off += wcnt[w * nb + b];
            const int slot = base[b] + running[b] + off + rank;
            pm[slot] = i;
            ip[i] = slot;
        }
        __syncthreads();
        if (valid && rank == 0) { atomicAdd(&running[b], cnt); wcnt[warp * nb + b] = 0; }
        __syncthreads();
    }
}

// --------------------------------------------------------------------------
// K3 (CUDA-core path): one CTA per (chunk, round, b*h).  Keys = the slots of
// the previous and the own chunk, gathered through perm into shared memory;
// each warp owns query rows of the chunk; lanes split the keys for the
// logits, then split the head dim for P.V.  Masks per pair: same bucket in
// this round, causal / no-self / padding on original positions, and "not an
// edge of an earlier round" (a pair is counted in its first round only).
// Writes o_r (normalised, fp32) and lse_r at the ORIGINAL position.
// --------------------------------------------------------------------------
constexpr int kAttnWarps = 8;

template <typename T, int DH>
__global__ void __launch_bounds__(kAttnWarps * 32)
lsh_chunk_attn_kernel(const T *__restrict__ QK, const T *__restrict__ V,
                      const int32_t *__restrict__ bucket, const int32_t *__restrict__ perm,
                      const int32_t *__restrict__ inv_perm, const int32_t *__restrict__ valid_len,
                      float *__restrict__ o_ws, float *__restrict__ lse_ws, int H, int n, int m,
                      int rounds, int causal, int no_self, int key_norm, float scale, int q_splits) {
    extern __shared__ float smf[];
    // blockIdx.x = chunk * q_splits + split: a small problem spreads a chunk's query
    // rows over several CTAs (each gathers the chunk's key window)
    const int c = blockIdx.x / q_splits, split = blockIdx.x - c * q_splits;
    const int r = blockIdx.y, bh = blockIdx.z;
    const int b = bh / H;
    const int vl = valid_len ? valid_len[b] : n;
    const int ks0 = max(0, (c - 1) * m), ks1 = min((c + 1) * m, n);
    const int nk = ks1 - ks0;                    // <= 2m
    const int rps = (m + q_splits - 1) / q_splits;
    const int qs0 = min(c * m + split * rps, n), qs1 = min(min(c * m + m, n), qs0 + rps);
    const int KM = 2 * m;
    float *Ks = smf;                             // [KM][DH+1]
    float *Vs = Ks + KM * (DH + 1);              // [KM][DH]
    float *inv_norm = Vs + KM * DH;              // [KM]
    float *prob = inv_norm + KM;                 // [kAttnWarps][KM]
    int *kpos = reinterpret_cast<int *>(prob + kAttnWarps * KM);  // [KM]
    int *kbkt = kpos + KM;                       // [KM]
    int *pinfo = kbkt + KM;                      // [KM][kMaxRounds-1][2] (slot, bucket) of earlier rounds

    const size_t seg_r = ((size_t)bh * rounds + r) * n;
    const int32_t *pm = perm + seg_r;
    const int32_t *bkr = bucket + seg_r;
    const T *Qb = QK + (size_t)bh * n * DH;
    const T *Vb = V + (size_t)bh * n * DH;
    const int tid = threadIdx.x;
    for (int j = tid; j < nk; j += blockDim.x) {
        int pos = pm[ks0 + j];
        int bkt;
        if (pos < 0 || pos >= n) {            // a caller-supplied permutation out of range
            raise_error(CRS_DEVERR_INDEX);
            pos = 0;
            bkt = -1;                         // matches no query: the key is never used
        } else {
            bkt = bkr[pos];
        }
        kpos[j] = pos;
        kbkt[j] = bkt;
        for (int rr = 0; rr < r; ++rr) {
            const size_t seg = ((size_t)bh * rounds + rr) * n;
            pinfo[(j * (kMaxRounds - 1) + rr) * 2 + 0] = inv_perm[seg + pos];
            pinfo[(j * (kMaxRounds - 1) + rr) * 2 + 1] = bucket[seg + pos];
        }
    }
    __syncthreads();
    for (int e = tid; e < nk * DH; e += blockDim.x) {
        const int j = e / DH, k = e - j * DH;
        const size_t g = (size_t)kpos[j] * DH + k;
        Ks[j * (DH + 1) + k] = to_f32(Qb[g]);
        Vs[j * DH + k] = to_f32(Vb[g]);
    }
    __syncthreads();
    for (int j = tid; j < nk; j += blockDim.x) {
        float ss = 0.0f;
        for (int k = 0; k < DH; ++k) ss = fmaf(Ks[j * (DH + 1) + k], Ks[j * (DH + 1) + k], ss);
        inv_norm[j] = key_norm ? (ss > 0.0f ? rsqrtf(ss) : 0.0f) : 1.0f;
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    float *pw = prob + warp * KM;
    for (int qs = qs0 + warp; qs < qs1; qs += kAttnWarps) {
        const int jq = qs - ks0;                 // the query row is one of the keys
        const int pos_i = kpos[jq];
        float *o_out = o_ws + (((size_t)r * gridDim.z + bh) * n + pos_i) * DH;
        float *l_out = lse_ws + ((size_t)r * gridDim.z + bh) * n + pos_i;
        if (pos_i >= vl) {
            for (int k = lane; k < DH; k += 32) o_out[k] = 0.0f;
            if (lane == 0) *l_out = -INFINITY;
            continue;
        }
        const int bk_i = kbkt[jq];
        int ps[kMaxRounds - 1], pb[kMaxRounds - 1];
#pragma unroll
        for (int rr = 0; rr < kMaxRounds - 1; ++rr) {
            if (rr < r) {
                ps[rr] = pinfo[(jq * (kMaxRounds - 1) + rr) * 2 + 0] / m;
                pb[rr] = pinfo[(jq * (kMaxRounds - 1) + rr) * 2 + 1];
            }
        }
        float mx = -INFINITY;
        for (int j = lane; j < nk; j += 32) {
            const int pj = kpos[j];
            bool ok = (kbkt[j] == bk_i) && (pj < vl) && !(causal && pj > pos_i) &&
                      !(no_self && pj == pos_i);
#pragma unroll
            for (int rr = 0; rr < kMaxRounds - 1; ++rr) {
                if (rr < r && ok) {
                    const int cj = pinfo[(j * (kMaxRounds - 1) + rr) * 2 + 0] / m;
                    const int bj = pinfo[(j * (kMaxRounds - 1) + rr) * 2 + 1];
                    if (bj == pb[rr] && (cj == ps[rr] || cj == ps[rr] - 1)) ok = false;
                }
            }
            float s = -INFINITY;
            if (ok) {
                float dot = 0.0f;
                const float *kr = Ks + j * (DH + 1);
                const float *qr = Ks + jq * (DH + 1);
#pragma unroll 16
                for (int k = 0; k < DH; ++k) dot = fmaf(qr[k], kr[k], dot);
                s = scale * dot * inv_norm[j];
                mx = fmaxf(mx, s);
            }
            pw[j] = s;
        }
        mx = warp_max(mx);
        __syncwarp();
        if (mx == -INFINITY) {
            for (int k = lane; k < DH; k += 32) o_out[k] = 0.0f;
            if (lane == 0) *l_out = -INFINITY;
            __syncwarp();
            continue;
        }
        float sum = 0.0f;
        for (int j = lane; j < nk; j += 32) {
            const float p = (pw[j] == -INFINITY) ? 0.0f : __expf(pw[j] - mx);
            pw[j] = p;
            sum += p;
        }
        sum = warp_sum(sum);
        __syncwarp();
        float acc[DH / 32 > 0 ? DH / 32 : 1];
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) acc[u] = 0.0f;
        for (int j = 0; j < nk; ++j) {
            const float p = pw[j];
            if (p != 0.0f) {
#pragma unroll
                for (int u = 0; u < DH / 32; ++u) acc[u] = fmaf(p, Vs[j * DH + lane + 32 * u], acc[u]);
            }
        }
        const float inv = 1.0f / sum;
#pragma unroll
        for (int u = 0; u < DH / 32; ++u) o_out[lane + 32 * u] = acc[u] * inv;
        if (lane == 0) *l_out = mx + logf(sum);
        __syncwarp();
    }
}

// --------------------------------------------------------------------------
// K4: merge the rounds.  One thread per (b*h, position, 4 output dims):
//   LSE = log sum_r exp(lse_r),  O = sum_r exp(lse_r - LSE) o_r.
// Padded positions and queries with no edge in any round give 0 / -inf.
// --------------------------------------------------------------------------
template <int DH>
__device__ __forceinline__ void lsh_merge_rounds(const float *__restrict__ o_ws, const float *__restrict__ lse_ws,
                                                 float *__restrict__ O, float *__restrict__ lse_out, int BH,
                                                 int n, int rounds, int bh, int pos, int g, bool padded) {
    // every round's lse and partial output are requested before any is used
    float l[kMaxRounds];
    float4 ov[kMaxRounds];
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
        if (r < rounds) {
            l[r] = __ldcs(lse_ws + ((size_t)r * BH + bh) * n + pos);
            ov[r] = __ldcs(reinterpret_cast<const float4 *>(o_ws + (((size_t)r * BH + bh) * n + pos) * DH) + g);
        } else {
            l[r] = -INFINITY;
            ov[r] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        mx = fmaxf(mx, l[r]);
    }
    float4 *o = reinterpret_cast<float4 *>(O + ((size_t)bh * n + pos) * DH) + g;
    if (padded || mx == -INFINITY) {
        *o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (lse_out && g == 0) lse_out[(size_t)bh * n + pos] = -INFINITY;
        return;
    }
    float z = 0.0f;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) z += (r < rounds && l[r] != -INFINITY) ? __expf(l[r] - mx) : 0.0f;
    const float LSE = mx + logf(z);
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
        if (r < rounds && l[r] != -INFINITY) {
            const float wgt = __expf(l[r] - LSE);
            const float4 v = ov[r];
            acc.x = fmaf(wgt, v.x, acc.x);
            acc.y = fmaf(wgt, v.y, acc.y);
            acc.z = fmaf(wgt, v.z, acc.z);
            acc.w = fmaf(wgt, v.w, acc.w);
        }
    }
    *o = acc;
    if (lse_out && g == 0) lse_out[(size_t)bh * n + pos] = LSE;
}

template <int DH>
__global__ void lsh_combine_kernel(const float *__restrict__ o_ws, const float *__restrict__ lse_ws,
                                   const int32_t *__restrict__ valid_len, float *__restrict__ O,
                                   float *__restrict__ lse_out, int BH, int H, int n, int rounds) {
    constexpr int G4 = DH / 4;                  // float4 groups per row
    const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gt >= (long long)BH * n * G4) return;
    const int g = (int)(gt % G4);
    const long long rowi = gt / G4;
    const int bh = (int)(rowi / n), pos = (int)(rowi - (long long)bh * n);
    const int vl = valid_len ? valid_len[bh / H] : n;
    lsh_merge_rounds<DH>(o_ws, lse_ws, O, lse_out, BH, n, rounds, bh, pos, g, pos >= vl);
}

// K4 after the fixed-shift round accumulation of the tensor-core attention: O holds
// sum_j 2^(s_ij - M_i) v_j over the union of the rounds' candidates, acc_L the matching
// sum of weights, acc_M the shift M_i (log2 units); O /= L and lse = (M_i + log2 L) ln 2.
// Rows the attention kept in the per-round form (acc_M = +inf) are merged as above.
// A thread takes four 16-byte groups of one row (a quarter row for d = 64) and
// issues all of its loads before using any: the pass is bound by how many bytes
// are in flight.
template <int DH>
__global__ void lsh_finish_kernel(const float *__restrict__ o_ws, const float *__restrict__ lse_ws,
                                  const float *__restrict__ acc_L, const float *__restrict__ acc_M,
                                  const int32_t *__restrict__ valid_len, float *__restrict__ O,
                                  float *__restrict__ lse_out, int BH, int H, int n, int rounds) {
    constexpr int G4 = DH / 4;                  // float4 groups per row
    constexpr int PER = G4 >= 4 ? 4 : G4;       // groups per thread
    constexpr int TPR = G4 / PER;               // threads per row
    const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gt >= (long long)BH * n * TPR) return;
    const int g0 = (int)(gt % TPR) * PER;
    const long long rowi = gt / TPR;
    const int bh = (int)(rowi / n), pos = (int)(rowi - (long long)bh * n);
    const float m = __ldcs(acc_M + rowi);
    const float L = __ldcs(acc_L + rowi);
    float4 *o = reinterpret_cast<float4 *>(O + (size_t)rowi * DH) + g0;
    float4 v[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) v[u] = __ldcs(o + u);
    const int vl = valid_len ? valid_len[bh / H] : n;
    if (m == INFINITY) {
#pragma unroll
        for (int u = 0; u < PER; ++u)
            lsh_merge_rounds<DH>(o_ws, lse_ws, O, u == 0 ? lse_out : nullptr, BH, n, rounds, bh, pos, g0 + u,
                                 pos >= vl);
        return;
    }
    const bool has = pos < vl && L > 0.0f;
    const float inv = has ? 1.0f / L : 0.0f;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        v[u].x *= inv; v[u].y *= inv; v[u].z *= inv; v[u].w *= inv;
        o[u] = v[u];
    }
    if (lse_out && g0 == 0) lse_out[rowi] = has ? (m + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

// ------------------------------------------------------------ host side --
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static int validate_lsh(const crs_lsh_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->B < 1 || p->H < 1 || p->n < 1) return CRS_ERR_INVALID_ARG;
    if (p->d < 8 || p->d % 8 != 0 || p->d > 128) return CRS_ERR_INVALID_ARG;
    if (p->n_buckets < 2 || p->n_buckets % 2 != 0 || p->n_buckets > 1024) return CRS_ERR_INVALID_ARG;
    if (p->n_rounds < 1 || p->n_rounds > kMaxRounds) return CRS_ERR_INVALID_ARG;
    if (p->dtype != CRS_F32 && p->dtype != CRS_BF16) return CRS_ERR_INVALID_ARG;
    if ((long long)p->n_buckets * p->n > 0x7fffffffLL) return CRS_ERR_INVALID_ARG;
    return CRS_OK;
}

}  // namespace crs

using namespace crs;

extern "C" size_t crs_lsh_route_workspace_size(const crs_lsh_params *) { return 0; }

extern "C" int crs_lsh_route(const crs_lsh_params *p, const void *X, const float *R,
                             int32_t *bucket, int32_t *perm, int32_t *inv_perm, void *,
                             size_t, void *stream) {
    int st = validate_lsh(p);
    if (st) return st;
    if (!X || !R || !bucket || !perm || !inv_perm) return CRS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int half = p->n_buckets / 2;
    const size_t smem = ((size_t)p->d * half + (size_t)kHashTok * (p->d + 1)) * sizeof(float);
    if (smem > 200 * 1024) return CRS_ERR_UNSUPPORTED;
    dim3 grid(ceil_div(p->n, kHashTok), p->n_rounds, p->B * p->H);
    PFN_cuTensorMapEncodeTiled_v12000 enc = tc::tensor_map_encoder();
    const long long rows_all = (long long)p->B * p->H * p->n;
    if (p->dtype == CRS_BF16 && p->d == kHtD && half == kHtHalf && p->n_rounds <= 4 && enc &&
        !(reinterpret_cast<uintptr_t>(X) & 15) && rows_all + kHtM < 0x7fffffffLL) {
        // tensor-core filter with the exact chain as fallback (identical bucket ids)
        CUtensorMap tx;
        cuuint64_t dims[2] = {(cuuint64_t)kHtD, (cuuint64_t)rows_all};
        cuuint64_t strides[1] = {(cuuint64_t)kHtD * 2};
        cuuint32_t box[2] = {(cuuint32_t)kHtD, (cuuint32_t)kHtM};
        cuuint32_t estr[2] = {1, 1};
        if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CRS_ERR_CUDA;
        const size_t hsm = sizeof(HtSmem) + 1024;
        CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_hash_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)hsm));
        const int tpc = ht_tiles_per_cta(p->n, p->B * p->H);
        dim3 gh(ceil_div(ceil_div(p->n, kHtM), tpc), p->B * p->H);
        ProfScope _ps(K_LSH_HASH, s);
        lsh_hash_tc_kernel<<<gh, kHtThreads, hsm, s>>>(tx, R, bucket, p->H, p->n, p->n_rounds, tpc);
    } else if (p->d == 64 && (half == 32 || half == 8)) {
        // specialised kernel: one CTA per 128 tokens covers every round
        dim3 g2(ceil_div(p->n, kHashTok), 1, p->B * p->H);
        ProfScope _ps(K_LSH_HASH, s);
        if (p->dtype == CRS_F32) {
            if (half == 32)
                lsh_hash_fixed_kernel<float, 64, 32><<<g2, kHashTok, 0, s>>>(
                    static_cast<const float *>(X), R, bucket, p->H, p->n, p->n_rounds);
            else
                lsh_hash_fixed_kernel<float, 64, 8><<<g2, kHashTok, 0, s>>>(
                    static_cast<const float *>(X), R, bucket, p->H, p->n, p->n_rounds);
        } else {
            dim3 g3(ceil_div(p->n, kHash2Tok), 1, p->B * p->H);
            if (half == 32)
                lsh_hash_bf16x2_kernel<64, 32><<<g3, kHashTok, 0, s>>>(
                    static_cast<const __nv_bfloat16 *>(X), R, bucket, p->H, p->n, p->n_rounds);
            else
                lsh_hash_bf16x2_kernel<64, 8><<<g3, kHashTok, 0, s>>>(
                    static_cast<const __nv_bfloat16 *>(X), R, bucket, p->H, p->n, p->n_rounds);
        }
    } else if (p->dtype == CRS_F32) {
        CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_hash_kernel<float>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        {
            ProfScope _ps(K_LSH_HASH, s);
            lsh_hash_kernel<float><<<grid, kHashTok, smem, s>>>(
                static_cast<const float *>(X), R, bucket, p->H, p->n, p->d, p->n_buckets, p->n_rounds);
        }
    } else {
        CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_hash_kernel<__nv_bfloat16>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        {
            ProfScope _ps(K_LSH_HASH, s);
            lsh_hash_kernel<__nv_bfloat16><<<grid, kHashTok, smem, s>>>(
                static_cast<const __nv_bfloat16 *>(X), R, bucket, p->H, p->n, p->d, p->n_buckets,
                p->n_rounds);
        }
    }
    CRS_CHECK_LAUNCH();
    const size_t ssm = (size_t)(3 + kSortThreads / 32) * p->n_buckets * sizeof(int);
    if (ssm > 200 * 1024) return CRS_ERR_UNSUPPORTED;
    CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_sort_cluster_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm));
    {
        ProfScope _ps(K_LSH_SORT, s);
        lsh_sort_cluster_kernel<<<dim3(kSortCluster, p->B * p->H * p->n_rounds), kSortThreads, ssm, s>>>(
            bucket, perm, inv_perm, p->n, p->n_buckets);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

extern "C" size_t crs_lsh_attn_workspace_size(const crs_lsh_attn_params *a) {
    if (!a || validate_lsh(&a->p)) return 0;
    const crs_lsh_params &p = a->p;
    const size_t rows = (size_t)p.n_rounds * p.B * p.H * p.n;
    // per-round (o_r, lse_r), then the accumulated weight sums and shifts of each row,
    // then the persistent kernel's counters and its list of items left to the per-item kernel
    const size_t items = (size_t)ceil_div(p.n, kTcM) * p.n_rounds * p.B * p.H;
    return align256(rows * p.d * sizeof(float)) + align256(rows * sizeof(float)) +
           2 * align256((size_t)p.B * p.H * p.n * sizeof(float)) + 256 + align256(items * sizeof(int32_t));
}

namespace crs {
template <typename T, int DH>
static int launch_lsh_attn(const crs_lsh_attn_params *a, const void *QK, const void *V,
                           const int32_t *bucket, const int32_t *perm, const int32_t *inv_perm,
                           const int32_t *valid_len, void *O, float *lse, float *o_ws,
                           float *lse_ws, float *acc_L, float *acc_M, cudaStream_t s) {
    const crs_lsh_params &p = a->p;
    bool tc_done = false;
    if constexpr (std::is_same<T, __nv_bfloat16>::value && DH == kTcD) {
        // 16-byte row pieces are read from QK and V: both must be 16-byte aligned
        const bool aligned = !(reinterpret_cast<uintptr_t>(QK) & 15) && !(reinterpret_cast<uintptr_t>(V) & 15);
        if (p.chunk == kTcM && aligned) {
            // tensor-core path: bf16, d = 64, chunk = 128
            const size_t smem = sizeof(LshTcSmem) + 1024;
            CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_chunk_attn_tc_kernel,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
            CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_chunk_attn_tc_kernel,
                                              cudaFuncAttributePreferredSharedMemoryCarveout,
                                              (int)cudaSharedmemCarveoutMaxShared));
            dim3 grid(ceil_div(p.n, kTcM), p.n_rounds, p.B * p.H);
            // normalised keys: the rounds accumulate into O with a fixed shift per row
            const bool acc = a->key_norm != 0;
            const size_t nrow = (size_t)p.B * p.H * p.n;
            if (acc) {
                CRS_TRY_CUDA(cudaMemsetAsync(O, 0, nrow * DH * sizeof(float), s));
                CRS_TRY_CUDA(cudaMemsetAsync(acc_L, 0, 2 * align256(nrow * sizeof(float)), s));
            }
            if (acc && p.n_rounds <= kRgEarlier + 1) {
                // persistent ring kernel, then the per-item kernel over the items it left
                int *ctr = reinterpret_cast<int *>(reinterpret_cast<char *>(acc_M) + align256(nrow * sizeof(float)));
                int32_t *deferred = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(ctr) + 256);
                CRS_TRY_CUDA(cudaMemsetAsync(ctr, 0, 2 * sizeof(int), s));
                int dev = 0, sms = 148;
                CRS_TRY_CUDA(cudaGetDevice(&dev));
                CRS_TRY_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
                const int nch = ceil_div(p.n, kTcM);
                const long long units = (long long)(rg_big_units(nch) + rg_small_units(nch)) * p.n_rounds * p.B * p.H;
                const size_t rsmem = sizeof(RgSmem) + 1024;
                CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_chunk_attn_ring_kernel,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem));
                CRS_TRY_CUDA(cudaFuncSetAttribute(lsh_chunk_attn_ring_kernel,
                                                  cudaFuncAttributePreferredSharedMemoryCarveout,
                                                  (int)cudaSharedmemCarveoutMaxShared));
                {
                    ProfScope _ps(K_LSH_ATTN_RING, s);
                    lsh_chunk_attn_ring_kernel<<<(unsigned)min((long long)2 * sms, units), kRgThreads, rsmem, s>>>(
                        static_cast<const __nv_bfloat16 *>(QK), static_cast<const __nv_bfloat16 *>(V), bucket, perm,
                        inv_perm, valid_len, static_cast<float *>(O), acc_L, acc_M, ctr, deferred, ctr + 1, p.H,
                        p.B * p.H, p.n, p.n_rounds, a->causal, a->no_self, a->scale * 1.4426950408889634f);
                }
                CRS_CHECK_LAUNCH();
                {
                    ProfScope _ps(K_LSH_ATTN_TC, s);
                    lsh_chunk_attn_tc_kernel<<<(unsigned)sms, kTcThreads, smem, s>>>(
                        static_cast<const __nv_bfloat16 *>(QK), static_cast<const __nv_bfloat16 *>(V),
                        bucket, perm, inv_perm, valid_len, o_ws, lse_ws, static_cast<float *>(O), acc_L, acc_M,
                        p.H, p.B * p.H, p.n, p.n_rounds, a->causal, a->no_self, a->key_norm,
                        a->scale * 1.4426950408889634f, deferred, ctr + 1);
                }
            } else {
                ProfScope _ps(K_LSH_ATTN_TC, s);
                lsh_chunk_attn_tc_kernel<<<grid, kTcThreads, smem, s>>>(
                    static_cast<const __nv_bfloat16 *>(QK), static_cast<const __nv_bfloat16 *>(V),
                    bucket, perm, inv_perm, valid_len, o_ws, lse_ws, acc ? static_cast<float *>(O) : nullptr,
                    acc ? acc_L : nullptr, acc ? acc_M : nullptr, p.H, p.B * p.H, p.n, p.n_rounds,
                    a->causal, a->no_self, a->key_norm, a->scale * 1.4426950408889634f, nullptr, nullptr);
            }
            CRS_CHECK_LAUNCH();
            if (acc) {
                constexpr int kPer = DH / 4 >= 4 ? 4 : DH / 4;
                const long long work = (long long)p.B * p.H * p.n * (DH / 4 / kPer);
                {
                    ProfScope _ps(K_LSH_COMBINE, s);
                    lsh_finish_kernel<DH><<<(unsigned)ceil_div_ll(work, 256), 256, 0, s>>>(
                        o_ws, lse_ws, acc_L, acc_M, valid_len, static_cast<float *>(O), lse, p.B * p.H, p.H,
                        p.n, p.n_rounds);
                }
                CRS_CHECK_LAUNCH();
                return CRS_OK;
            }
            tc_done = true;
        }
    }
    const int KM = 2 * p.chunk;
    const size_t smem = (size_t)KM * (DH + 1) * 4 + (size_t)KM * DH * 4 + (size_t)KM * 4 +
                        (size_t)kAttnWarps * KM * 4 + (size_t)KM * 4 * 2 +
                        (size_t)KM * (kMaxRounds - 1) * 2 * 4;
    if (!tc_done) {
    if (smem > 227 * 1024) return CRS_ERR_UNSUPPORTED;
    auto kern = lsh_chunk_attn_kernel<T, DH>;
    CRS_TRY_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    // query splits per chunk: about two CTAs per SM when the problem is small, at
    // least one warp's worth of rows (8) per CTA
    const long long base_ctas = (long long)ceil_div(p.n, p.chunk) * p.n_rounds * p.B * p.H;
    const int q_splits = (int)max(1LL, min((long long)max(1, p.chunk / kAttnWarps), ceil_div_ll(2 * 148, base_ctas)));
    dim3 grid(ceil_div(p.n, p.chunk) * q_splits, p.n_rounds, p.B * p.H);
    {
        ProfScope _ps(K_LSH_ATTN, s);
        kern<<<grid, kAttnWarps * 32, smem, s>>>(static_cast<const T *>(QK), static_cast<const T *>(V),
                                                  bucket, perm, inv_perm, valid_len, o_ws, lse_ws, p.H,
                                                  p.n, p.chunk, p.n_rounds, a->causal, a->no_self,
                                                  a->key_norm, a->scale, q_splits);
    }
    CRS_CHECK_LAUNCH();
    }
    const long long work = (long long)p.B * p.H * p.n * (DH / 4);
    const int threads = 256;
    {
        ProfScope _ps(K_LSH_COMBINE, s);
        lsh_combine_kernel<DH><<<(unsigned)ceil_div_ll(work, threads), threads, 0, s>>>(
            o_ws, lse_ws, valid_len, static_cast<float *>(O), lse, p.B * p.H, p.H, p.n, p.n_rounds);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}
}  // namespace crs

extern "C" int crs_lsh_attn(const crs_lsh_attn_params *a, const void *QK, const void *V,
                            const int32_t *bucket, const int32_t *perm, const int32_t *inv_perm,
                            const int32_t *valid_len, void *O, float *lse, void *ws,
                            size_t ws_bytes, void *stream) {
    if (!a) return CRS_ERR_INVALID_ARG;
    int st = validate_lsh(&a->p);
    if (st) return st;
    const crs_lsh_params &p = a->p;
    if (p.chunk < 1 || p.chunk > 128) return CRS_ERR_INVALID_ARG;
    if (!QK || !V || !bucket || !perm || !inv_perm || !O) return CRS_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(O) & 15) return CRS_ERR_INVALID_ARG;   // 16-byte row stores
    if (!(a->scale == a->scale)) return CRS_ERR_INVALID_ARG;
    const size_t need = crs_lsh_attn_workspace_size(a);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    const size_t rows = (size_t)p.n_rounds * p.B * p.H * p.n;
    float *o_ws = static_cast<float *>(ws);
    float *lse_ws = reinterpret_cast<float *>(static_cast<char *>(ws) +
                                              align256(rows * p.d * sizeof(float)));
    float *acc_L = reinterpret_cast<float *>(reinterpret_cast<char *>(lse_ws) + align256(rows * sizeof(float)));
    float *acc_M = reinterpret_cast<float *>(reinterpret_cast<char *>(acc_L) +
                                             align256((size_t)p.B * p.H * p.n * sizeof(float)));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p.d == 64) {
        if (p.dtype == CRS_F32)
            return launch_lsh_attn<float, 64>(a, QK, V, bucket, perm, inv_perm, valid_len, O, lse,
                                              o_ws, lse_ws, acc_L, acc_M, s);
        return launch_lsh_attn<__nv_bfloat16, 64>(a, QK, V, bucket, perm, inv_perm, valid_len, O,
                                                  lse, o_ws, lse_ws, acc_L, acc_M, s);
    }
    if (p.d == 32) {
        if (p.dtype == CRS_F32)
            return launch_lsh_attn<float, 32>(a, QK, V, bucket, perm, inv_perm, valid_len, O, lse,
                                              o_ws, lse_ws, acc_L, acc_M, s);
        return launch_lsh_attn<__nv_bfloat16, 32>(a, QK, V, bucket, perm, inv_perm, valid_len, O,
                                                  lse, o_ws, lse_ws, acc_L, acc_M, s);
    }
    return CRS_ERR_UNSUPPORTED;
}
