// Routing (k-means) attention with quota execution, sm_100a.
//
// [P1] PaperTrace 2.1.1 §3.1: frozen centres M (inference), routing scores
// S_Q = Q M^T and S_K = K M^T; each centre c keeps its m best queries and m best
// keys, J_c^Q = Top_m(S_Q[:, c]) and J_c^K = Top_m(S_K[:, c]) ("定额执行"); a
// token may sit in several centres, so each query's outputs over its centres
// are combined at its original index.  Query i attends to the union of J_c^K
// over its centres, each key once: pair (i, j) is taken in the first centre
// holding both.
//
//   route_score_kernel    s = x . mu_c as one fp32 FMA per term in index order
//                         (an integer decision, taken as the oracle takes it),
//                         stored as order-preserving keys [role][c][token]
//   route_quota_kernel    one 1024-thread CTA per (b, h, role, c): 4-pass 8-bit
//                         radix select of the m-th key (one shared histogram per
//                         warp, then summed), ties to the smaller index by prefix sums,
//                         the kept tokens ascending + membership bitmaps
//   route_attn_tc_kernel  one CTA per (b, h, c) for m <= 128: S = Q K^T and P V on
//                         mma.sync tiles, masks per element, exact softmax;
//   route_attn_kernel     (m > 128) one CTA per (b, h, c): thread = query of the centre,
//                         the centre's keys and values staged in shared memory,
//                         causal / self / earlier-centre pairs masked, online
//                         softmax; partial (o, lse, count) per (c, slot)
//   route_merge_kernel    one warp per query: its centres' partials combined
//                         by log-sum-exp (slots recorded by the quota kernel)
#include "common.cuh"

namespace crs {

constexpr int kRtD = 64;
constexpr int kRtMaxC = 256;
constexpr int kRtMaxM = 256;
constexpr int kRtScoreTok = 64;            // tokens per score CTA

struct RtArgs {
    const __nv_bfloat16 *Q, *K, *V;        // [B, H, n, d]
    const float *M;                        // [H, C, d]
    uint32_t *keys;                        // [B, H, 2, C, n]
    uint32_t *memb;                        // [B, H, 2, n, C/32]
    uint8_t *qslot;                        // [B, H, n, C]: slot of query i in J_c^Q
    int32_t *JQ, *JK;                      // [B, H, C, m]
    float *part_o, *part_lse;              // [B, H, C, m, d], [B, H, C, m]
    int32_t *part_cnt;                     // [B, H, C, m]
    float *O, *lse;                        // [B, H, n, d], [B, H, n]
    int32_t *count;                        // [B, H, n]
    int B, H, n, C, m, mm, words, causal, no_self;
    float scale;
};

// grid (ceil(n / 64), B * H * 2), 256 threads: thread (token t = tid % 64, centres tid / 64 + 4k)
__global__ void __launch_bounds__(256) route_score_kernel(RtArgs a) {
    extern __shared__ float rt_mu[];                                   // [C][d]
    const int bhr = blockIdx.y, role = bhr & 1, bh = bhr >> 1, h = bh % a.H;
    const int t = blockIdx.x * kRtScoreTok + (threadIdx.x & 63);
    for (int e = threadIdx.x; e < a.C * kRtD; e += 256) rt_mu[e] = a.M[(size_t)h * a.C * kRtD + e];
    __syncthreads();
    if (t >= a.n) return;
    const __nv_bfloat16 *x = (role == 0 ? a.Q : a.K) + ((size_t)bh * a.n + t) * kRtD;
    float xv[kRtD];
#pragma unroll
    for (int c = 0; c < kRtD / 8; ++c) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(x) + c);
        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 f = __bfloat1622float2(p2[u]);
            xv[c * 8 + 2 * u] = f.x;
            xv[c * 8 + 2 * u + 1] = f.y;
        }
    }
    uint32_t *out = a.keys + ((size_t)bh * 2 + role) * a.C * a.n;
    // two centres at a time (two independent chains), the centre read 4 values per load;
    // each chain is still one FMA per term in index order from 0
    for (int c = threadIdx.x >> 6; c < a.C; c += 8) {
        const int c2 = c + 4 < a.C ? c + 4 : c;
        const float4 *mu0 = reinterpret_cast<const float4 *>(rt_mu + c * kRtD);
        const float4 *mu1 = reinterpret_cast<const float4 *>(rt_mu + c2 * kRtD);
        float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
        for (int i4 = 0; i4 < kRtD / 4; ++i4) {
            const float4 m0 = mu0[i4], m1 = mu1[i4];
            acc0 = fmaf(xv[4 * i4], m0.x, acc0);
            acc1 = fmaf(xv[4 * i4], m1.x, acc1);
            acc0 = fmaf(xv[4 * i4 + 1], m0.y, acc0);
            acc1 = fmaf(xv[4 * i4 + 1], m1.y, acc1);
            acc0 = fmaf(xv[4 * i4 + 2], m0.z, acc0);
            acc1 = fmaf(xv[4 * i4 + 2], m1.z, acc1);
            acc0 = fmaf(xv[4 * i4 + 3], m0.w, acc0);
            acc1 = fmaf(xv[4 * i4 + 3], m1.w, acc1);
        }
        out[(size_t)c * a.n + t] = score_key(acc0);
        if (c2 != c) out[(size_t)c2 * a.n + t] = score_key(acc1);
    }
}

template <int KPT>
__global__ void __launch_bounds__(kPickT) route_quota_kernel(RtArgs a) {
    __shared__ uint32_t whist[kPickT / 32][256];           // one histogram per warp
    __shared__ uint32_t hist[256];
    __shared__ int sbin, sneed;
    __shared__ int2 wtot[kPickT / 32 + 1];
    const int c = blockIdx.x, bhr = blockIdx.y, role = bhr & 1, bh = bhr >> 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t *kc = a.keys + (((size_t)bh * 2 + role) * a.C + c) * a.n;
    uint32_t key[KPT];
    bool valid[KPT];
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        const int i = tid * KPT + u;
        valid[u] = i < a.n;
        key[u] = valid[u] ? kc[i] : 0u;
    }
    // m-th largest key by 8-bit digits from the top
    uint32_t prefix = 0u, mask = 0u;
    int need = a.mm;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int e = lane; e < 256; e += 32) whist[warp][e] = 0u;
        __syncwarp();
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            if (valid[u] && (key[u] & mask) == prefix) atomicAdd(&whist[warp][(key[u] >> shift) & 255u], 1u);
        __syncthreads();
        for (int e = tid; e < 256; e += kPickT) {
            uint32_t v = 0u;
#pragma unroll 8
            for (int w = 0; w < kPickT / 32; ++w) v += whist[w][e];
            hist[e] = v;
        }
        __syncthreads();
        if (warp == 0) {
            int nd = need;
            const int bin = warp_top_bin(hist, nd);
            if (lane == 0) {
                sbin = bin;
                sneed = nd;
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sbin << shift;
        mask |= 0xffu << shift;
        need = sneed;
        __syncthreads();
    }
    const uint32_t T = prefix;
    int n_eq = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) n_eq += (valid[u] && key[u] == T) ? 1 : 0;
    int eq_before, d0, t0, t1;
    cta_exscan2(n_eq, 0, eq_before, d0, t0, t1, wtot);
    bool take[KPT];
    int n_take = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        const bool eq = valid[u] && key[u] == T;
        take[u] = (valid[u] && key[u] > T) || (eq && eq_before < need);
        eq_before += eq ? 1 : 0;
        n_take += take[u] ? 1 : 0;
    }
    int slot, d1, n_sel, t2;
    cta_exscan2(n_take, 0, slot, d1, n_sel, t2, wtot);
    int32_t *J = (role == 0 ? a.JQ : a.JK) + ((size_t)bh * a.C + c) * a.m;
    uint32_t *mb = a.memb + ((size_t)bh * 2 + role) * a.n * a.words;
#pragma unroll
    for (int u = 0; u < KPT; ++u)
        if (take[u]) {
            const int i = tid * KPT + u;
            if (role == 0) a.qslot[((size_t)bh * a.n + i) * a.C + c] = (uint8_t)slot;
            J[slot++] = i;
            atomicOr(&mb[(size_t)i * a.words + (c >> 5)], 1u << (c & 31));
        }
    for (int e = n_sel + tid; e < a.m; e += kPickT) J[e] = -1;
}

// one CTA per (b, h, c); thread s < mm = the centre's s-th query
constexpr int kRtRow = kRtD + 8;            // staged row stride (bf16): 16-byte rows, no bank conflicts

__host__ __device__ inline size_t rt_attn_smem(int mm) { return (size_t)mm * (2 * kRtRow * 2 + 4); }

__global__ void __launch_bounds__(kRtMaxM) route_attn_kernel(RtArgs a) {
    extern __shared__ __align__(16) unsigned char rt_smem[];
    __nv_bfloat16 (*sk)[kRtRow] = reinterpret_cast<__nv_bfloat16 (*)[kRtRow]>(rt_smem);
    __nv_bfloat16 (*sv)[kRtRow] = reinterpret_cast<__nv_bfloat16 (*)[kRtRow]>(rt_smem + (size_t)a.mm * kRtRow * 2);
    int *sj = reinterpret_cast<int *>(rt_smem + (size_t)a.mm * kRtRow * 4);
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const int32_t *JQ = a.JQ + ((size_t)bh * a.C + c) * a.m, *JK = a.JK + ((size_t)bh * a.C + c) * a.m;
    for (int e = tid; e < a.mm * (kRtD / 8); e += blockDim.x) {
        const int r = e / (kRtD / 8), q8 = e - r * (kRtD / 8);
        const int j = JK[r];
        const size_t row = ((size_t)bh * a.n + j) * kRtD + q8 * 8;
        *reinterpret_cast<uint4 *>(&sk[r][q8 * 8]) = __ldg(reinterpret_cast<const uint4 *>(a.K + row));
        *reinterpret_cast<uint4 *>(&sv[r][q8 * 8]) = __ldg(reinterpret_cast<const uint4 *>(a.V + row));
        if (q8 == 0) sj[r] = j;
    }
    __syncthreads();
    if (tid >= a.mm) return;
    const int i = JQ[tid];
    const size_t ps = ((size_t)bh * a.C + c) * a.m + tid;
    float q[kRtD];
    {
        const uint4 *qr = reinterpret_cast<const uint4 *>(a.Q + ((size_t)bh * a.n + i) * kRtD);
#pragma unroll
        for (int c8 = 0; c8 < kRtD / 8; ++c8) {
            const uint4 raw = __ldg(qr + c8);
            const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(p2[u]);
                q[c8 * 8 + 2 * u] = a.scale * f.x;
                q[c8 * 8 + 2 * u + 1] = a.scale * f.y;
            }
        }
    }
    // earlier centres that also hold query i (as a query)
    const uint32_t *mq = a.memb + ((size_t)bh * 2 + 0) * a.n * a.words + (size_t)i * a.words;
    const uint32_t *mk_base = a.memb + ((size_t)bh * 2 + 1) * a.n * a.words;
    uint32_t qlow[kRtMaxC / 32];
#pragma unroll
    for (int w = 0; w < kRtMaxC / 32; ++w) {
        uint32_t v = w < a.words ? mq[w] : 0u;
        if (w > (c >> 5)) v = 0u;
        else if (w == (c >> 5)) v &= (1u << (c & 31)) - 1u;
        qlow[w] = v;
    }
    float mx = -INFINITY, l = 0.0f, o[kRtD];
#pragma unroll
    for (int t = 0; t < kRtD; ++t) o[t] = 0.0f;
    int cnt = 0;
    for (int r = 0; r < a.mm; ++r) {
        const int j = sj[r];
        if ((a.causal && j > i) || (a.no_self && j == i)) continue;
        bool met = false;
        const uint32_t *mk = mk_base + (size_t)j * a.words;
        for (int w = 0; w <= (c >> 5) && !met; ++w) met = (qlow[w] & mk[w]) != 0u;
        if (met) continue;
        float dot = 0.0f;
#pragma unroll
        for (int t = 0; t < kRtD; t += 2) {
            const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&sk[r][t]));
            dot = fmaf(q[t], kv.x, fmaf(q[t + 1], kv.y, dot));
        }
        const float mn = fmaxf(mx, dot), corr = __expf(mx - mn), p = __expf(dot - mn);
        l = l * corr + p;
#pragma unroll
        for (int t = 0; t < kRtD; t += 2) {
            const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&sv[r][t]));
            o[t] = fmaf(p, vv.x, o[t] * corr);
            o[t + 1] = fmaf(p, vv.y, o[t + 1] * corr);
        }
        mx = mn;
        ++cnt;
    }
    float *po = a.part_o + ps * kRtD;
    const float inv = cnt > 0 ? 1.0f / l : 0.0f;
#pragma unroll
    for (int t = 0; t < kRtD; ++t) po[t] = o[t] * inv;
    a.part_lse[ps] = cnt > 0 ? mx + logf(l) : -INFINITY;
    a.part_cnt[ps] = cnt;
}

// The same per-centre attention on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate) for quotas up to 128: the centre's query, key and value rows
// are staged in 128B-swizzled shared rows; warp w takes query slots 16w..16w+15
// against all 128 key slots: S = Q K^T (16 n-tiles), the causal / self /
// earlier-centre masks per element (key membership words in shared memory,
// the query's earlier-centre words in registers), an exact softmax over the
// 128 slots, then O = P V with P carried as a bf16 value + bf16 residual.
constexpr int kRtTcM = 128;
constexpr int kRtMaxWords = kRtMaxC / 32;

__device__ __forceinline__ uint32_t rt_sw(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

struct RtTcSmem {
    unsigned char q[kRtTcM * 128], k[kRtTcM * 128], v[kRtTcM * 128];   // 64 bf16 per row
    int qi[kRtTcM], kj[kRtTcM];
    uint32_t km[kRtTcM][kRtMaxWords];
};

__global__ void __launch_bounds__(256) route_attn_tc_kernel(RtArgs a) {
    extern __shared__ __align__(128) unsigned char rt_tc_raw[];
    RtTcSmem &S = *reinterpret_cast<RtTcSmem *>(rt_tc_raw);
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int32_t *JQ = a.JQ + ((size_t)bh * a.C + c) * a.m, *JK = a.JK + ((size_t)bh * a.C + c) * a.m;
    const uint32_t *mkb = a.memb + ((size_t)bh * 2 + 1) * a.n * a.words;
    for (int e = tid; e < kRtTcM * 8; e += 256) {
        const int r = e >> 3, ch = e & 7;
        const int i = r < a.mm ? JQ[r] : -1, j = r < a.mm ? JK[r] : -1;
        uint4 qv = make_uint4(0, 0, 0, 0), kv = qv, vv = qv;
        if (i >= 0) qv = __ldg(reinterpret_cast<const uint4 *>(a.Q + ((size_t)bh * a.n + i) * kRtD) + ch);
        if (j >= 0) {
            kv = __ldg(reinterpret_cast<const uint4 *>(a.K + ((size_t)bh * a.n + j) * kRtD) + ch);
            vv = __ldg(reinterpret_cast<const uint4 *>(a.V + ((size_t)bh * a.n + j) * kRtD) + ch);
        }
        *reinterpret_cast<uint4 *>(S.q + rt_sw(r, ch)) = qv;
        *reinterpret_cast<uint4 *>(S.k + rt_sw(r, ch)) = kv;
        *reinterpret_cast<uint4 *>(S.v + rt_sw(r, ch)) = vv;
        if (ch == 0) {
            S.qi[r] = i;
            S.kj[r] = j;
        }
        if (ch < kRtMaxWords) S.km[r][ch] = (j >= 0 && ch < a.words) ? mkb[(size_t)j * a.words + ch] : 0u;
    }
    __syncthreads();
    const int r0 = warp * 16;
    if (r0 >= a.mm) return;
    const int g_row = lane >> 2, tig = lane & 3;
    // query fragments: 16 rows x 64 dims, 4 k-steps
    uint32_t qf[4][4];
    {
        const uint32_t qb = smem_u32(S.q);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int mi = lane >> 3, r = r0 + (lane & 7) + ((mi & 1) << 3), ch = kk * 2 + (mi >> 1);
            ldsm_x4(qb + rt_sw(r, ch), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
    }
    float sc[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
    {
        const uint32_t kb = smem_u32(S.k);
#pragma unroll
        for (int np = 0; np < 8; ++np)                  // pairs of n-tiles: 16 keys
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int mi = lane >> 3;
                const int r = np * 16 + (lane & 7) + ((mi >> 1) << 3), ch = kk * 2 + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + rt_sw(r, ch), b0, b1, b2, b3);
                mma_bf16(sc[2 * np], qf[kk], b0, b1);
                mma_bf16(sc[2 * np + 1], qf[kk], b2, b3);
            }
    }
    // masks: rows g_row (lo) and g_row + 8 (hi) of this warp's 16
    const int rl = r0 + g_row, rh = r0 + g_row + 8;
    const int il = rl < a.mm ? S.qi[rl] : -1, ih = rh < a.mm ? S.qi[rh] : -1;
    uint32_t ql[kRtMaxWords], qh[kRtMaxWords];
    const uint32_t *mqb = a.memb + ((size_t)bh * 2 + 0) * a.n * a.words;
#pragma unroll
    for (int w = 0; w < kRtMaxWords; ++w) {
        const uint32_t lowmask = w < (c >> 5) ? 0xffffffffu : (w == (c >> 5) ? (1u << (c & 31)) - 1u : 0u);
        ql[w] = (il >= 0 && w < a.words) ? mqb[(size_t)il * a.words + w] & lowmask : 0u;
        qh[w] = (ih >= 0 && w < a.words) ? mqb[(size_t)ih * a.words + w] & lowmask : 0u;
    }
    const float sl2 = a.scale * 1.4426950408889634f;
    float mxl = -INFINITY, mxh = -INFINITY;
    int cl = 0, ch_ = 0;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int col = nt * 8 + tig * 2 + e;
            const int j = S.kj[col];
            bool metl = false, meth = false;
#pragma unroll
            for (int w = 0; w < kRtMaxWords; ++w) {
                const uint32_t kw = S.km[col][w];
                metl |= (ql[w] & kw) != 0u;
                meth |= (qh[w] & kw) != 0u;
            }
            const bool okl = il >= 0 && j >= 0 && !(a.causal && j > il) && !(a.no_self && j == il) && !metl;
            const bool okh = ih >= 0 && j >= 0 && !(a.causal && j > ih) && !(a.no_self && j == ih) && !meth;
            sc[nt][e] = okl ? sc[nt][e] * sl2 : -INFINITY;
            sc[nt][2 + e] = okh ? sc[nt][2 + e] * sl2 : -INFINITY;
            mxl = fmaxf(mxl, sc[nt][e]);
            mxh = fmaxf(mxh, sc[nt][2 + e]);
            cl += okl ? 1 : 0;
            ch_ += okh ? 1 : 0;
        }
    mxl = fmaxf(mxl, __shfl_xor_sync(0xffffffffu, mxl, 1));
    mxl = fmaxf(mxl, __shfl_xor_sync(0xffffffffu, mxl, 2));
    mxh = fmaxf(mxh, __shfl_xor_sync(0xffffffffu, mxh, 1));
    mxh = fmaxf(mxh, __shfl_xor_sync(0xffffffffu, mxh, 2));
    float sum_l = 0.0f, sum_h = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            sc[nt][e] = sc[nt][e] == -INFINITY ? 0.0f : exp2f(sc[nt][e] - mxl);
            sc[nt][2 + e] = sc[nt][2 + e] == -INFINITY ? 0.0f : exp2f(sc[nt][2 + e] - mxh);
            sum_l += sc[nt][e];
            sum_h += sc[nt][2 + e];
        }
    sum_l += __shfl_xor_sync(0xffffffffu, sum_l, 1);
    sum_l += __shfl_xor_sync(0xffffffffu, sum_l, 2);
    sum_h += __shfl_xor_sync(0xffffffffu, sum_h, 1);
    sum_h += __shfl_xor_sync(0xffffffffu, sum_h, 2);
    cl += __shfl_xor_sync(0xffffffffu, cl, 1);
    cl += __shfl_xor_sync(0xffffffffu, cl, 2);
    ch_ += __shfl_xor_sync(0xffffffffu, ch_, 1);
    ch_ += __shfl_xor_sync(0xffffffffu, ch_, 2);
    // O = P V
    float o[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
    const uint32_t vb = smem_u32(S.v);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {                      // 16 key slots per k-step
        uint32_t pa[4], pl[4];
        pack_bf16_split(sc[2 * kk][0], sc[2 * kk][1], pa[0], pl[0]);
        pack_bf16_split(sc[2 * kk][2], sc[2 * kk][3], pa[1], pl[1]);
        pack_bf16_split(sc[2 * kk + 1][0], sc[2 * kk + 1][1], pa[2], pl[2]);
        pack_bf16_split(sc[2 * kk + 1][2], sc[2 * kk + 1][3], pa[3], pl[3]);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {                  // 16 dims per step
            const int mi = lane >> 3;
            const int r = kk * 16 + (lane & 7) + ((mi & 1) << 3), chn = jj * 2 + (mi >> 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vb + rt_sw(r, chn), b0, b1, b2, b3);
            mma_bf16(o[2 * jj], pa, b0, b1);
            mma_bf16(o[2 * jj], pl, b0, b1);
            mma_bf16(o[2 * jj + 1], pa, b2, b3);
            mma_bf16(o[2 * jj + 1], pl, b2, b3);
        }
    }
    const float il_ = sum_l > 0.0f ? 1.0f / sum_l : 0.0f, ih_ = sum_h > 0.0f ? 1.0f / sum_h : 0.0f;
    const size_t pbase = ((size_t)bh * a.C + c) * a.m;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int col = nt * 8 + tig * 2;
        if (rl < a.mm)
            *reinterpret_cast<float2 *>(a.part_o + (pbase + rl) * kRtD + col) = make_float2(o[nt][0] * il_, o[nt][1] * il_);
        if (rh < a.mm)
            *reinterpret_cast<float2 *>(a.part_o + (pbase + rh) * kRtD + col) = make_float2(o[nt][2] * ih_, o[nt][3] * ih_);
    }
    if (tig == 0) {
        const float ln2 = 0.6931471805599453f;
        if (rl < a.mm) {
            a.part_lse[pbase + rl] = cl > 0 ? (mxl + log2f(sum_l)) * ln2 : -INFINITY;
            a.part_cnt[pbase + rl] = cl;
        }
        if (rh < a.mm) {
            a.part_lse[pbase + rh] = ch_ > 0 ? (mxh + log2f(sum_h)) * ln2 : -INFINITY;
            a.part_cnt[pbase + rh] = ch_;
        }
    }
}

// one warp per (b, h, i): lanes own dims 2l, 2l + 1
__global__ void __launch_bounds__(256) route_merge_kernel(RtArgs a) {
    const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= (long long)a.B * a.H * a.n) return;
    const int i = (int)(w % a.n), bh = (int)(w / a.n);
    const uint32_t *mq = a.memb + ((size_t)bh * 2 + 0) * a.n * a.words + (size_t)i * a.words;
    float M = -INFINITY;
    for (int pass = 0; pass < 2; ++pass) {
        float z = 0.0f, o0 = 0.0f, o1 = 0.0f;
        int cnt = 0;
        for (int wd = 0; wd < a.words; ++wd) {
            uint32_t bits = mq[wd];
            while (bits) {
                const int c = wd * 32 + __ffs(bits) - 1;
                bits &= bits - 1u;
                const int slot = a.qslot[((size_t)bh * a.n + i) * a.C + c];
                const size_t ps = ((size_t)bh * a.C + c) * a.m + slot;
                const float ls = a.part_lse[ps];
                if (pass == 0) {
                    M = fmaxf(M, ls);
                } else if (ls != -INFINITY) {
                    const float f = __expf(ls - M);
                    z += f;
                    const float2 po = *reinterpret_cast<const float2 *>(a.part_o + ps * kRtD + 2 * lane);
                    o0 = fmaf(f, po.x, o0);
                    o1 = fmaf(f, po.y, o1);
                }
                cnt += a.part_cnt[ps];
            }
        }
        if (pass == 1) {
            const size_t oi = (size_t)bh * a.n + i;
            const float iz = z > 0.0f ? 1.0f / z : 0.0f;
            *reinterpret_cast<float2 *>(a.O + oi * kRtD + 2 * lane) = make_float2(o0 * iz, o1 * iz);
            if (lane == 0) {
                a.lse[oi] = z > 0.0f ? M + logf(z) : -INFINITY;
                if (a.count) a.count[oi] = cnt;
            }
        }
    }
}

struct RtWs {
    uint32_t *keys, *memb;
    uint8_t *qslot;
    float *part_o, *part_lse;
    int32_t *part_cnt;
    size_t total;
};

static int rt_validate(const crs_route_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->B < 1 || p->H < 1 || p->n < 1 || p->C < 1 || p->m < 1) return CRS_ERR_INVALID_ARG;
    if (p->d != kRtD || p->C > kRtMaxC || p->m > kRtMaxM || p->n > 16 * kPickT) return CRS_ERR_UNSUPPORTED;
    return CRS_OK;
}

static void rt_ws_layout(const crs_route_params *p, RtWs &w, char *base) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t bh = (size_t)p->B * p->H;
    const int words = (p->C + 31) / 32;
    size_t off = 0;
    auto take = [&](size_t bytes) { char *q = base ? base + off : nullptr; off += al(bytes); return q; };
    w.keys = reinterpret_cast<uint32_t *>(take(bh * 2 * p->C * p->n * 4));
    w.memb = reinterpret_cast<uint32_t *>(take(bh * 2 * p->n * words * 4));
    w.qslot = reinterpret_cast<uint8_t *>(take(bh * p->n * p->C));
    w.part_o = reinterpret_cast<float *>(take(bh * p->C * p->m * kRtD * 4));
    w.part_lse = reinterpret_cast<float *>(take(bh * p->C * p->m * 4));
    w.part_cnt = reinterpret_cast<int32_t *>(take(bh * p->C * p->m * 4));
    w.total = off;
}

}  // namespace crs

using namespace crs;

extern "C" size_t crs_route_attn_workspace_size(const crs_route_params *p) {
    if (rt_validate(p)) return 0;
    RtWs w;
    rt_ws_layout(p, w, nullptr);
    return w.total;
}

extern "C" int crs_route_attn(const crs_route_params *p, const void *Q, const void *K, const void *V,
                              const float *M, int32_t *JQ, int32_t *JK, float *O, float *lse, int32_t *count,
                              void *ws, size_t ws_bytes, void *stream) {
    int st = rt_validate(p);
    if (st) return st;
    if (!Q || !K || !V || !M || !JQ || !JK || !O || !lse) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) & 15)
        return CRS_ERR_INVALID_ARG;
    const size_t need = crs_route_attn_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    RtWs w;
    rt_ws_layout(p, w, static_cast<char *>(ws));
    RtArgs a{};
    a.Q = static_cast<const __nv_bfloat16 *>(Q);
    a.K = static_cast<const __nv_bfloat16 *>(K);
    a.V = static_cast<const __nv_bfloat16 *>(V);
    a.M = M;
    a.keys = w.keys;
    a.memb = w.memb;
    a.qslot = w.qslot;
    a.JQ = JQ;
    a.JK = JK;
    a.part_o = w.part_o;
    a.part_lse = w.part_lse;
    a.part_cnt = w.part_cnt;
    a.O = static_cast<float *>(O);
    a.lse = lse;
    a.count = count;
    a.B = p->B;
    a.H = p->H;
    a.n = p->n;
    a.C = p->C;
    a.m = p->m;
    a.mm = min(p->m, p->n);
    a.words = (p->C + 31) / 32;
    a.causal = p->causal;
    a.no_self = p->no_self;
    a.scale = p->scale;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int BH = p->B * p->H;
    const size_t smem_score = (size_t)p->C * kRtD * 4;
    CRS_TRY_CUDA(cudaFuncSetAttribute(route_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem_score));
    ProfScope _ps(K_ROUTE, s);
    CRS_TRY_CUDA(cudaMemsetAsync(w.memb, 0, (size_t)BH * 2 * p->n * a.words * 4, s));
    route_score_kernel<<<dim3(ceil_div(p->n, kRtScoreTok), BH * 2), 256, smem_score, s>>>(a);
    const dim3 gq(p->C, BH * 2);
    const int kpt = ceil_div(p->n, kPickT);
    if (kpt <= 1) route_quota_kernel<1><<<gq, kPickT, 0, s>>>(a);
    else if (kpt <= 2) route_quota_kernel<2><<<gq, kPickT, 0, s>>>(a);
    else if (kpt <= 4) route_quota_kernel<4><<<gq, kPickT, 0, s>>>(a);
    else if (kpt <= 8) route_quota_kernel<8><<<gq, kPickT, 0, s>>>(a);
    else route_quota_kernel<16><<<gq, kPickT, 0, s>>>(a);
    if (a.mm <= kRtTcM) {
        CRS_TRY_CUDA(cudaFuncSetAttribute(route_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)sizeof(RtTcSmem)));
        route_attn_tc_kernel<<<dim3(p->C, BH), 256, sizeof(RtTcSmem), s>>>(a);
    } else {
        CRS_TRY_CUDA(cudaFuncSetAttribute(route_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)rt_attn_smem(a.mm)));
        route_attn_kernel<<<dim3(p->C, BH), max(32, ceil_div(a.mm, 32) * 32), rt_attn_smem(a.mm), s>>>(a);
    }
    route_merge_kernel<<<(unsigned)ceil_div((long long)BH * p->n, 8), 256, 0, s>>>(a);
    _ps.more(3);                                  // score, quota, attention, merge
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}
