// K1 on the tensor cores: LSH bucket ids for bf16 rows, d = 64, b = 64 buckets.
//
// [P1] PaperTrace 2.1.1 §2.1 Eq.(4): u = x R_{h,r}, bucket = argmax [u ; -u]
// (first maximum).  The bucket is an integer decided by floating point; its
// definition here is the fp32 chain u_k = fma(x_63, r_63k, ... fma(x_0, r_0k, 0)),
// terms in index order, which the CUDA-core kernels evaluate directly.
//
// This kernel reaches the same integers through a filter with an exact
// fallback:
//   1. approximate u~ = x (R_hi + R_lo) on tcgen05 (R split into two bf16
//      parts, x exact in bf16, every product exact, fp32 accumulation in
//      tensor memory) for all rounds at once (N = 32 x rounds columns);
//   2. per (token, round): with E_k = 2^-12 |x| |r_k| (Cauchy-Schwarz bounds
//      S_k = sum_i |x_i| |r_ik| by |x| |r_k|), the largest |u~_k| wins by more
//      than E_k1 + E_k2 over the runner-up and by more than E_k1 over its own
//      negation -> it is the argmax of the chain values as well (see the bound
//      below), and its sign picks the +u or -u half;
//   3. otherwise (a near tie, or all u~ ~ 0) the warp recomputes that token's
//      32 chains exactly, one per lane, in index order, and takes the first
//      maximum as the definition does.
// The bound: |u~_k - u_k| <= |x . (R - R_hi - R_lo)| + (tensor-core
// accumulation) + (chain rounding) <= (2^-16 + 128 * 2^-22 + gamma_64) S_k
// < 5e-5 S_k <= 5e-5 |x| |r_k|; E_k = 2^-12 |x| |r_k| (norms in fp32) covers it
// with a factor of about 4.9.  A winner by more than the two bounds therefore
// wins in the chain values.
//
// Persistent, warp-specialised CTA walking the 128-token tiles of one
// (batch, head): warp 0 loads X tiles with TMA into a 2-stage ring, warp 1
// issues the MMAs into two tensor-memory buffers, warps 2..9 (one token row
// per thread; two warps per row quadrant, each taking half of the rounds) read
// the scores, decide the buckets and release the buffers.
// R is split into its operand tiles once per CTA.
#include "common.cuh"
#include "tc.cuh"

namespace crs {

constexpr int kHtM = 128;                 // tokens per tile (MMA M)
constexpr int kHtHalf = 32;               // b / 2
constexpr int kHtD = 64;
constexpr int kHtMaxN = 128;              // 32 x rounds, rounds <= 4
constexpr int kHtStages = 2;                  // X tiles in flight (the fp32 R copy takes the third's room)
constexpr int kHtEpiWarps = 8;            // two per tensor-memory lane quadrant, each half the rounds
constexpr int kHtThreads = 32 * (2 + kHtEpiWarps);
constexpr float kHtErr = 2.44140625e-4f;  // 2^-12
constexpr uint64_t kHtWaitNs = 1000000000ull;
constexpr uint32_t kHtSuspendNs = 256;

struct HtSmem {
    unsigned char x[kHtStages][kHtM * 128];   // X tiles, 128B swizzle
    unsigned char bhi[kHtMaxN * 128];         // B operand: R_hi, row r*32 + k = column k of R_{h,r}
    unsigned char blo[kHtMaxN * 128];         //            R_lo
    float rf[kHtMaxN * kHtD];                 // R_{h,r} in fp32, [r][t][k] as in global memory: the
                                              // exact chains of the near ties read it here
    float rnorm[kHtMaxN];                     // |r_k| per column
    uint64_t xfull[kHtStages], xempty[kHtStages], tfull[2], tempty[2];
    uint32_t tmem_base;
    int fail;
};

// The definition's bucket of token row rl of the X tile xa for one round (R_{h,r} at Rr,
// fp32, [t][k]): lane k evaluates the chain u_k = fma(x_63, r_63k, ... fma(x_0, r_0k, 0)) in
// index order, then the first maximum of [u ; -u].  Warp-collective; out of line so that
// the common path of the epilogue keeps its registers.
__device__ __noinline__ int ht_exact_bucket(const unsigned char *xa, int rl, const float *Rr, int lane) {
    // token row rl: eight 16-byte broadcast reads; column `lane` of R from shared memory
    uint32_t xw[kHtD / 2];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 w4 = *reinterpret_cast<const uint4 *>(xa + tc::sw128(rl, c));
        xw[4 * c] = w4.x;
        xw[4 * c + 1] = w4.y;
        xw[4 * c + 2] = w4.z;
        xw[4 * c + 3] = w4.w;
    }
    float u = 0.0f;
#pragma unroll
    for (int t = 0; t < kHtD; ++t) {
        const float xt = __uint_as_float((t & 1) ? (xw[t >> 1] & 0xffff0000u) : (xw[t >> 1] << 16));
        u = __fmaf_rn(xt, Rr[t * kHtHalf + lane], u);
    }
    const float bp = warp_max(u);
    const int ap = __ffs(__ballot_sync(0xffffffffu, u == bp)) - 1;
    const float bn = warp_max(-u);
    const int an = __ffs(__ballot_sync(0xffffffffu, -u == bn)) - 1;
    return (bp >= bn) ? ap : kHtHalf + an;
}

__global__ void __launch_bounds__(kHtThreads, 2)
lsh_hash_tc_kernel(const __grid_constant__ CUtensorMap tx, const float *__restrict__ R,
                   int32_t *__restrict__ bucket, int H, int n, int rounds, int tiles_per_cta) {
    extern __shared__ unsigned char ht_raw[];
    const uint32_t mis = smem_u32(ht_raw) & 1023u;
    HtSmem &S = *reinterpret_cast<HtSmem *>(ht_raw + ((1024u - mis) & 1023u));
    const int N = rounds * kHtHalf;
    const int bh = blockIdx.y, h = bh % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tiles = (n + kHtM - 1) / kHtM;
    const int t_first = blockIdx.x * tiles_per_cta;
    const int nt = min(n_tiles, t_first + tiles_per_cta) - t_first;
    if (nt <= 0) return;                          // uniform over the CTA
    const float *Rh = R + (size_t)h * rounds * kHtD * kHtHalf;

    if (tid == 0) {
        for (int i = 0; i < kHtStages; ++i) {
            tc::mbar_init(&S.xfull[i], 1);
            tc::mbar_init(&S.xempty[i], kHtEpiWarps);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&S.tfull[i], 1);
            tc::mbar_init(&S.tempty[i], kHtEpiWarps);
        }
        tc::mbar_fence_init();
        S.fail = 0;
    }
    // B operand tiles (K-major) and column norms; eight loads in flight per thread
    for (int e0 = tid; e0 < N * kHtD; e0 += 8 * kHtThreads) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * kHtThreads;
            v[u] = e < N * kHtD ? __ldg(Rh + e) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * kHtThreads;
            if (e >= N * kHtD) break;
            const int k = e & (kHtHalf - 1), t = (e >> 5) & (kHtD - 1), r = e >> 11;
            const uint32_t off = tc::sw128(r * kHtHalf + k, t >> 3) + (t & 7) * 2;
            S.rf[e] = v[u];
            const __nv_bfloat16 hi = __float2bfloat16_rn(v[u]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v[u] - __bfloat162float(hi));
            *reinterpret_cast<__nv_bfloat16 *>(S.bhi + off) = hi;
            *reinterpret_cast<__nv_bfloat16 *>(S.blo + off) = lo;
        }
    }
    for (int c = tid; c < N; c += kHtThreads) {
        const int r = c / kHtHalf, k = c - r * kHtHalf;
        const float *col = Rh + (size_t)r * kHtD * kHtHalf + k;
        float ss = 0.0f;
#pragma unroll 16
        for (int t = 0; t < kHtD; ++t) ss = fmaf(col[t * kHtHalf], col[t * kHtHalf], ss);
        S.rnorm[c] = sqrtf(ss);
    }
    if (warp == 1) tc::tmem_alloc(&S.tmem_base, 2 * kHtMaxN);
    tc::fence_proxy_async();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = S.tmem_base;
    const volatile int *abort_flag = &S.fail;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            if (*reinterpret_cast<volatile uint32_t *>(&g_force_wait_timeout) != 0u) {
                // test switch: give up before the first load (nothing is in flight)
                raise_error(CRS_DEVERR_TIMEOUT);
                diag_record(K_LSH_HASH, 1, 0u, threadIdx.x, 0u, 0u);
                atomicOr(&S.fail, 1);
            }
            for (int i = 0; i < nt && !*abort_flag; ++i) {
                const int s = i % kHtStages, u = i / kHtStages;
                if (u > 0 && !tc::mbar_wait_bounded(&S.xempty[s], (u - 1) & 1, kHtWaitNs, K_LSH_HASH, 2,
                                                    kHtSuspendNs, false, abort_flag)) {
                    atomicOr(&S.fail, 1);
                    break;
                }
                tc::mbar_arrive_expect_tx(&S.xfull[s], kHtM * 128);
                tc::tma_load_2d(S.x[s], &tx, 0, bh * n + (t_first + i) * kHtM, &S.xfull[s]);
                ++issued;
            }
            // the loads in flight land before the CTA may leave
            for (int i = max(0, issued - kHtStages); i < issued; ++i)
                tc::mbar_wait_bounded(&S.xfull[i % kHtStages], (i / kHtStages) & 1, kHtWaitNs, K_LSH_HASH, 3);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(kHtM, (uint32_t)N, 0, 0);
            int last = -1;
            for (int i = 0; i < nt; ++i) {
                const int s = i % kHtStages, u = i / kHtStages, b = i & 1, v = i >> 1;
                bool ok = tc::mbar_wait_bounded(&S.xfull[s], u & 1, kHtWaitNs, K_LSH_HASH, 4, kHtSuspendNs,
                                                false, abort_flag);
                if (ok && v > 0)
                    ok = tc::mbar_wait_bounded(&S.tempty[b], (v - 1) & 1, kHtWaitNs, K_LSH_HASH, 5, kHtSuspendNs,
                                               false, abort_flag);
                if (!ok) {
                    atomicOr(&S.fail, 1);
                    break;
                }
                tc::fence_after();
                const uint32_t xs = smem_u32(S.x[s]), hs = smem_u32(S.bhi), ls = smem_u32(S.blo);
                const uint32_t d = tmem + (uint32_t)(b * kHtMaxN);
#pragma unroll
                for (int k = 0; k < kHtD / 16; ++k)
                    tc::mma_bf16(d, tc::smem_desc(xs + k * 32, 16, 1024, tc::kLayoutSW128),
                                 tc::smem_desc(hs + k * 32, 16, 1024, tc::kLayoutSW128), idesc, k > 0 ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < kHtD / 16; ++k)
                    tc::mma_bf16(d, tc::smem_desc(xs + k * 32, 16, 1024, tc::kLayoutSW128),
                                 tc::smem_desc(ls + k * 32, 16, 1024, tc::kLayoutSW128), idesc, 1u);
                tc::commit(&S.tfull[b]);
                last = i;
            }
            // the MMAs issued finish before the tensor memory may be freed
            if (last >= 0) tc::mbar_wait_bounded(&S.tfull[last & 1], (last >> 1) & 1, kHtWaitNs, K_LSH_HASH, 6);
        }
    } else {
        // ---------------- epilogue: thread = token row quad * 32 + lane of the tile;
        // the two warps of a quadrant take rounds [r_lo, r_hi)
        const int quad = warp & 3, row = quad * 32 + lane;
        const int half = (warp - 2) >> 2;
        const int r_lo = half == 0 ? 0 : (rounds + 1) / 2, r_hi = half == 0 ? (rounds + 1) / 2 : rounds;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        for (int i = 0; i < nt; ++i) {
            const int s = i % kHtStages, b = i & 1, v = i >> 1;
            const bool ok = tc::mbar_wait_bounded(&S.tfull[b], v & 1, kHtWaitNs, K_LSH_HASH, 7, kHtSuspendNs,
                                                  false, abort_flag);
            if (__any_sync(0xffffffffu, !ok)) {
                if (lane == 0) atomicOr(&S.fail, 1);
                break;
            }
            tc::fence_after();
            const unsigned char *xa = S.x[s];
            const int tok = (t_first + i) * kHtM + row;
            float ss = 0.0f;                      // |x|^2 of this row (16-byte reads of the swizzled tile)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w4 = *reinterpret_cast<const uint4 *>(xa + tc::sw128(row, c));
                const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a0 = __uint_as_float(ww[q] << 16), a1 = __uint_as_float(ww[q] & 0xffff0000u);
                    ss = fmaf(a0, a0, ss);
                    ss = fmaf(a1, a1, ss);
                }
            }
            const float xerr = kHtErr * sqrtf(ss);
            if (r_lo >= r_hi) {                   // nothing for this warp (a single round)
                tc::fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&S.tempty[b]);
            }
            for (int r = r_lo; r < r_hi; ++r) {
                uint32_t uv[32];
                tc::tmem_ld32(tl + (uint32_t)(b * kHtMaxN + r * kHtHalf), uv);
                tc::tmem_ld_wait();
                if (r == r_hi - 1) {              // this warp's reads of the buffer are done
                    tc::fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&S.tempty[b]);
                }
                // The two largest |u~_k| as integer keys: |u~| with its low 6 mantissa bits
                // replaced by (sign, k), so one unsigned max finds value, sign and index
                // (truncating |u~| moves it by less than 2^-17 of itself, added to the margin).
                uint32_t best1 = 0u, best2 = 0u;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const uint32_t key = (uv[k] & 0x7FFFFFC0u) | ((uv[k] >> 26) & 32u) | (uint32_t)k;
                    best2 = max(best2, min(best1, key));
                    best1 = max(best1, key);
                }
                const int k1 = (int)(best1 & 31u), k2 = (int)(best2 & 31u);
                const float m1 = __uint_as_float(best1 & 0xFFFFFFC0u), m2 = __uint_as_float(best2 & 0xFFFFFFC0u);
                int bk = (best1 & 32u) ? kHtHalf + k1 : k1;
                const float E1 = xerr * S.rnorm[r * kHtHalf + k1], E2 = xerr * S.rnorm[r * kHtHalf + k2];
                // written as "not a clear winner" so that a NaN anywhere also takes the exact path
                const bool amb = !((m1 - (E1 + E2) - m1 * 0x1p-16f > m2) && (m1 > E1));
                // exact chains for the undecided tokens of this warp, one token at a time
                uint32_t pend = __ballot_sync(0xffffffffu, amb && tok < n);
                const float *Rr = S.rf + r * kHtD * kHtHalf;
                while (pend) {
                    const int l = __ffs(pend) - 1;
                    pend &= pend - 1;
                    const int e = ht_exact_bucket(xa, quad * 32 + l, Rr, lane);
                    if (lane == l) bk = e;
                }
                if (tok < n) bucket[((size_t)bh * rounds + r) * n + tok] = bk;
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&S.xempty[s]);   // the X stage is free (MMA and fallbacks done)
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 2 * kHtMaxN);
}

// Tiles per CTA so that the grid is about two CTAs per SM.
static int ht_tiles_per_cta(int n, int BH) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        sms = 148;
    }
    const int tiles = (n + kHtM - 1) / kHtM;
    const int per_bh = max(1, min(tiles, (2 * sms) / BH));     // the grid fits one wave
    return (tiles + per_bh - 1) / per_bh;
}

}  // namespace crs
