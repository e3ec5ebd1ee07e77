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
//      tensor memory), and S~ = |x| |R| (the absolute sums that bound every
//      rounding error), for all rounds at once (N = 32 x rounds columns);
//   2. per (token, round): with E_k = 2^-13 S~_k, the largest |u~_k| wins by
//      more than E_k1 + E_k2 over the runner-up and by more than E_k1 over its own
//      negation -> it is the argmax of the chain values as well (see the bound
//      below), and its sign picks the +u or -u half;
//   3. otherwise (a near tie, or all u~ ~ 0) the warp recomputes that token's
//      32 chains exactly, one per lane, in index order, and takes the first
//      maximum as the definition does.
// The bound: |u~_k - u_k| <= |x . (R - R_hi - R_lo)| + (tensor-core
// accumulation) + (chain rounding) <= (2^-16 + 128 * 2^-22 + gamma_64) S_k
// < 5e-5 S_k, S_k = sum_i |x_i| |r_ik| <= 1.01 S~_k (|R| rounded to bf16 at
// most 2^-8 relative); E_k = 2^-13 S~_k >= 1.2e-4 S~_k covers it with a factor
// 2.4.  A winner by more than the two bounds therefore wins in the chain values.
//
// One CTA (4 warps, one token row per thread in the epilogue) walks several
// 128-token tiles of one (batch, head): R is split into its operand tiles once,
// the next X tile is prefetched while the current one is in the epilogue.
#include "common.cuh"
#include "tc.cuh"

namespace crs {

constexpr int kHtM = 128;                 // tokens per tile (MMA M)
constexpr int kHtThreads = 128;
constexpr int kHtHalf = 32;               // b / 2
constexpr int kHtD = 64;
constexpr float kHtErr = 1.220703125e-4f; // 2^-13
constexpr uint64_t kHtWaitNs = 1000000000ull;

__host__ __device__ constexpr size_t ht_smem_bytes(int N) {
    // X double buffer, |X|, three B tiles (R_hi, R_lo, |R|) of N rows, barrier + TMEM slot
    return 2 * 16384 + 16384 + 3 * (size_t)N * 128 + 64;
}

__device__ __forceinline__ float ht_x(const unsigned char *xt, int row, int t) {
    const uint16_t b = *reinterpret_cast<const uint16_t *>(xt + tc::sw128(row, t >> 3) + (t & 7) * 2);
    return __uint_as_float((uint32_t)b << 16);
}

__global__ void __launch_bounds__(kHtThreads, 2)
lsh_hash_tc_kernel(const __nv_bfloat16 *__restrict__ X, const float *__restrict__ R,
                   int32_t *__restrict__ bucket, int H, int n, int rounds, int tiles_per_cta) {
    extern __shared__ unsigned char ht_raw[];
    const uint32_t mis = smem_u32(ht_raw) & 1023u;
    unsigned char *base = ht_raw + ((1024u - mis) & 1023u);
    const int N = rounds * kHtHalf;
    unsigned char *xbuf[2] = {base, base + 16384};
    unsigned char *xab = base + 32768;
    unsigned char *bhi = base + 49152;
    unsigned char *blo = bhi + (size_t)N * 128;
    unsigned char *bab = blo + (size_t)N * 128;
    uint64_t *bar = reinterpret_cast<uint64_t *>(bab + (size_t)N * 128);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 1);

    const int bh = blockIdx.y, h = bh % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tiles = (n + kHtM - 1) / kHtM;
    const int t_first = blockIdx.x * tiles_per_cta;
    const int t_end = min(n_tiles, t_first + tiles_per_cta);
    if (t_first >= t_end) return;                 // uniform over the CTA
    const __nv_bfloat16 *Xb = X + (size_t)bh * n * kHtD;
    const float *Rh = R + (size_t)h * rounds * kHtD * kHtHalf;

    auto load_x = [&](int tile, unsigned char *dst) {
        const int i0 = tile * kHtM;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + u * kHtThreads;
            const int row = e >> 3, ch = e & 7;
            const bool ok = i0 + row < n;
            cp_async16_zfill(dst + tc::sw128(row, ch), Xb + (size_t)(ok ? i0 + row : 0) * kHtD + ch * 8, ok);
        }
        cp_async_commit();
    };
    load_x(t_first, xbuf[0]);

    // B operand tiles, K-major: row r*32 + k holds column k of R_{h,r} (64 values)
    for (int e = tid; e < N * kHtD; e += kHtThreads) {
        const int k = e & (kHtHalf - 1), t = (e >> 5) & (kHtD - 1), r = e >> 11;
        const float v = Rh[e];
        const uint32_t off = tc::sw128(r * kHtHalf + k, t >> 3) + (t & 7) * 2;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        const __nv_bfloat16 ab = __float2bfloat16_rn(fabsf(v));
        *reinterpret_cast<__nv_bfloat16 *>(bhi + off) = hi;
        *reinterpret_cast<__nv_bfloat16 *>(blo + off) = lo;
        *reinterpret_cast<__nv_bfloat16 *>(bab + off) = ab;
    }
    const uint32_t ncols = N * 2 <= 32 ? 32u : (N * 2 <= 64 ? 64u : (N * 2 <= 128 ? 128u : (N * 2 <= 256 ? 256u : 512u)));
    if (warp == 0) tc::tmem_alloc(tslot, ncols);
    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::mbar_fence_init();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t idesc = tc::idesc_bf16_f32(kHtM, (uint32_t)N, 0, 0);

    for (int tile = t_first, it = 0; tile < t_end; ++tile, ++it) {
        unsigned char *xa = xbuf[it & 1];
        cp_async_wait<0>();
        __syncthreads();                          // X tile landed; the last epilogue is done
        // |X|: clear the sign bits
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = tid + u * kHtThreads;
            const uint32_t off = tc::sw128(e >> 3, e & 7);
            uint4 v = *reinterpret_cast<const uint4 *>(xa + off);
            v.x &= 0x7fff7fffu; v.y &= 0x7fff7fffu; v.z &= 0x7fff7fffu; v.w &= 0x7fff7fffu;
            *reinterpret_cast<uint4 *>(xab + off) = v;
        }
        tc::fence_proxy_async();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        if (tid == 0) {
            const uint32_t xs = smem_u32(xa), xb = smem_u32(xab);
            const uint32_t hs = smem_u32(bhi), ls = smem_u32(blo), as = smem_u32(bab);
#pragma unroll
            for (int k = 0; k < kHtD / 16; ++k)
                tc::mma_bf16(tmem, tc::smem_desc(xs + k * 32, 16, 1024, tc::kLayoutSW128),
                             tc::smem_desc(hs + k * 32, 16, 1024, tc::kLayoutSW128), idesc, k > 0 ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < kHtD / 16; ++k)
                tc::mma_bf16(tmem, tc::smem_desc(xs + k * 32, 16, 1024, tc::kLayoutSW128),
                             tc::smem_desc(ls + k * 32, 16, 1024, tc::kLayoutSW128), idesc, 1u);
#pragma unroll
            for (int k = 0; k < kHtD / 16; ++k)
                tc::mma_bf16(tmem + (uint32_t)N, tc::smem_desc(xb + k * 32, 16, 1024, tc::kLayoutSW128),
                             tc::smem_desc(as + k * 32, 16, 1024, tc::kLayoutSW128), idesc, k > 0 ? 1u : 0u);
            tc::commit(bar);
        }
        // the other buffer was last read by the previous tile's MMAs, which completed
        if (tile + 1 < t_end) load_x(tile + 1, xbuf[(it + 1) & 1]);
        const bool ok = tc::mbar_wait_bounded(bar, (uint32_t)(it & 1), kHtWaitNs, K_LSH_HASH, 1, 10000u, true);
        if (__syncthreads_or(!ok)) {
            tc::mbar_wait_bounded(bar, (uint32_t)(it & 1), kHtWaitNs, K_LSH_HASH, 2);   // drain
            cp_async_wait<0>();
            break;
        }
        tc::fence_after();

        const int row = warp * 32 + lane;
        const int i = tile * kHtM + row;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        for (int r = 0; r < rounds; ++r) {
            uint32_t uv[32], sv[32];
            tc::tmem_ld32(trow + (uint32_t)(r * kHtHalf), uv);
            tc::tmem_ld32(trow + (uint32_t)(N + r * kHtHalf), sv);
            tc::tmem_ld_wait();
            // the two largest |u~_k| with their absolute sums (error scales)
            float m1 = -1.0f, m2 = -1.0f, s1 = 0.0f, s2 = 0.0f, u1 = 0.0f;
            int k1 = 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float uk = __uint_as_float(uv[k]), sk = __uint_as_float(sv[k]);
                const float a = fabsf(uk);
                if (a > m1) { m2 = m1; s2 = s1; m1 = a; s1 = sk; k1 = k; u1 = uk; }
                else if (a > m2) { m2 = a; s2 = sk; }
            }
            // every other entry of [u~ ; -u~] is at most m2 (or -m1 for the winner's own
            // negation); the winner is certain when it leads both by the two bounds
            int bk = u1 > 0.0f ? k1 : kHtHalf + k1;
            const float E1 = kHtErr * s1, E2 = kHtErr * s2;
            const bool amb = (m2 >= m1 - (E1 + E2)) || (m1 <= E1);
            // exact chains for the undecided tokens of this warp, one token at a time
            uint32_t pend = __ballot_sync(0xffffffffu, amb && i < n);
            const float *Rr = Rh + (size_t)r * kHtD * kHtHalf;
            while (pend) {
                const int l = __ffs(pend) - 1;
                pend &= pend - 1;
                const int rl = warp * 32 + l;
                float rv[kHtD];                       // column `lane` of R_{h,r}, all loads in flight
#pragma unroll
                for (int t = 0; t < kHtD; ++t) rv[t] = __ldg(Rr + t * kHtHalf + lane);
                float u = 0.0f;
#pragma unroll
                for (int t = 0; t < kHtD; ++t) u = __fmaf_rn(ht_x(xa, rl, t), rv[t], u);
                const float bp = warp_max(u);
                const int ap = __ffs(__ballot_sync(0xffffffffu, u == bp)) - 1;
                const float bn = warp_max(-u);
                const int an = __ffs(__ballot_sync(0xffffffffu, -u == bn)) - 1;
                if (lane == l) bk = (bp >= bn) ? ap : kHtHalf + an;
            }
            if (i < n) bucket[((size_t)bh * rounds + r) * n + i] = bk;
        }
        tc::fence_before();
    }
    cp_async_wait<0>();
    tc::fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, ncols);
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
