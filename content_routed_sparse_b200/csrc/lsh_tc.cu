// K3 on the tensor cores: chunked LSH attention for bf16, d = 64, chunk m = 128.
//
// [P1] PaperTrace 2.1.1 §2.1-2.2 (sorted array cut into chunks of m slots; a
// chunk attends to itself and the previous chunk; edges need the same bucket
// and are judged on original positions), "重复候选和归一化" (a pair counts once).
//
// One CTA (8 warps, two CTAs resident per SM) per (chunk, round, batch*head):
//   1. per key slot of the 256-slot window (previous + own chunk): original
//      position (via perm), bucket, earlier-round (bucket, chunk) codes;
//   2. 16-byte cp.async gathers of the 256 rows of Q(=K) and V into
//      128B-swizzled shared tiles; the own chunk's 128 rows are also the
//      query tile (A operand);
//   3. one thread issues S = Q K^T (M=128, N=256, K=64) into TMEM;
//   4. the masked softmax reads S from TMEM (pass 1: row maxima, warpgroup g
//      owns columns [128g, 128g+128)).  Slots are sorted by (bucket, position),
//      so the keys of a query that share its bucket and precede it form ONE
//      contiguous column range [run start, own slot]: the bucket, causal and
//      padding masks are a range test, and 32-column chunks outside the range
//      are skipped warp-uniformly (tcgen05.ld is warp-collective).  Pairs seen
//      in an earlier round are masked per element (specialised per round).
//      Pass 2 writes P = exp(S - max) for one 128-key half at a time into
//      shared memory as a bf16 value plus a bf16 residual (K-major tiles),
//      reusing the K tile's space (S is complete by then);
//   5. after each half, one thread issues O += P_hi V_half + P_lo V_half
//      (M=128, N=64, V as an MN-major operand) into TMEM columns [0, 64),
//      which the first half's S no longer needs.  When every row bound is
//      small and V is fp16-representable (the usual case), the CTA instead
//      converts its V tile to fp16, writes P = 2^(S - bound + 15) for all 256
//      keys as fp16 in one sweep and issues a single fp16 chain O = P V;
//   6. the epilogue divides by the row sum and writes o_r and lse_r at the
//      ORIGINAL position; lsh_combine_kernel merges the rounds.
// Resources per CTA: 256 TMEM columns, ~107 KB shared memory, 256 threads,
// so two CTAs share an SM and overlap each other's latency.
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "tc.cuh"

namespace crs {

constexpr int kTcM = 128;        // queries per chunk
constexpr int kTcN = 256;        // keys: previous + own chunk
constexpr int kTcD = 64;
constexpr int kTcThreads = 256;  // 2 warpgroups
constexpr uint32_t kTcCols = 256;
constexpr uint64_t kTcWaitNs = 1000000000ull;   // 1 s: a wait that long means a fault
constexpr int kBktBefore = -1;                  // absent slot before the sequence
constexpr int kBktAfter = 0x7fffffff;           // absent slot after the sequence
constexpr float kTcBoundMax = 48.0f;            // single pass while 2^(-2 bound) stays normal
constexpr float kTcBoundMax16 = 14.0f;          // fp16 P while 2^(15 - 2 bound) stays fp16-normal
constexpr float kTcAccBoundMax = 63.0f;         // fixed-shift round accumulation while 2^(-2 bound) is normal

struct LshTcSmem {
    // K tile (rows = keys; rows 128..255 = Q tile) until S is computed, then
    // the P buffer of one 128-key half: hi[2 blocks], lo[2 blocks] (K-major)
    unsigned char kp[4][kTcM * 128];
    unsigned char v[kTcN * 128];        // V tile, rows = keys
    int kpos[kTcN];
    union {                             // lifetimes do not overlap:
        int kbkt[kTcN];                 //   buckets (nondecreasing), until the runs are known
        uint32_t mbits[kTcN / 32][kTcM];//   pass-1 masks: [32-key chunk][row]
    } u1;
    union {
        uint32_t krun[kTcN];            //   bucket run of a key: first slot | (last slot with
                                        //   position < valid_len) << 16, read before pass 1
        float rowsum[2][kTcM];          //   written after pass 2
    } u2;
    int kcode[kMaxRounds - 1][kTcN];    // earlier rounds: bucket * C1 + chunk + 1
    float kscale[kTcN];                 // scale * log2(e) / |k_j|
    float rowmax[2][kTcM];
    float rbound[kTcM];                 // scale |q_i| in log2 units (normalised keys)
    uint64_t bar[3];
    uint32_t tmem_base;
};

// o[0..3] += (a, b, c, d) in global memory, one vector reduction (no return value)
__device__ __forceinline__ void red_add_v4(float *o, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(o), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {   // 2^x, PTX ex2.approx (rel. err ~2^-22)
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

struct LshTcRow {
    int row, jq, lo, hi, pos_i;
    bool qvalid, excl_self;
};

// Pass 1 for a query row with R earlier rounds: warpgroup wg scans columns
// [128 wg, 128 wg + 128); stores the per-chunk masks, returns the partial max.
template <int R>
__device__ __forceinline__ float lsh_tc_pass1(LshTcSmem &S, const LshTcRow &q, uint32_t trow, int wg) {
    int code_i[R > 0 ? R : 1];
#pragma unroll
    for (int rr = 0; rr < R; ++rr) code_i[rr] = S.kcode[rr][q.jq];
    float mx = -INFINITY;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        const int col0 = wg * 128 + cc * 32;
        const bool need = q.qvalid && col0 <= q.hi && col0 + 31 >= q.lo;
        uint32_t mb = 0;
        if (__any_sync(0xffffffffu, need)) {
            uint32_t v[32];
            tc::tmem_ld32(trow + col0, v);
            tc::tmem_ld_wait();
            if (need) {
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const int j = col0 + t;
                    bool ok = j >= q.lo && j <= q.hi && !(q.excl_self && j == q.jq);
#pragma unroll
                    for (int rr = 0; rr < R; ++rr)
                        ok = ok && ((uint32_t)(code_i[rr] - S.kcode[rr][j]) > 1u);
                    if (ok) {
                        mx = fmaxf(mx, __uint_as_float(v[t]) * S.kscale[j]);
                        mb |= 1u << t;
                    }
                }
            }
        }
        S.u1.mbits[col0 >> 5][q.row] = mb;
    }
    return mx;
}

// Pass 2 for the 64 keys [col0, col0 + 64) of one row: P into K-block `blk`
// of the P buffer (value and residual); returns the partial row sum.
__device__ __forceinline__ float lsh_tc_pass2(LshTcSmem &S, const LshTcRow &q, uint32_t trow,
                                              int col0, int blk, float M) {
    float sum = 0.0f;
    unsigned char *p_hi = S.kp[blk];
    unsigned char *p_lo = S.kp[2 + blk];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int c0 = col0 + cc * 32;
        const uint32_t mb = S.u1.mbits[c0 >> 5][q.row];
        uint32_t hi[16], lo[16];
        if (__any_sync(0xffffffffu, mb != 0u)) {
            uint32_t v[32];
            tc::tmem_ld32(trow + c0, v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int t2 = 0; t2 < 16; ++t2) {
                float pv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int t = t2 * 2 + e;
                    pv[e] = ((mb >> t) & 1u) ? ex2_approx(__uint_as_float(v[t]) * S.kscale[c0 + t] - M)
                                             : 0.0f;
                    sum += pv[e];
                }
                __nv_bfloat162 h2 = __floats2bfloat162_rn(pv[0], pv[1]);
                const float2 hf = __bfloat1622float2(h2);
                __nv_bfloat162 l2 = __floats2bfloat162_rn(pv[0] - hf.x, pv[1] - hf.y);
                hi[t2] = *reinterpret_cast<uint32_t *>(&h2);
                lo[t2] = *reinterpret_cast<uint32_t *>(&l2);
            }
        } else {
#pragma unroll
            for (int t2 = 0; t2 < 16; ++t2) hi[t2] = lo[t2] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t off = tc::sw128(q.row, cc * 4 + u);
            *reinterpret_cast<uint4 *>(p_hi + off) =
                make_uint4(hi[u * 4], hi[u * 4 + 1], hi[u * 4 + 2], hi[u * 4 + 3]);
            *reinterpret_cast<uint4 *>(p_lo + off) =
                make_uint4(lo[u * 4], lo[u * 4 + 1], lo[u * 4 + 2], lo[u * 4 + 3]);
        }
    }
    return sum;
}

// Bits t of the 32 columns [c0, c0 + 32) with lo <= c0 + t <= hi.
__device__ __forceinline__ uint32_t range_bits(int lo, int hi, int c0) {
    const int a = lo - c0, b = hi - c0;
    if (b < 0 || a > 31 || a > b) return 0u;
    const uint32_t low = a <= 0 ? 0xffffffffu : (0xffffffffu << a);
    const uint32_t high = b >= 31 ? 0xffffffffu : ((2u << b) - 1u);
    return low & high;
}

// Single pass for normalised keys: every logit of row i is at most
// M_i = scale |q_i| (log2 units), so P = 2^(S - M_i) needs no row maximum.
// Keys [col0, col0 + 64) of the row: masks (range bits, earlier-round
// pairs), P into K-block `blk` of the P buffer (value and residual); returns
// the partial row sum.  NR = earlier rounds (R < 0: runtime count r).
template <int NR>
__device__ __forceinline__ float lsh_tc_fused(LshTcSmem &S, const LshTcRow &q, uint32_t trow,
                                              int col0, int blk, float M, int r) {
    const int R = NR >= 0 ? NR : r;
    float sum = 0.0f;
    unsigned char *p_hi = S.kp[blk];
    unsigned char *p_lo = S.kp[2 + blk];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int c0 = col0 + cc * 32;
        uint32_t mb = q.qvalid ? range_bits(q.lo, q.hi, c0) : 0u;
        if (q.excl_self && q.jq >= c0 && q.jq < c0 + 32) mb &= ~(1u << (q.jq - c0));
        uint32_t hi[16], lo[16];
        if (__any_sync(0xffffffffu, mb != 0u)) {
            uint32_t v[32];
            tc::tmem_ld32(trow + c0, v);
            // pairs met in an earlier round (same bucket, key chunk = query chunk or the one before)
#pragma unroll
            for (int rr = 0; rr < (NR >= 0 ? NR : kMaxRounds - 1); ++rr) {
                if (NR < 0 && rr >= R) break;
                const int4 *kc = reinterpret_cast<const int4 *>(&S.kcode[rr][c0]);
                const int ci = S.kcode[rr][q.jq];
                uint32_t dup = 0u;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int4 k4 = kc[u];
                    dup |= ((uint32_t)(ci - k4.x) <= 1u ? 1u : 0u) << (4 * u);
                    dup |= ((uint32_t)(ci - k4.y) <= 1u ? 1u : 0u) << (4 * u + 1);
                    dup |= ((uint32_t)(ci - k4.z) <= 1u ? 1u : 0u) << (4 * u + 2);
                    dup |= ((uint32_t)(ci - k4.w) <= 1u ? 1u : 0u) << (4 * u + 3);
                }
                mb &= ~dup;
            }
            tc::tmem_ld_wait();
            const float4 *ks = reinterpret_cast<const float4 *>(&S.kscale[c0]);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 k4 = ks[u];
                const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
                float pv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = 4 * u + e;
                    pv[e] = ((mb >> t) & 1u) ? ex2_approx(fmaf(__uint_as_float(v[t]), kk[e], -M)) : 0.0f;
                    sum += pv[e];
                }
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(pv[2 * e2], pv[2 * e2 + 1]);
                    const float2 hf = __bfloat1622float2(h2);
                    __nv_bfloat162 l2 = __floats2bfloat162_rn(pv[2 * e2] - hf.x, pv[2 * e2 + 1] - hf.y);
                    hi[2 * u + e2] = *reinterpret_cast<uint32_t *>(&h2);
                    lo[2 * u + e2] = *reinterpret_cast<uint32_t *>(&l2);
                }
            }
        } else {
#pragma unroll
            for (int t2 = 0; t2 < 16; ++t2) hi[t2] = lo[t2] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t off = tc::sw128(q.row, cc * 4 + u);
            *reinterpret_cast<uint4 *>(p_hi + off) =
                make_uint4(hi[u * 4], hi[u * 4 + 1], hi[u * 4 + 2], hi[u * 4 + 3]);
            *reinterpret_cast<uint4 *>(p_lo + off) =
                make_uint4(lo[u * 4], lo[u * 4 + 1], lo[u * 4 + 2], lo[u * 4 + 3]);
        }
    }
    return sum;
}

// Single pass with fp16 P for all 256 keys at once (the CTA has checked that
// every bound is at most kTcBoundMax16 and that every V value is below 2^16 in
// magnitude, so its fp16 copy is exact from 2^-14 up and within 2^-25 below):
// P = 2^(S - M) with M = bound - 15 lies in [2^(15 - 2 bound), 2^15], inside
// the fp16 normal range, so one rounding (relative 2^-12) is the only error P
// adds.  Warpgroup wg writes keys [128 wg, 128 wg + 128) = P blocks 2wg, 2wg+1.
// The earlier-round pair test is folded into each element's predicate.
template <int NR>
__device__ __forceinline__ float lsh_tc_fused16(LshTcSmem &S, const LshTcRow &q, uint32_t trow, int wg,
                                                float M, int r) {
    constexpr int NRR = NR >= 0 ? NR : kMaxRounds - 1;
    const int R = NR >= 0 ? NR : r;
    int ci[NRR > 0 ? NRR : 1];
#pragma unroll
    for (int rr = 0; rr < NRR; ++rr) ci[rr] = rr < R ? S.kcode[rr][q.jq] : 0;
    float2 sum2 = make_float2(0.0f, 0.0f);
    const float2 negM = make_float2(-M, -M);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        const int c0 = wg * 128 + cc * 32;
        uint32_t mb = q.qvalid ? range_bits(q.lo, q.hi, c0) : 0u;
        if (q.excl_self && q.jq >= c0 && q.jq < c0 + 32) mb &= ~(1u << (q.jq - c0));
        uint32_t ph[16];
        if (__any_sync(0xffffffffu, mb != 0u)) {
            uint32_t v[32];
            tc::tmem_ld32(trow + c0, v);
            tc::tmem_ld_wait();
            const float4 *ks = reinterpret_cast<const float4 *>(&S.kscale[c0]);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 k4 = ks[u];
                bool ok[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) ok[e] = (mb >> (4 * u + e)) & 1u;
#pragma unroll
                for (int rr = 0; rr < NRR; ++rr) {
                    if (NR < 0 && rr >= R) break;
                    const int4 kc = reinterpret_cast<const int4 *>(&S.kcode[rr][c0])[u];
                    ok[0] = ok[0] && (uint32_t)(ci[rr] - kc.x) > 1u;
                    ok[1] = ok[1] && (uint32_t)(ci[rr] - kc.y) > 1u;
                    ok[2] = ok[2] && (uint32_t)(ci[rr] - kc.z) > 1u;
                    ok[3] = ok[3] && (uint32_t)(ci[rr] - kc.w) > 1u;
                }
                const float2 a = __ffma2_rn(make_float2(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1])),
                                            make_float2(k4.x, k4.y), negM);
                const float2 b = __ffma2_rn(make_float2(__uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3])),
                                            make_float2(k4.z, k4.w), negM);
                const float2 p01 = make_float2(ok[0] ? ex2_approx(a.x) : 0.0f, ok[1] ? ex2_approx(a.y) : 0.0f);
                const float2 p23 = make_float2(ok[2] ? ex2_approx(b.x) : 0.0f, ok[3] ? ex2_approx(b.y) : 0.0f);
                sum2 = __fadd2_rn(sum2, p01);
                sum2 = __fadd2_rn(sum2, p23);
                const __half2 h01 = __floats2half2_rn(p01.x, p01.y);
                const __half2 h23 = __floats2half2_rn(p23.x, p23.y);
                ph[2 * u] = *reinterpret_cast<const uint32_t *>(&h01);
                ph[2 * u + 1] = *reinterpret_cast<const uint32_t *>(&h23);
            }
        } else {
#pragma unroll
            for (int t2 = 0; t2 < 16; ++t2) ph[t2] = 0u;
        }
        unsigned char *pb = S.kp[2 * wg + (cc >> 1)];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4 *>(pb + tc::sw128(q.row, (cc & 1) * 4 + u)) =
                make_uint4(ph[u * 4], ph[u * 4 + 1], ph[u * 4 + 2], ph[u * 4 + 3]);
    }
    return sum2.x + sum2.y;
}

// O (TMEM columns [0, 64)) = P V over all 256 keys, fp16 operands (P K-major
// in blocks of 64 keys, V MN-major), one chain of 16 MMAs.
__device__ __forceinline__ void lsh_tc_issue_pv16(LshTcSmem &S, uint32_t tmem) {
    constexpr uint32_t idesc = tc::idesc_f16_f32(kTcM, kTcD, 0, 1);
    const uint32_t vbase = smem_u32(S.v);
#pragma unroll
    for (int kk = 0; kk < kTcN / 16; ++kk) {
        const uint64_t a = tc::smem_desc(smem_u32(S.kp[kk >> 2]) + (kk & 3) * 32, 16, 1024, tc::kLayoutSW128);
        const uint64_t bd = tc::smem_desc(vbase + kk * 16 * 128, 32768, 1024, tc::kLayoutSW128);
        tc::mma_bf16(tmem, a, bd, idesc, kk > 0 ? 1u : 0u);
    }
}

// O (TMEM columns [0, 64)) += P_hi V_half + P_lo V_half for keys [128 half, +128).
__device__ __forceinline__ void lsh_tc_issue_pv(LshTcSmem &S, uint32_t tmem, int half,
                                                bool first) {
    constexpr uint32_t idesc = tc::idesc_bf16_f32(kTcM, kTcD, 0, 1);
    const uint32_t vbase = smem_u32(S.v);
    uint32_t acc = first ? 0u : 1u;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
            const uint32_t pbase = smem_u32(S.kp[part * 2 + blk]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t a = tc::smem_desc(pbase + k * 32, 16, 1024, tc::kLayoutSW128);
                const uint64_t bd = tc::smem_desc(vbase + (half * 128 + blk * 64 + k * 16) * 128,
                                                  32768, 1024, tc::kLayoutSW128);
                tc::mma_bf16(tmem, a, bd, idesc, acc);
                acc = 1u;
            }
        }
    }
}

// One (chunk c, round r, batch*head bh) item of the CTA; false when a wait gave up.
// ph holds the parity each barrier completes with next.
__device__ __forceinline__ bool lsh_tc_item(LshTcSmem &S, uint32_t tmem, uint32_t (&ph)[3],
                                            const __nv_bfloat16 *__restrict__ QK, const __nv_bfloat16 *__restrict__ V,
                                            const int32_t *__restrict__ bucket, const int32_t *__restrict__ perm,
                                            const int32_t *__restrict__ inv_perm, const int32_t *__restrict__ valid_len,
                                            float *__restrict__ o_ws, float *__restrict__ lse_ws, float *__restrict__ acc_O,
                                            float *__restrict__ acc_L, float *__restrict__ acc_M, int H, int BH, int n,
                                            int rounds, int causal, int no_self, int key_norm, float scale_log2,
                                            int c, int r, int bh) {
    const int b = bh / H;
    const int vl = valid_len ? valid_len[b] : n;
    __syncthreads();                              // the previous item's reads of shared memory are done
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int C1 = (n + kTcM - 1) / kTcM + 1;      // chunk-code stride
    const size_t seg_r = ((size_t)bh * rounds + r) * n;

    // ---- 1. key metadata; window key j = tid is slot (c-1)*128 + j
    {
        const int j = tid;
        const int s = (c - 1) * kTcM + j;
        int pos = -1, bk = (s < 0) ? kBktBefore : kBktAfter;
        if (s >= 0 && s < n) {
            pos = perm[seg_r + s];
            if (pos < 0 || pos >= n) {
                raise_error(CRS_DEVERR_INDEX);
                pos = -1;
            } else {
                bk = bucket[seg_r + pos];
            }
        }
        S.kpos[j] = pos;
        S.u1.kbkt[j] = bk;
        for (int rr = 0; rr < r; ++rr) {
            int code = -8;                        // matches no query code
            if (pos >= 0) {
                const size_t sg = ((size_t)bh * rounds + rr) * n;
                code = bucket[sg + pos] * C1 + inv_perm[sg + pos] / kTcM + 1;
            }
            S.kcode[rr][j] = code;
        }
    }
    __syncthreads();

    // ---- 2. gather K (= Q) and V rows; bucket runs of the window
    {
        const __nv_bfloat16 *Qb = QK + (size_t)bh * n * kTcD;
        const __nv_bfloat16 *Vb = V + (size_t)bh * n * kTcD;
#pragma unroll
        for (int u = 0; u < (kTcN * 8) / kTcThreads; ++u) {
            const int e = tid + u * kTcThreads;
            const int j = e >> 3, ch = e & 7;
            const int pos = S.kpos[j];
            const bool ok = pos >= 0;
            const size_t off = ok ? (size_t)pos * kTcD + ch * 8 : 0;
            cp_async16_zfill(&S.kp[0][0] + tc::sw128(j, ch), Qb + off, ok);
            cp_async16_zfill(S.v + tc::sw128(j, ch), Vb + off, ok);
        }
        cp_async_commit();
    }
    {
        // the window's buckets are nondecreasing: binary searches give the run
        const int j = tid, bk = S.u1.kbkt[j];
        int a = 0, z = j;                         // first index with kbkt >= bk
        while (a < z) {
            const int mid = (a + z) >> 1;
            if (S.u1.kbkt[mid] < bk) a = mid + 1; else z = mid;
        }
        const int run0 = a;
        a = j;                                    // last index in the run with pos < vl
        z = kTcN - 1;
        while (a < z) {
            const int mid = (a + z + 1) >> 1;
            if (S.u1.kbkt[mid] == bk && S.kpos[mid] < vl) a = mid; else z = mid - 1;
        }
        S.u2.krun[j] = (uint32_t)run0 | ((uint32_t)a << 16);
    }
    cp_async_wait<0>();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    bool big = false, no16 = false;
    uint4 v16[8];                                 // row j of V as fp16, stored if the CTA takes fp16 P
    {
        const int j = tid;
        uint32_t vbad = 0u;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const uint4 w = *reinterpret_cast<const uint4 *>(S.v + tc::sw128(j, ch));
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            uint32_t hh[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                // |bf16| >= 2^16 (or Inf / NaN) does not convert exactly: bit 15 of each half of
                // (w & 0x7fff7fff) + 0x38803880 is set exactly when the half's magnitude bits reach 0x4780
                vbad |= ((ww[t] & 0x7fff7fffu) + 0x38803880u) & 0x80008000u;
                const __half2 h = __floats2half2_rn(__uint_as_float(ww[t] << 16), __uint_as_float(ww[t] & 0xffff0000u));
                hh[t] = *reinterpret_cast<const uint32_t *>(&h);
            }
            v16[ch] = make_uint4(hh[0], hh[1], hh[2], hh[3]);
        }
        no16 = vbad != 0u;
        float ss = 0.0f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const uint4 v = *reinterpret_cast<const uint4 *>(&S.kp[0][0] + tc::sw128(j, ch));
            const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 f = __bfloat1622float2(p2[t]);
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
        const float inv = key_norm ? (ss > 0.0f ? rsqrtf(ss) : 0.0f) : 1.0f;
        S.kscale[j] = inv * scale_log2;
        // own-chunk row: with normalised keys its logits are at most scale |q| (log2 units)
        if (j >= kTcM) {
            const float bound = sqrtf(ss) * fabsf(scale_log2);
            S.rowmax[1][j - kTcM] = bound;
            S.rbound[j - kTcM] = bound;
            big = bound > kTcBoundMax;
            no16 = no16 || !(bound <= kTcBoundMax16);
        }
    }
    // single pass unless keys are raw or some bound is so large that 2^(S - bound) could underflow;
    // fp16 P when, in addition, all of V is exact in fp16 and 2^(S - bound + 15) stays fp16-normal
    const bool single = key_norm && !__syncthreads_or(big);
    const bool use16 = single && !__syncthreads_or(no16);
    if (use16) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4 *>(S.v + tc::sw128(tid, ch)) = v16[ch];
    }
    tc::fence_proxy_async();

    // ---- 3. S = Q K^T into TMEM columns [0, 256)
    if (tid == 0) {
        constexpr uint32_t idesc = tc::idesc_bf16_f32(kTcM, kTcN, 0, 0);
        const uint32_t kbase = smem_u32(&S.kp[0][0]);
#pragma unroll
        for (int k = 0; k < kTcD / 16; ++k) {
            const uint64_t a = tc::smem_desc(kbase + kTcM * 128 + k * 32, 16, 1024, tc::kLayoutSW128);
            const uint64_t bd = tc::smem_desc(kbase + k * 32, 16, 1024, tc::kLayoutSW128);
            tc::mma_bf16(tmem, a, bd, idesc, k > 0 ? 1u : 0u);
        }
        tc::commit(&S.bar[0]);
    }
    bool ok_wait = tc::mbar_wait_bounded(&S.bar[0], ph[0], kTcWaitNs, K_LSH_ATTN_TC, 1, 10000u, true);
    if (__syncthreads_or(!ok_wait)) {
        tc::mbar_wait_bounded(&S.bar[0], ph[0], kTcWaitNs, K_LSH_ATTN_TC, 2);   // let the MMA drain
        return false;
    }
    ph[0] ^= 1u;
    tc::fence_after();

    {
        const int wg = warp >> 2, quad = warp & 3;
        LshTcRow q;
        q.row = quad * 32 + lane;
        q.jq = kTcM + q.row;
        q.pos_i = S.kpos[q.jq];
        q.qvalid = q.pos_i >= 0 && q.pos_i < vl;
        const uint32_t run = S.u2.krun[q.jq];
        q.lo = (int)(run & 0xffffu);
        q.hi = causal ? (no_self ? q.jq - 1 : q.jq) : (int)(run >> 16);
        q.excl_self = (!causal) && no_self;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);

        // ---- 4a. the exponent shift M: the row bound (single pass), or pass 1's
        // masks and row maxima
        float M;
        if (use16) {
            M = S.rowmax[1][q.row] - 15.0f;
        } else if (single) {
            M = S.rowmax[1][q.row];
        } else {
            float mx;
            switch (r) {
                case 0: mx = lsh_tc_pass1<0>(S, q, trow, wg); break;
                case 1: mx = lsh_tc_pass1<1>(S, q, trow, wg); break;
                case 2: mx = lsh_tc_pass1<2>(S, q, trow, wg); break;
                case 3: mx = lsh_tc_pass1<3>(S, q, trow, wg); break;
                case 4: mx = lsh_tc_pass1<4>(S, q, trow, wg); break;
                case 5: mx = lsh_tc_pass1<5>(S, q, trow, wg); break;
                case 6: mx = lsh_tc_pass1<6>(S, q, trow, wg); break;
                default: mx = lsh_tc_pass1<7>(S, q, trow, wg); break;
            }
            __syncthreads();                     // row bounds in rowmax[1] are no longer needed
            S.rowmax[wg][q.row] = mx;
            __syncthreads();
            M = fmaxf(S.rowmax[0][q.row], S.rowmax[1][q.row]);
        }

        // ---- 4b/5. fp16 P: all 256 keys, then O = P V in one chain; otherwise per
        // 128-key half: P (value + residual) into the buffer, then O += P V_half
        float sum = 0.0f;
        if (use16) {
            switch (r) {
                case 0: sum = lsh_tc_fused16<0>(S, q, trow, wg, M, r); break;
                case 1: sum = lsh_tc_fused16<1>(S, q, trow, wg, M, r); break;
                case 2: sum = lsh_tc_fused16<2>(S, q, trow, wg, M, r); break;
                case 3: sum = lsh_tc_fused16<3>(S, q, trow, wg, M, r); break;
                default: sum = lsh_tc_fused16<-1>(S, q, trow, wg, M, r); break;
            }
            tc::fence_proxy_async();
            tc::fence_before();
            __syncthreads();
            tc::fence_after();
            if (tid == 0) {
                lsh_tc_issue_pv16(S, tmem);
                tc::commit(&S.bar[2]);
            }
        }
        for (int half = 0; half < 2 && !use16; ++half) {
            if (half == 1) {
                // the buffer is free once the first half's P.V has completed
                ok_wait = tc::mbar_wait_bounded(&S.bar[1], ph[1], kTcWaitNs, K_LSH_ATTN_TC, 3);
                if (__syncthreads_or(!ok_wait)) return false;
                ph[1] ^= 1u;
                tc::fence_after();
            }
            const int col0 = half * 128 + wg * 64;
            if (single) {
                switch (r) {
                    case 0: sum += lsh_tc_fused<0>(S, q, trow, col0, wg, M, r); break;
                    case 1: sum += lsh_tc_fused<1>(S, q, trow, col0, wg, M, r); break;
                    case 2: sum += lsh_tc_fused<2>(S, q, trow, col0, wg, M, r); break;
                    case 3: sum += lsh_tc_fused<3>(S, q, trow, col0, wg, M, r); break;
                    default: sum += lsh_tc_fused<-1>(S, q, trow, col0, wg, M, r); break;
                }
            } else {
                sum += lsh_tc_pass2(S, q, trow, col0, wg, M);
            }
            tc::fence_proxy_async();
            tc::fence_before();
            __syncthreads();
            tc::fence_after();
            if (tid == 0) {
                lsh_tc_issue_pv(S, tmem, half, half == 0);
                tc::commit(&S.bar[1 + half]);
            }
        }
        S.u2.rowsum[wg][q.row] = sum;
        ok_wait = tc::mbar_wait_bounded(&S.bar[2], ph[2], kTcWaitNs, K_LSH_ATTN_TC, 4);
        if (__syncthreads_or(!ok_wait)) return false;
        ph[2] ^= 1u;
        tc::fence_after();

        // ---- 6. epilogue: warpgroup wg writes output columns [32 wg, 32 wg + 32).
        // tcgen05.ld is warp-collective: every lane loads; rows without a
        // position (a partial last chunk) only skip the stores.
        uint32_t v[32];
        tc::tmem_ld32(trow + wg * 32, v);
        tc::tmem_ld_wait();
        // Round accumulation with a fixed shift (normalised keys): every logit of row i
        // is at most bound_i = scale |q_i| (log2 units), the same value in every round,
        // so the rounds' numerators sum_j 2^(s_ij - bound_i) v_j and denominators add up
        // directly; with bound_i <= 63 no term leaves the fp32 normal range.  This
        // round's terms were taken relative to M (bound - 15 for fp16 P, bound in the
        // single pass, the row maximum in the two-pass path): they are rescaled by
        // 2^(M - bound).  Pairs are counted in their first round only, so the sums are
        // over the union of the rounds' candidates ([P1] "重复候选和归一化").  Rows with
        // a larger bound keep the per-round (o_r, lse_r) form, merged afterwards.
        bool stored = false, acc_row = false;
        float f = 0.0f;
        if (acc_O && q.pos_i >= 0) {
            const float bnd = S.rbound[q.row];
            if (bnd <= kTcAccBoundMax) {
                const float L = S.u2.rowsum[0][q.row] + S.u2.rowsum[1][q.row];
                const size_t orow = (size_t)bh * n + q.pos_i;
                if (q.qvalid && L > 0.0f) {
                    f = use16 ? 0x1p-15f : (single ? 1.0f : exp2f(M - bnd));
                    acc_row = true;
                    if (wg == 0) atomicAdd(acc_L + orow, L * f);
                }
                if (wg == 0) acc_M[orow] = bnd;
                stored = true;
            } else if (wg == 0) {
                acc_M[(size_t)bh * n + q.pos_i] = INFINITY;   // merged from the per-round form
            }
        }
        // The accumulated rows go through shared memory (the P buffer is free once P.V has
        // completed): each warp stages its 32 rows x 32 columns, then every vector reduction
        // covers 128 contiguous bytes of one row, four rows per instruction.
        const uint32_t acc_mask = __ballot_sync(0xffffffffu, acc_row);
        if (acc_mask) {
            unsigned char *tile = &S.kp[0][0] + warp * 4096;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                *reinterpret_cast<float4 *>(tile + tc::sw128(lane, u)) =
                    make_float4(__uint_as_float(v[u * 4 + 0]) * f, __uint_as_float(v[u * 4 + 1]) * f,
                                __uint_as_float(v[u * 4 + 2]) * f, __uint_as_float(v[u * 4 + 3]) * f);
            __syncwarp();
#pragma unroll
            for (int pp = 0; pp < 8; ++pp) {
                const int rr = (lane >> 3) + 4 * pp, ch = lane & 7;
                if ((acc_mask >> rr) & 1u) {
                    const float4 x = *reinterpret_cast<const float4 *>(tile + tc::sw128(rr, ch));
                    const int pos = S.kpos[kTcM + quad * 32 + rr];
                    red_add_v4(acc_O + ((size_t)bh * n + pos) * kTcD + wg * 32 + ch * 4, x.x, x.y, x.z, x.w);
                }
            }
        }
        if (q.pos_i >= 0 && !stored) {
            const float L = S.u2.rowsum[0][q.row] + S.u2.rowsum[1][q.row];
            float *o = o_ws + (((size_t)r * BH + bh) * n + q.pos_i) * kTcD + wg * 32;
            const bool has = q.qvalid && L > 0.0f;
            const float inv = has ? 1.0f / L : 0.0f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float4 f;
                f.x = __uint_as_float(v[u * 4 + 0]) * inv;
                f.y = __uint_as_float(v[u * 4 + 1]) * inv;
                f.z = __uint_as_float(v[u * 4 + 2]) * inv;
                f.w = __uint_as_float(v[u * 4 + 3]) * inv;
                *reinterpret_cast<float4 *>(o + u * 4) = f;
            }
            if (wg == 0)
                lse_ws[((size_t)r * BH + bh) * n + q.pos_i] =
                    has ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
        }
    }

    return true;
}

// Grid mode (items == nullptr): CTA (x, y, z) is the item (chunk x, round y, batch*head z).
// List mode: the CTAs share the item ids items[0 .. *item_count), id = (bh * rounds + r) * chunks + c.
__global__ void __launch_bounds__(kTcThreads, 2)
lsh_chunk_attn_tc_kernel(const __nv_bfloat16 *__restrict__ QK, const __nv_bfloat16 *__restrict__ V,
                         const int32_t *__restrict__ bucket, const int32_t *__restrict__ perm,
                         const int32_t *__restrict__ inv_perm, const int32_t *__restrict__ valid_len,
                         float *__restrict__ o_ws, float *__restrict__ lse_ws, float *__restrict__ acc_O,
                         float *__restrict__ acc_L, float *__restrict__ acc_M, int H, int BH, int n,
                         int rounds, int causal, int no_self, int key_norm, float scale_log2,
                         const int32_t *__restrict__ items, const int32_t *__restrict__ item_count) {
    extern __shared__ unsigned char lsh_tc_raw[];
    const uint32_t mis = smem_u32(lsh_tc_raw) & 1023u;
    LshTcSmem &S = *reinterpret_cast<LshTcSmem *>(lsh_tc_raw + ((1024u - mis) & 1023u));
    const int count = items ? *item_count : 1;
    if (items && (int)blockIdx.x >= count) return;    // uniform over the CTA, before any setup
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        tc::mbar_init(&S.bar[0], 1);
        tc::mbar_init(&S.bar[1], 1);
        tc::mbar_init(&S.bar[2], 1);
        tc::mbar_fence_init();
    }
    if (warp == 0) tc::tmem_alloc(&S.tmem_base, kTcCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = S.tmem_base;
    uint32_t ph[3] = {0u, 0u, 0u};
    const int nch = (n + kTcM - 1) / kTcM;
    for (int t = items ? (int)blockIdx.x : 0; t < count; t += items ? (int)gridDim.x : 1) {
        int c = blockIdx.x, r = blockIdx.y, bh = blockIdx.z;
        if (items) {
            const int id = items[t];
            c = id % nch;
            r = (id / nch) % rounds;
            bh = id / (nch * rounds);
        }
        if (!lsh_tc_item(S, tmem, ph, QK, V, bucket, perm, inv_perm, valid_len, o_ws, lse_ws, acc_O, acc_L,
                         acc_M, H, BH, n, rounds, causal, no_self, key_norm, scale_log2, c, r, bh))
            break;
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTcCols);
}

}  // namespace crs
