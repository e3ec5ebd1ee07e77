// Attention over explicit index lists (the gather stage shared by all selectors), sm_100a.
//
// [P1] PaperTrace 2.1.1 §1.1 Eq.(1) restricted to the candidate set; [P2]
// PaperTrace 2.2 §1.1 (one selected set shared by the main heads) and §2.1
// ("主 KV gather 的物理代价": ascending positions, one load per key serves
// every head that shares it); [P4] ch.26 §26.2 (GQA grouping).
//
// One CTA = one (row, KV head, split of the list).  The G <= 16 query heads
// of the KV head form the M = 16 side of mma.sync.m16n8k16 (bf16 in, fp32
// accumulate).  Keys are gathered 64 per stage with 16-byte cp.async into
// XOR-swizzled shared rows (a ring of 2 tiles, one in flight while the other is
// consumed; one barrier per tile); each of the 4 warps owns 16
// keys of a stage and keeps its own online-softmax state; the warps merge at
// the end.  The path is bound by gather latency: with two tiles (64 KB) and the
// query tile placed over the second ring slot until that slot's first gather,
// three CTAs share an SM at a 2048-key list (a three-tile ring held two:
// 6.6 -> 4.8 ms at prefill).
#include <math.h>

#include "common.cuh"

namespace crs {

constexpr int kSaD = 128;          // head dim
constexpr int kSaKeys = 64;        // keys per stage
constexpr int kSaWarps = 4;
constexpr int kSaThreads = kSaWarps * 32;
constexpr int kSaRowBytes = kSaD * 2;                 // 256 B per K or V row
constexpr int kSaTileBytes = kSaKeys * kSaRowBytes;   // 16 KB
constexpr int kSaStages = 2;                          // K/V tiles in the ring
constexpr float kLog2e = 1.4426950408889634f;

// 2^x by the hardware approximation (relative error about 2^-22, far inside the
// output tolerance); 2^-inf = 0
__device__ __forceinline__ float sa_ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// swizzled byte offset of 16-byte chunk c (0..15) of row r inside a tile
__device__ __forceinline__ int sw_off(int r, int c) { return r * kSaRowBytes + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
// (x, y) -> bf16 pair of the rounded values and bf16 pair of the residuals
__device__ __forceinline__ void pack_bf16_split(float x, float y, uint32_t &hi, uint32_t &lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    const float2 hf = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<uint32_t *>(&h);
    lo = *reinterpret_cast<uint32_t *>(&l);
}

struct SaArgs {
    const __nv_bfloat16 *Q, *K, *V;
    const int64_t *kv_base;
    const int32_t *I;
    const uint8_t *key_valid;   // [n_keys] or null: padding mask
    const int32_t *q_pos;       // [n_rows] or null: causal limit per row
    float *O;
    float *lse;
    float *part_o;      // [rows*n_q][splits][D] (splits > 1)
    float *part_ml;     // [rows*n_q][splits][2]  (m in log2 units, l)
    int n_rows, n_q, n_kv, G, max_idx, n_lists, n_keys, splits, split_len;
    float scale_log2;   // scale * log2(e)
};

// kOff32: the list holds each token's offset from K (and V) in 16-byte units, which fits
// an int when the cache is below 32 GB (the host checks), so a gather piece needs one
// 32-bit multiply instead of the 64-bit position arithmetic; -1 marks a skipped entry
// either way.
template <bool kOff32>
__global__ void __launch_bounds__(kSaThreads) sparse_attn_kernel(SaArgs a) {
    extern __shared__ __align__(128) unsigned char sa_smem[];
    unsigned char *sK = sa_smem;                                  // [kSaStages][kSaTileBytes]
    unsigned char *sV = sK + kSaStages * kSaTileBytes;            // [kSaStages][kSaTileBytes]
    // [16 rows][256 B] swizzled, over ring slot 1: its first gather is issued after every
    // warp has read the query fragments (they are read before the loop's first barrier)
    unsigned char *sQ = sK + 1 * kSaTileBytes;
    float *sRed = reinterpret_cast<float *>(sV + kSaStages * kSaTileBytes);   // [4][16] m, [4][16] l
    int *sIdx = reinterpret_cast<int *>(sRed + kSaWarps * 16 * 2);      // the split's list, -1 padded

    const int split = blockIdx.x;
    const int item = blockIdx.y;                 // row * n_kv + h
    const int row = item / a.n_kv, h = item - row * a.n_kv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G;
    const int64_t kbase = a.kv_base ? a.kv_base[row] : 0;
    const int32_t *idx = a.I + ((size_t)row * a.n_lists + (a.n_lists == 1 ? 0 : h)) * a.max_idx;
    const int s0 = split * a.split_len;
    const int s1 = min(a.max_idx, s0 + a.split_len);
    const int n_tiles = (s1 > s0) ? ceil_div(s1 - s0, kSaKeys) : 0;
    const size_t tok_stride = (size_t)a.n_kv * kSaD;       // elements between tokens
    const __nv_bfloat16 *Kh = a.K + (size_t)h * kSaD;
    const __nv_bfloat16 *Vh = a.V + (size_t)h * kSaD;

    // ---- Q tile: rows g < G hold head h*G+g, the rest are zero
    for (int e = tid; e < 16 * 16; e += kSaThreads) {
        const int r = e >> 4, c = e & 15;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < G)
            v = *reinterpret_cast<const uint4 *>(a.Q + ((size_t)row * a.n_q + h * G + r) * kSaD + c * 8);
        *reinterpret_cast<uint4 *>(sQ + sw_off(r, c)) = v;
    }

    // the split's index list, once, into shared memory (padded with -1 to whole
    // tiles).  An entry outside K/V is flagged and skipped; masked entries (after
    // the row's causal limit, or on a padding key) are skipped ([P1] §1.1 Eq.(2)).
    const int qlim = a.q_pos ? a.q_pos[row] : 0x7fffffff;
    for (int i = tid; i < n_tiles * kSaKeys; i += kSaThreads) {
        int j = (s0 + i < s1) ? __ldg(idx + s0 + i) : -1;
        if (j < -1 || (j >= 0 && kbase + j >= (int64_t)a.n_keys)) {
            raise_error(CRS_DEVERR_INDEX);
            j = -1;
        }
        if (j > qlim) j = -1;
        if (j >= 0 && a.key_valid && a.key_valid[kbase + j] == 0) j = -1;
        if constexpr (kOff32) sIdx[i] = j >= 0 ? (int)((kbase + j) * (int64_t)(tok_stride / 8)) : -1;
        else sIdx[i] = j;
    }
    __syncthreads();

    // Issue the gathers of tile t into ring slot t % kSaStages (one commit group per
    // call, empty past the last tile).
    auto load_tile = [&](int t) {
        if (t < n_tiles) {
            const int buf = t % kSaStages;
            const int *si = sIdx + t * kSaKeys;
            unsigned char *k_dst = sK + buf * kSaTileBytes;
            unsigned char *v_dst = sV + buf * kSaTileBytes;
#pragma unroll
            for (int u = 0; u < (kSaKeys * 16) / kSaThreads; ++u) {
                const int e = tid + u * kSaThreads;
                const int r = e >> 4, c = e & 15;
                const int j = si[r];
                const bool ok = j >= 0;
                size_t off;                            // elements from Kh / Vh
                if constexpr (kOff32) off = ok ? ((size_t)(unsigned)j + (unsigned)c) * 8u : 0;
                else off = ok ? ((size_t)(kbase + j) * tok_stride + c * 8) : 0;
                cp_async16_zfill(k_dst + sw_off(r, c), Kh + off, ok);
                cp_async16_zfill(v_dst + sw_off(r, c), Vh + off, ok);
            }
        }
        cp_async_commit();
    };

#pragma unroll
    for (int t = 0; t < kSaStages - 1; ++t) load_tile(t);
    __syncthreads();

    // ---- Q fragments (A operand, 16 x 128): 8 k-steps x 4 regs
    uint32_t qf[8][4];
    {
        const uint32_t qbase = smem_u32(sQ);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            // matrices: (rows 0-7, k lo), (rows 8-15, k lo), (rows 0-7, k hi), (rows 8-15, k hi)
            const int mi = lane >> 3, r = (lane & 7) + ((mi & 1) << 3), c = kk * 2 + (mi >> 1);
            ldsm_x4(qbase + sw_off(r, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
    }

    float o[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;
    const int g_row = lane >> 2, tig = lane & 3;

    for (int t = 0; t < n_tiles; ++t) {
        const int buf = t % kSaStages;
        cp_async_wait<kSaStages - 2>();          // tile t has landed (this thread's copies)
        __syncthreads();                         // ... everyone's; tile t-1 is no longer read
        load_tile(t + kSaStages - 1);            // into the slot tile t-1 used
        const int *si = sIdx + t * kSaKeys;
        const int kw = warp * 16;        // this warp's 16 keys
        const bool any = (si[kw + (lane & 15)] >= 0);
        if (__any_sync(0xffffffffu, any)) {
            const uint32_t kb = smem_u32(sK + buf * kSaTileBytes);
            const uint32_t vb = smem_u32(sV + buf * kSaTileBytes);
            float s[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                // (keys 0-7, dims lo), (keys 0-7, dims hi), (keys 8-15, lo), (keys 8-15, hi)
                const int mi = lane >> 3;
                const int r = kw + (lane & 7) + ((mi >> 1) << 3);
                const int c = kk * 2 + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + sw_off(r, c), b0, b1, b2, b3);
                mma_bf16(s[0], qf[kk], b0, b1);
                mma_bf16(s[1], qf[kk], b2, b3);
            }
            // mask + scale (log2 domain)
            float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int key = kw + nt * 8 + tig * 2 + e;
                    const bool ok = si[key] >= 0;
                    s[nt][e] = ok ? s[nt][e] * a.scale_log2 : -INFINITY;
                    s[nt][2 + e] = ok ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
                    mx_lo = fmaxf(mx_lo, s[nt][e]);
                    mx_hi = fmaxf(mx_hi, s[nt][2 + e]);
                }
            }
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
            const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
            const float c_lo = (mn_lo == -INFINITY) ? 1.0f : sa_ex2(m_lo - mn_lo);
            const float c_hi = (mn_hi == -INFINITY) ? 1.0f : sa_ex2(m_hi - mn_hi);
            float ps_lo = 0.0f, ps_hi = 0.0f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    s[nt][e] = (s[nt][e] == -INFINITY) ? 0.0f : sa_ex2(s[nt][e] - mn_lo);
                    s[nt][2 + e] = (s[nt][2 + e] == -INFINITY) ? 0.0f : sa_ex2(s[nt][2 + e] - mn_hi);
                    ps_lo += s[nt][e];
                    ps_hi += s[nt][2 + e];
                }
            }
            l_lo = l_lo * c_lo + ps_lo;
            l_hi = l_hi * c_hi + ps_hi;
            m_lo = mn_lo;
            m_hi = mn_hi;
            // the running maxima rarely move after the first tiles: rescale only when one did
            if (c_lo != 1.0f || c_hi != 1.0f) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    o[j][0] *= c_lo; o[j][1] *= c_lo;
                    o[j][2] *= c_hi; o[j][3] *= c_hi;
                }
            }
            // P = P_hi + P_lo, both bf16: the pair carries ~16 significant bits, so
            // rounding P for the tensor core stays far below the output tolerance
            uint32_t pa[4], pl[4];
            pack_bf16_split(s[0][0], s[0][1], pa[0], pl[0]);
            pack_bf16_split(s[0][2], s[0][3], pa[1], pl[1]);
            pack_bf16_split(s[1][0], s[1][1], pa[2], pl[2]);
            pack_bf16_split(s[1][2], s[1][3], pa[3], pl[3]);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                // (keys 0-7, dims 16jj..), (keys 8-15, dims 16jj..), (keys 0-7, 16jj+8..), (keys 8-15, 16jj+8..)
                const int mi = lane >> 3;
                const int r = kw + (lane & 7) + ((mi & 1) << 3);
                const int c = jj * 2 + (mi >> 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vb + sw_off(r, c), b0, b1, b2, b3);
                mma_bf16(o[2 * jj], pa, b0, b1);
                mma_bf16(o[2 * jj], pl, b0, b1);
                mma_bf16(o[2 * jj + 1], pa, b2, b3);
                mma_bf16(o[2 * jj + 1], pl, b2, b3);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();                             // the ring is free: it holds the merge scratch

    // ---- merge the 4 warps: row sums across the quad, then across warps in smem
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    float *sM = sRed;                        // [4 warps][16]
    float *sL = sM + kSaWarps * 16;          // [4][16]
    float *sO = reinterpret_cast<float *>(sK);   // [4][16][128], over the K/V ring
    if (tig == 0) {
        sM[warp * 16 + g_row] = m_lo;
        sM[warp * 16 + g_row + 8] = m_hi;
        sL[warp * 16 + g_row] = l_lo;
        sL[warp * 16 + g_row + 8] = l_hi;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int col = j * 8 + tig * 2;
        sO[(warp * 16 + g_row) * kSaD + col] = o[j][0];
        sO[(warp * 16 + g_row) * kSaD + col + 1] = o[j][1];
        sO[(warp * 16 + g_row + 8) * kSaD + col] = o[j][2];
        sO[(warp * 16 + g_row + 8) * kSaD + col + 1] = o[j][3];
    }
    __syncthreads();
    for (int e = tid; e < G * kSaD; e += kSaThreads) {
        const int r = e / kSaD, col = e - r * kSaD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kSaWarps; ++w) M = fmaxf(M, sM[w * 16 + r]);
        float L = 0.0f, acc = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kSaWarps; ++w) {
                const float f = (sM[w * 16 + r] == -INFINITY) ? 0.0f : exp2f(sM[w * 16 + r] - M);
                L += f * sL[w * 16 + r];
                acc += f * sO[(w * 16 + r) * kSaD + col];
            }
        }
        const size_t qrow = (size_t)row * a.n_q + h * G + r;
        if (a.splits == 1) {
            const float val = (L > 0.0f) ? acc / L : 0.0f;
            a.O[qrow * kSaD + col] = val;
            if (a.lse && col == 0)
                a.lse[qrow] = (L > 0.0f) ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
        } else {
            a.part_o[(qrow * a.splits + split) * kSaD + col] = (L > 0.0f) ? acc / L : 0.0f;
            if (col == 0) {
                a.part_ml[(qrow * a.splits + split) * 2 + 0] = M;
                a.part_ml[(qrow * a.splits + split) * 2 + 1] = L;
            }
        }
    }
}

// merge split partials: one warp per (row, q head)
__global__ void sparse_attn_merge_kernel(const float *__restrict__ part_o,
                                         const float *__restrict__ part_ml,
                                         float *__restrict__ O, float *__restrict__ lse,
                                         int n_qrows, int splits) {
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= n_qrows) return;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part_ml[((size_t)gw * splits + s) * 2]);
    float L = 0.0f;
    float acc[kSaD / 32] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (M != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float m = part_ml[((size_t)gw * splits + s) * 2];
            const float l = part_ml[((size_t)gw * splits + s) * 2 + 1];
            if (m == -INFINITY || l == 0.0f) continue;
            const float f = exp2f(m - M) * l;
            L += f;
#pragma unroll
            for (int u = 0; u < kSaD / 32; ++u)
                acc[u] += f * part_o[((size_t)gw * splits + s) * kSaD + lane + 32 * u];
        }
    }
#pragma unroll
    for (int u = 0; u < kSaD / 32; ++u)
        O[(size_t)gw * kSaD + lane + 32 * u] = L > 0.0f ? acc[u] / L : 0.0f;
    if (lse && lane == 0) lse[gw] = (L > 0.0f) ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

constexpr int kSaMaxSplit = 4096;     // keys per split: the split's list sits in shared memory

static size_t sa_smem_bytes(int split_len) {
    static_assert((size_t)kSaWarps * 16 * kSaD * 4 <= 2 * kSaStages * (size_t)kSaTileBytes,
                  "merge scratch must fit in the K/V ring");
    static_assert(kSaStages >= 2, "the query tile sits over ring slot 1");
    return 2 * kSaStages * (size_t)kSaTileBytes + (size_t)kSaWarps * 16 * 2 * 4 +
           (size_t)split_len * 4;
}

// Splits per (row, KV head), chosen on a makespan model of the grid.  A wave
// runs n CTAs of k tiles on the SMs; an SM's gather rate is set by the CTAs it
// holds, c = n / SMs: one CTA per SM gives rate 1 (c <= 1: the busy SMs' share),
// each further resident CTA adds 0.35 (a lone CTA's gather is latency-bound).
// A wave costs n k / (SMs rate(c)); splitting adds a merge pass, costed as
// 4 + s/2 tiles (its partial rows grow with s).  At least 256 keys and at most kSaMaxSplit keys per split.
static int sa_splits(const crs_attn_params *p) {
    const long long items = (long long)p->n_rows * p->n_kv;
    const int s_min = ceil_div(p->max_idx, kSaMaxSplit);
    const int s_max = max(s_min, min(16, ceil_div(p->max_idx, 256)));
    int dev = 0, sms = 148, smem_sm = 233472, smem_rsv = 1024;
    cudaFuncAttributes fa;
    fa.numRegs = 255;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, sparse_attn_kernel<true>) != cudaSuccess) {
        cudaGetLastError();          // model with the defaults; the launch reports real errors
        sms = 148;
    }
    const int by_regs = 65536 / (kSaThreads * max(fa.numRegs, 1));
    int best = s_min;
    double best_cost = -1.0;
    for (int s = s_min; s <= s_max; ++s) {
        const int len = min(kSaMaxSplit, ceil_div(ceil_div(p->max_idx, s), kSaKeys) * kSaKeys);
        const int per_sm = max(1, min(by_regs, smem_sm / (int)(sa_smem_bytes(len) + smem_rsv)));
        const long long slots = (long long)per_sm * sms;
        const long long ctas = items * ceil_div(p->max_idx, len);
        const int k = len / kSaKeys;
        double cost = s > 1 ? 4.0 + 0.5 * s : 0.0;
        for (long long left = ctas; left > 0; left -= slots) {
            const double n = (double)min(left, slots), c = n / sms;
            const double rate = c <= 1.0 ? c : 1.0 + 0.35 * (min(c, (double)per_sm) - 1.0);
            cost += n * k / (sms * rate);
        }
        if (best_cost < 0.0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

static int sa_validate(const crs_attn_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->n_rows < 1 || p->n_q < 1 || p->n_kv < 1 || p->max_idx < 1) return CRS_ERR_INVALID_ARG;
    if (p->n_q % p->n_kv != 0 || p->n_q / p->n_kv > 16) return CRS_ERR_UNSUPPORTED;
    if (p->D != kSaD) return CRS_ERR_UNSUPPORTED;
    if (p->n_lists != 1 && p->n_lists != p->n_kv) return CRS_ERR_INVALID_ARG;
    if (p->n_keys < 1) return CRS_ERR_INVALID_ARG;
    if ((long long)p->n_rows * p->n_kv > 0x7fffffffLL) return CRS_ERR_UNSUPPORTED;
    return CRS_OK;
}

}  // namespace crs

using namespace crs;

extern "C" size_t crs_sparse_attn_workspace_size(const crs_attn_params *p) {
    if (sa_validate(p)) return 0;
    const int s = sa_splits(p);
    if (s == 1) return 0;
    const size_t qrows = (size_t)p->n_rows * p->n_q;
    return ((qrows * s * kSaD * 4 + 255) & ~size_t(255)) + qrows * s * 2 * 4;
}

extern "C" int crs_sparse_attn(const crs_attn_params *p, const void *Q, const void *K,
                               const void *V, const int64_t *kv_base, const int32_t *I,
                               const uint8_t *key_valid, const int32_t *q_pos, void *O,
                               float *lse, void *ws, size_t ws_bytes, void *stream) {
    int st = sa_validate(p);
    if (st) return st;
    if (!Q || !K || !V || !I || !O) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) |
         reinterpret_cast<uintptr_t>(ws)) & 15)
        return CRS_ERR_INVALID_ARG;                       // 16-byte row pieces
    const size_t need = crs_sparse_attn_workspace_size(p);
    if (need > 0 && (!ws || ws_bytes < need)) return CRS_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SaArgs a;
    a.Q = static_cast<const __nv_bfloat16 *>(Q);
    a.K = static_cast<const __nv_bfloat16 *>(K);
    a.V = static_cast<const __nv_bfloat16 *>(V);
    a.kv_base = kv_base;
    a.I = I;
    a.key_valid = key_valid;
    a.q_pos = q_pos;
    a.O = static_cast<float *>(O);
    a.lse = lse;
    a.n_rows = p->n_rows;
    a.n_q = p->n_q;
    a.n_kv = p->n_kv;
    a.G = p->n_q / p->n_kv;
    a.max_idx = p->max_idx;
    a.n_lists = p->n_lists;
    a.n_keys = p->n_keys;
    a.splits = sa_splits(p);
    a.split_len = min(kSaMaxSplit, ceil_div(ceil_div(p->max_idx, a.splits), kSaKeys) * kSaKeys);
    a.splits = ceil_div(p->max_idx, a.split_len);
    a.scale_log2 = p->scale * kLog2e;
    const size_t qrows = (size_t)p->n_rows * p->n_q;
    a.part_o = a.splits > 1 ? static_cast<float *>(ws) : nullptr;
    a.part_ml = a.splits > 1 ? reinterpret_cast<float *>(static_cast<char *>(ws) +
                                                         ((qrows * a.splits * kSaD * 4 + 255) &
                                                          ~size_t(255)))
                             : nullptr;
    const size_t smem = sa_smem_bytes(a.split_len);
    // 16-byte offsets of every token fit an int below 32 GB of K (or V)
    const bool off32 = (long long)p->n_keys * p->n_kv * (kSaD / 8) <= 0x7fffffffLL;
    auto kern = off32 ? sparse_attn_kernel<true> : sparse_attn_kernel<false>;
    CRS_TRY_CUDA(cudaFuncSetAttribute(kern,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    dim3 grid(a.splits, p->n_rows * p->n_kv);
    {
        ProfScope _ps(K_SA_MAIN, s);
        kern<<<grid, kSaThreads, smem, s>>>(a);
    }
    CRS_CHECK_LAUNCH();
    if (a.splits > 1) {
        const long long warps = (long long)qrows;
        {
            ProfScope _ps(K_SA_MERGE, s);
            sparse_attn_merge_kernel<<<(unsigned)ceil_div_ll(warps * 32, 256), 256, 0, s>>>(
                a.part_o, a.part_ml, a.O, lse, (int)qrows, a.splits);
        }
        CRS_CHECK_LAUNCH();
    }
    return CRS_OK;
}
