// K3 on the tensor cores, persistent form: chunked LSH attention for bf16, d = 64,
// chunk m = 128, normalised keys, at most four rounds.
//
// [P1] PaperTrace 2.1.1 §2.1-2.2 (sorted array cut into chunks of m slots; a
// chunk attends to itself and the previous chunk; edges need the same bucket
// and are judged on original positions), "重复候选和归一化" (a pair counts once),
// §4.2 (gather -> chunked attention -> scatter).
//
// The per-item arithmetic is that of lsh_chunk_attn_tc_kernel's fp16 single
// pass (P = 2^(S - bound + 15) in fp16, O += P V, the rounds accumulated into O
// with the fixed shift of each row); what changes is the schedule:
//   * two persistent CTAs per SM take work units (one (round, batch*head) and
//     up to kRgUnit consecutive chunks) from a counter, costliest rounds first;
//   * the K/V rows of a chunk live in one of three 32 KB ring slots.  Item c
//     (queries = chunk c) reads the slots of chunks c-1 and c, so each row is
//     gathered once per unit and round instead of twice; the slot of chunk c+1
//     is filled (positions, buckets, earlier-round codes, 16-byte cp.async row
//     gathers) while item c computes, and prepared (V to fp16, key norms, row
//     bounds) while its P.V runs;
//   * S = Q K^T goes to tensor memory as two N = 128 halves, P is written back
//     over the S columns already read (tcgen05.st, fp16, two keys per column)
//     and P V takes its A operand from tensor memory, so the shared memory
//     holds only the ring;
//   * the accumulated O rows are staged in the slot of chunk c-1 (free once
//     P V has completed) so that each vector reduction covers 128 contiguous
//     bytes of a row.
// Items whose V is not exact in fp16 or whose row bounds exceed the fp16 range
// are appended to a list for lsh_chunk_attn_tc_kernel's list mode (bf16 P with
// a residual, or the two-pass form), which runs right after this kernel.
//
// Tensor memory (256 columns per CTA): S of window key j in column j.  The two
// warps that share a row's lanes split its eight 32-key chunks by parity (the
// causal mask empties the high chunks of the low rows, so halves would be
// unbalanced); the k-th chunk a warp handles (chunk 2k + wg) puts its P (16
// columns) at rg_pcol(k, wg), inside the S columns that warp has already read.
// P fills [0,128); O goes to [128,192).
//
// One item, slots P (chunk c-1), O (chunk c), F (free), all 256 threads:
//   A  positions of chunk c+1 into F's metadata; barrier (the previous item's
//      epilogue reads of P's slot and of tensor memory are done);
//   B  thread 0 issues S (mbarrier bar[0]); the rows of c+1 go to F by cp.async
//      (during C for an fp16 item); F's buckets, earlier-round slots and the
//      perm entries of c+2 by 4-byte cp.async into shared memory;
//   C  wait bar[0] with a CTA vote; softmax of the item's rows, P stored to tensor
//      memory; tcgen05.wait::st, barrier; thread 0 issues P V (bar[1]);
//   E  cp.async wait; F's metadata finished from the staged words; barrier;
//      F prepared (V to fp16, norms, bounds, bucket runs; proxy fence);
//   F  wait bar[1] with a CTA vote; O rows staged in P's slot, reductions into O;
//   G  barrier; the ring turns (P <- O <- F <- P).
// Every wait is bounded; a CTA that gives up drains its MMA and leaves the loop.
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace crs {

constexpr int kRgThreads = 256;
constexpr int kRgEarlier = 3;                   // earlier rounds kept per key: rounds <= 4
constexpr int kRgUnit = 8;                      // chunks per work unit (the first 7/8 of a segment)
constexpr int kRgSmall = 2;                     // chunks per work unit (the rest: a short tail)
constexpr int kRgFlagV = 1;                     // some V value of the slot is not exact in fp16
constexpr int kRgFlagBound = 2;                 // some row bound of the slot exceeds kTcBoundMax16

struct RgMeta {
    int pos[kTcM];                  // original position of each slot row (-1: none)
    int bkt[kTcM];                  // bucket (kBktBefore / kBktAfter for absent slots)
    int code[kRgEarlier][kTcM];     // earlier rounds: bucket * C1 + chunk + 1 (-8: none)
    float kscale[kTcM];             // scale * log2(e) / |k_j|
    float bound[kTcM];              // scale |k_j| in log2 units (the row bound as a query)
    uint32_t run[kTcM];             // within the slot: first row of the row's bucket run | last row
                                    // of the run's prefix with position < valid_len from it << 16
    int flags;
    int pad[3];
};

struct RgSmem {
    unsigned char kv[3][2][kTcM * 128];   // ring slots: [0] K rows (128B swizzle), [1] V rows
    RgMeta meta[3];
    int scan[2][4];                       // per warp of a slot's rows: last run start, first run stop
    int stage[1 + kRgEarlier][kTcM];      // next chunk's earlier-round slots and the chunk after's perm
                                          // entries, copied in by cp.async (its buckets go to its metadata)
    float rowsum[2][kTcM];
    uint64_t bar[2];                      // S complete, O complete
    uint32_t tmem_base;
    int unit;
};
// two CTAs per SM: 228 KB of shared memory, 1 KB of it reserved per CTA, 1 KB of alignment slack
static_assert(sizeof(RgSmem) + 1024 <= 228 * 1024 / 2 - 1024, "ring kernel: two CTAs per SM");

// Work units of a (round, batch*head) segment of nch chunks: about 7/8 of the
// chunks in units of kRgUnit, the rest in units of kRgSmall.
__host__ __device__ __forceinline__ int rg_big_units(int nch) { return (nch * 7 / 8) / kRgUnit; }
__host__ __device__ __forceinline__ int rg_small_units(int nch) {
    return (nch - rg_big_units(nch) * kRgUnit + kRgSmall - 1) / kRgSmall;
}

// Original position of slot s of a (round, batch*head) segment; -1 outside [0, n) or
// for a perm entry out of range (flagged).
__device__ __forceinline__ int rg_slot_pos(const int32_t *__restrict__ perm, size_t seg, int n, int s) {
    if (s < 0 || s >= n) return -1;
    const int pos = perm[seg + s];
    if (pos < 0 || pos >= n) {
        raise_error(CRS_DEVERR_INDEX);
        return -1;
    }
    return pos;
}

// Bucket and earlier-round codes of a slot row whose position is known, in two
// steps: the loads (raw values), then, once they are needed, the codes.  Nothing
// between the two consumes the loaded registers, so the warp does not wait for
// them until the second step.
struct RgRowRaw {
    int bkt, eb[kRgEarlier], es[kRgEarlier];
};
struct RgRowMeta {
    int bkt;
    int code[kRgEarlier];
};
__device__ __forceinline__ RgRowRaw rg_row_load(const int32_t *__restrict__ bucket, const int32_t *__restrict__ inv_perm,
                                                int bh, int rounds, int r, int n, int pos) {
    RgRowRaw w;
    w.bkt = 0;
#pragma unroll
    for (int rr = 0; rr < kRgEarlier; ++rr) w.eb[rr] = w.es[rr] = 0;
    if (pos >= 0) {
        w.bkt = bucket[((size_t)bh * rounds + r) * n + pos];
#pragma unroll
        for (int rr = 0; rr < kRgEarlier; ++rr) {
            if (rr < r) {
                const size_t sg = ((size_t)bh * rounds + rr) * n;
                w.eb[rr] = bucket[sg + pos];
                w.es[rr] = inv_perm[sg + pos];
            }
        }
    }
    return w;
}
__device__ __forceinline__ RgRowMeta rg_row_finish(const RgRowRaw &w, int r, int C1, int s, int pos) {
    RgRowMeta m;
    m.bkt = pos >= 0 ? w.bkt : (s < 0 ? kBktBefore : kBktAfter);
#pragma unroll
    for (int rr = 0; rr < kRgEarlier; ++rr)      // -8 matches no query code
        m.code[rr] = (rr < r && pos >= 0) ? w.eb[rr] * C1 + w.es[rr] / kTcM + 1 : -8;
    return m;
}

// Validated position from a raw perm entry (-1 and a flag when out of range).
__device__ __forceinline__ int rg_checked_pos(int raw, int n) {
    if (raw < 0 || raw >= n) {
        raise_error(CRS_DEVERR_INDEX);
        return -1;
    }
    return raw;
}

__device__ __forceinline__ void rg_store_row_meta(RgMeta &M, int row, const RgRowMeta &m) {
    M.bkt[row] = m.bkt;
#pragma unroll
    for (int rr = 0; rr < kRgEarlier; ++rr) M.code[rr][row] = m.code[rr];
}

// 16-byte gathers of the slot's K and V rows (positions from its metadata); four
// pieces of each per thread, one commit group.
__device__ __forceinline__ void rg_gather(RgSmem &S, int slot, const __nv_bfloat16 *__restrict__ Kb,
                                          const __nv_bfloat16 *__restrict__ Vb, int tid) {
#pragma unroll
    for (int u = 0; u < (kTcM * 8) / kRgThreads; ++u) {
        const int e = tid + u * kRgThreads;
        const int row = e >> 3, ch = e & 7;
        const int pos = S.meta[slot].pos[row];
        const bool ok = pos >= 0;
        const size_t off = ok ? (size_t)pos * kTcD + ch * 8 : 0;
        cp_async16_zfill(S.kv[slot][0] + tc::sw128(row, ch), Kb + off, ok);
        cp_async16_zfill(S.kv[slot][1] + tc::sw128(row, ch), Vb + off, ok);
    }
    cp_async_commit();
}

// Piece u (of four) of rg_gather, without the commit: the row gathers are spread
// over the softmax so that they never fill the load/store queues at once.
struct RgGather {
    unsigned char *kdst, *vdst;
    const int *pos;
    const __nv_bfloat16 *Kb, *Vb;
};
__device__ __forceinline__ void rg_gather_piece(const RgGather &g, int tid, int u) {
    const int e = tid + u * kRgThreads;
    const int row = e >> 3, ch = e & 7;
    const int pos = g.pos[row];
    const bool ok = pos >= 0;
    const size_t off = ok ? (size_t)pos * kTcD + ch * 8 : 0;
    cp_async16_zfill(g.kdst + tc::sw128(row, ch), g.Kb + off, ok);
    cp_async16_zfill(g.vdst + tc::sw128(row, ch), g.Vb + off, ok);
}

// Prepare a slot whose rows have landed (metadata written): V to fp16 in place
// (flagging values that do not convert exactly), key norms, row bounds and the
// bucket runs inside the slot.  Two threads per row.
__device__ __forceinline__ void rg_prep(RgSmem &S, int slot, int tid, float scale_log2, int vl) {
    const int row = tid >> 1, h = tid & 1;
    RgMeta &M = S.meta[slot];
    uint32_t vbad = 0u;
    float ss = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int ch = h * 4 + q;
        unsigned char *vp = S.kv[slot][1] + tc::sw128(row, ch);
        const uint4 w = *reinterpret_cast<const uint4 *>(vp);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        uint32_t hh[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            // |bf16| >= 2^16 (or Inf / NaN) does not convert exactly: bit 15 of each half of
            // (w & 0x7fff7fff) + 0x38803880 is set exactly when the half's magnitude bits reach 0x4780
            vbad |= ((ww[t] & 0x7fff7fffu) + 0x38803880u) & 0x80008000u;
            const __half2 hv = __floats2half2_rn(__uint_as_float(ww[t] << 16), __uint_as_float(ww[t] & 0xffff0000u));
            hh[t] = *reinterpret_cast<const uint32_t *>(&hv);
        }
        *reinterpret_cast<uint4 *>(vp) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
        const uint4 k = *reinterpret_cast<const uint4 *>(S.kv[slot][0] + tc::sw128(row, ch));
        const uint32_t kk[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float a0 = __uint_as_float(kk[t] << 16), a1 = __uint_as_float(kk[t] & 0xffff0000u);
            ss = fmaf(a1, a1, fmaf(a0, a0, ss));
        }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    const float bound = sqrtf(ss) * fabsf(scale_log2);
    if (h == 0) {
        M.kscale[row] = (ss > 0.0f ? rsqrtf(ss) : 0.0f) * scale_log2;
        M.bound[row] = bound;
    }
    // Bucket runs inside the slot (rows are sorted by bucket, then position): a run starts
    // where the bucket changes; from row j its valid part goes on while the next row has
    // the same bucket and a position below vl.  One row per thread of warps 0..3; a warp
    // with no start (stop) of its own takes the nearest one of the warps before (after) it.
    if (tid < kTcM) {
        const int j = tid, w = j >> 5, l = j & 31;
        const int bk = M.bkt[j];
        const bool start = j == 0 || M.bkt[j - 1] != bk;
        const bool stop = j == kTcM - 1 || M.bkt[j + 1] != bk || !(M.pos[j + 1] < vl);
        const uint32_t sm = __ballot_sync(0xffffffffu, start), tm = __ballot_sync(0xffffffffu, stop);
        if (l == 0) {
            S.scan[0][w] = sm ? 32 * w + 31 - __clz(sm) : -1;
            S.scan[1][w] = tm ? 32 * w + __ffs(tm) - 1 : kTcM;
        }
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        const uint32_t le = sm & (0xffffffffu >> (31 - l)), ge = tm & (0xffffffffu << l);
        int first = le ? 32 * w + 31 - __clz(le) : -1, last = ge ? 32 * w + __ffs(ge) - 1 : kTcM;
        for (int w2 = w - 1; first < 0; --w2) first = S.scan[0][w2];   // row 0 always starts a run
        for (int w2 = w + 1; last == kTcM; ++w2) last = S.scan[1][w2];  // row 127 always stops one
        M.run[j] = (uint32_t)first | ((uint32_t)last << 16);
    }
    const int fl = (vbad ? kRgFlagV : 0) | (!(bound <= kTcBoundMax16) ? kRgFlagBound : 0);
    const int wfl = __reduce_or_sync(0xffffffffu, fl);
    if ((tid & 31) == 0 && wfl) atomicOr(&M.flags, wfl);
    tc::fence_proxy_async();                      // the fp16 V rows are read by tcgen05.mma
}

// Tensor-memory column of the P of the k-th chunk (0..3) of warp half wg: chunks
// 2k + wg = 0, 2 | 1, 3 | 4, 6 | 5, 7 land in [0,32) | [32,64) | [64,96) | [96,128),
// each inside the S columns of chunk 2 (k / 2) + wg, read by the same warp before.
__host__ __device__ constexpr int rg_pcol(int k, int wg) { return 64 * (k >> 1) + 32 * wg + 16 * (k & 1); }

// Masked fp16 P of one query row for the window chunks 2k + wg, k = 0..3 (keys of
// the previous chunk's slot MP for k < 2, of the own chunk's MO after), written to
// tensor memory at rg_pcol; returns the row's partial sum.  NR = earlier rounds
// whose pairs are excluded.
template <int NR>
__device__ __forceinline__ float rg_softmax16(const RgMeta &MP, const RgMeta &MO, const LshTcRow &q,
                                              uint32_t trow, int wg, float M, const RgGather &g, bool gather,
                                              int tid) {
    const RgMeta &Mq = MO;
    int ci[NR > 0 ? NR : 1];
#pragma unroll
    for (int rr = 0; rr < NR; ++rr) ci[rr] = Mq.code[rr][q.row];
    float2 sum2[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                      make_float2(0.0f, 0.0f)};           // four independent chains
    const float2 negM = make_float2(-M, -M);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        const int c0 = (2 * cc + wg) * 32;        // window column of the chunk
        const RgMeta &Mk = cc < 2 ? MP : MO;
        const int kr = c0 & (kTcM - 1);           // its first row in that slot
        uint32_t mb = q.qvalid ? range_bits(q.lo, q.hi, c0) : 0u;
        if (q.excl_self && q.jq >= c0 && q.jq < c0 + 32) mb &= ~(1u << (q.jq - c0));
        uint32_t ph[16];
        if (__any_sync(0xffffffffu, mb != 0u)) {
            uint32_t v[32];
            tc::tmem_ld32(trow + c0, v);
            tc::tmem_ld_wait();
            const float4 *ks = reinterpret_cast<const float4 *>(&Mk.kscale[kr]);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 k4 = ks[u];
                bool ok[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) ok[e] = (mb >> (4 * u + e)) & 1u;
#pragma unroll
                for (int rr = 0; rr < NR; ++rr) {
                    const int4 kc = reinterpret_cast<const int4 *>(&Mk.code[rr][kr])[u];
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
                sum2[2 * (u & 1)] = __fadd2_rn(sum2[2 * (u & 1)], p01);
                sum2[2 * (u & 1) + 1] = __fadd2_rn(sum2[2 * (u & 1) + 1], p23);
                const __half2 h01 = __floats2half2_rn(p01.x, p01.y);
                const __half2 h23 = __floats2half2_rn(p23.x, p23.y);
                ph[2 * u] = *reinterpret_cast<const uint32_t *>(&h01);
                ph[2 * u + 1] = *reinterpret_cast<const uint32_t *>(&h23);
            }
        } else {
#pragma unroll
            for (int t2 = 0; t2 < 16; ++t2) ph[t2] = 0u;
        }
        tc::tmem_st16(trow + rg_pcol(cc, wg), ph);
        if (gather) rg_gather_piece(g, tid, cc);
    }
    const float2 t = __fadd2_rn(__fadd2_rn(sum2[0], sum2[1]), __fadd2_rn(sum2[2], sum2[3]));
    return t.x + t.y;
}

__global__ void __launch_bounds__(kRgThreads, 2)
lsh_chunk_attn_ring_kernel(const __nv_bfloat16 *__restrict__ QK, const __nv_bfloat16 *__restrict__ V,
                           const int32_t *__restrict__ bucket, const int32_t *__restrict__ perm,
                           const int32_t *__restrict__ inv_perm, const int32_t *__restrict__ valid_len,
                           float *__restrict__ acc_O, float *__restrict__ acc_L, float *__restrict__ acc_M,
                           int *__restrict__ unit_counter, int32_t *__restrict__ deferred,
                           int *__restrict__ deferred_count, int H, int BH, int n, int rounds, int causal,
                           int no_self, float scale_log2) {
    extern __shared__ unsigned char rg_raw[];
    const uint32_t mis = smem_u32(rg_raw) & 1023u;
    RgSmem &S = *reinterpret_cast<RgSmem *>(rg_raw + ((1024u - mis) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nch = (n + kTcM - 1) / kTcM;
    const int nbig = rg_big_units(nch), nsmall = rg_small_units(nch);   // per (round, batch*head)
    const int n_big = nbig * BH * rounds, n_units = n_big + nsmall * BH * rounds;
    const int C1 = nch + 1;                            // chunk-code stride

    if (tid == 0) {
        tc::mbar_init(&S.bar[0], 1);
        tc::mbar_init(&S.bar[1], 1);
        tc::mbar_fence_init();
    }
    if (warp == 0) tc::tmem_alloc(&S.tmem_base, kTcCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = S.tmem_base;
    uint32_t ph0 = 0u, ph1 = 0u;
    bool failed = false;

    const int wg = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;                  // query row of this thread (own chunk)
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);

    for (;;) {
        if (tid == 0) S.unit = atomicAdd(unit_counter, 1);
        __syncthreads();
        const int u = S.unit;
        if (u >= n_units) break;
        // long units first, then the short ones; within each, costliest rounds (most
        // earlier-round tests) first
        const bool big = u < n_big;
        const int uu = big ? u : u - n_big, per = big ? nbig : nsmall;
        const int r = rounds - 1 - uu / (BH * per);
        const int rem = uu % (BH * per);
        const int bh = rem / per, part = rem % per;
        const int c_begin = big ? part * kRgUnit : nbig * kRgUnit + part * kRgSmall;
        const int c_end = min(nch, c_begin + (big ? kRgUnit : kRgSmall));
        const int vl = valid_len ? valid_len[bh / H] : n;
        const size_t seg_r = ((size_t)bh * rounds + r) * n;
        const __nv_bfloat16 *Kb = QK + (size_t)bh * n * kTcD;
        const __nv_bfloat16 *Vb = V + (size_t)bh * n * kTcD;

        // ---- prologue: slot 0 = chunk c_begin - 1, slot 1 = chunk c_begin
        int sP = 0, sO = 1, sF = 2;
        {
            const int slot = tid >> 7, j = tid & (kTcM - 1);
            const int s = (c_begin - 1 + slot) * kTcM + j;
            const int pos = rg_slot_pos(perm, seg_r, n, s);
            S.meta[slot].pos[j] = pos;
            rg_store_row_meta(S.meta[slot], j,
                              rg_row_finish(rg_row_load(bucket, inv_perm, bh, rounds, r, n, pos), r, C1, s, pos));
            if (j == 0) S.meta[slot].flags = 0;
        }
        __syncthreads();
        rg_gather(S, 0, Kb, Vb, tid);
        rg_gather(S, 1, Kb, Vb, tid);
        int pos_next = -1;                             // position of row tid of the chunk after the next one
        if (tid < kTcM && c_begin + 1 < c_end) pos_next = rg_slot_pos(perm, seg_r, n, (c_begin + 1) * kTcM + tid);
        cp_async_wait<0>();
        __syncthreads();
        rg_prep(S, 0, tid, scale_log2, vl);
        __syncthreads();                               // the run scratch is reused
        rg_prep(S, 1, tid, scale_log2, vl);

        for (int c = c_begin; c < c_end; ++c) {
            const bool has_next = c + 1 < c_end, has_next2 = c + 2 < c_end;
            // ---- A. positions of chunk c+1 into the free slot
            if (has_next && tid < kTcM) S.meta[sF].pos[tid] = pos_next;
            if (has_next && tid == 0) S.meta[sF].flags = 0;
            tc::fence_before();
            __syncthreads();
            tc::fence_after();
            const RgMeta &MP = S.meta[sP], &MO = S.meta[sO];
            const bool use16 = ((MP.flags & kRgFlagV) | (MO.flags & (kRgFlagV | kRgFlagBound))) == 0;
            // ---- B. S = Q K^T for item c; the gathers of chunk c+1 and its metadata
            if (use16 && tid == 0) {
                constexpr uint32_t idesc = tc::idesc_bf16_f32(kTcM, kTcM, 0, 0);
                const uint32_t qs = smem_u32(S.kv[sO][0]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t ks = smem_u32(S.kv[h == 0 ? sP : sO][0]);
#pragma unroll
                    for (int k = 0; k < kTcD / 16; ++k)
                        tc::mma_bf16(tmem + (uint32_t)(h * kTcM),
                                     tc::smem_desc(qs + k * 32, 16, 1024, tc::kLayoutSW128),
                                     tc::smem_desc(ks + k * 32, 16, 1024, tc::kLayoutSW128), idesc, k > 0 ? 1u : 0u);
                }
                tc::commit(&S.bar[0]);
            }
            if (!use16 && tid == 0) deferred[atomicAdd(deferred_count, 1)] = (bh * rounds + r) * nch + c;
            // the next chunk's rows: during the softmax, or here for an item left to the per-item kernel
            if (has_next && !use16) rg_gather(S, sF, Kb, Vb, tid);
            // the next chunk's buckets and codes and the chunk after's perm entries go to shared
            // memory by cp.async: no register waits on them before they are used, after the softmax
            const int s2 = (c + 2) * kTcM + tid;
            const bool want2 = has_next2 && tid < kTcM && s2 < n;
            if (tid < kTcM) {
                if (has_next && pos_next >= 0) {
                    RgMeta &MF = S.meta[sF];
                    cp_async4(&MF.bkt[tid], bucket + seg_r + pos_next);
#pragma unroll
                    for (int rr = 0; rr < kRgEarlier; ++rr) {
                        if (rr < r) {
                            const size_t sg = ((size_t)bh * rounds + rr) * n;
                            cp_async4(&MF.code[rr][tid], bucket + sg + pos_next);   // raw bucket for now
                            cp_async4(&S.stage[rr][tid], inv_perm + sg + pos_next);
                        }
                    }
                }
                if (want2) cp_async4(&S.stage[kRgEarlier][tid], perm + seg_r + s2);
            }
            cp_async_commit();
            LshTcRow q;
            float sum = 0.0f, bnd = 0.0f;
            if (use16) {
                // ---- C. masked fp16 P into tensor memory
                const bool ok = tc::mbar_wait_bounded(&S.bar[0], ph0, kTcWaitNs, K_LSH_ATTN_TC, 1, 10000u, true);
                if (__syncthreads_or(!ok)) {
                    tc::mbar_wait_bounded(&S.bar[0], ph0, kTcWaitNs, K_LSH_ATTN_TC, 2);   // let the MMA drain
                    failed = true;
                    break;
                }
                ph0 ^= 1u;
                tc::fence_after();
                q.row = row;
                q.jq = kTcM + row;
                q.pos_i = MO.pos[row];
                q.qvalid = q.pos_i >= 0 && q.pos_i < vl;
                // the query's bucket run in the window (key j < 128: row j of the previous
                // chunk's slot, j >= 128: row j - 128 of its own): it starts in the own chunk,
                // or, when the own chunk's first run continues the previous chunk's last,
                // where that one starts; its valid part ends in the own chunk
                const uint32_t run = MO.run[row];
                const int f = (int)(run & 0xffffu);
                q.lo = f > 0 || MP.bkt[kTcM - 1] != MO.bkt[row] ? kTcM + f : (int)(MP.run[kTcM - 1] & 0xffffu);
                q.hi = causal ? (no_self ? q.jq - 1 : q.jq) : kTcM + (int)(run >> 16);
                q.excl_self = (!causal) && no_self;
                bnd = MO.bound[row];
                const float Mx = bnd - 15.0f;
                const RgGather g{S.kv[sF][0], S.kv[sF][1], S.meta[sF].pos, Kb, Vb};
                switch (r) {
                    case 0: sum = rg_softmax16<0>(MP, MO, q, trow, wg, Mx, g, has_next, tid); break;
                    case 1: sum = rg_softmax16<1>(MP, MO, q, trow, wg, Mx, g, has_next, tid); break;
                    case 2: sum = rg_softmax16<2>(MP, MO, q, trow, wg, Mx, g, has_next, tid); break;
                    default: sum = rg_softmax16<3>(MP, MO, q, trow, wg, Mx, g, has_next, tid); break;
                }
                if (has_next) cp_async_commit();
                tc::tmem_st_wait();
                S.rowsum[wg][row] = sum;
                tc::fence_before();
                __syncthreads();
                tc::fence_after();
                // ---- D. O = P V (A = P in tensor memory, B = fp16 V rows of the two slots)
                if (tid == 0) {
                    constexpr uint32_t idesc = tc::idesc_f16_f32(kTcM, kTcD, 0, 1);
#pragma unroll
                    for (int kk = 0; kk < 16; ++kk) {
                        const int j = kk >> 1, hh = kk & 1;   // keys [32 j + 16 hh, +16)
                        const uint32_t vs = smem_u32(S.kv[j < 4 ? sP : sO][1]) + ((j & 3) * 32 + hh * 16) * 128;
                        tc::mma_f16_ts(tmem + 128, tmem + (uint32_t)(rg_pcol(j >> 1, j & 1) + hh * 8),
                                       tc::smem_desc(vs, 32768, 1024, tc::kLayoutSW128), idesc, kk > 0 ? 1u : 0u);
                    }
                    tc::commit(&S.bar[1]);
                }
            }
            // ---- E. the next slot: metadata, rows, preparation (overlaps P V)
            cp_async_wait<0>();
            if (tid < kTcM) {
                if (has_next) {
                    RgMeta &MF = S.meta[sF];
                    RgRowRaw w;
                    w.bkt = MF.bkt[tid];
#pragma unroll
                    for (int rr = 0; rr < kRgEarlier; ++rr) {
                        w.eb[rr] = MF.code[rr][tid];
                        w.es[rr] = S.stage[rr][tid];
                    }
                    rg_store_row_meta(MF, tid, rg_row_finish(w, r, C1, (c + 1) * kTcM + tid, pos_next));
                }
                pos_next = want2 ? rg_checked_pos(S.stage[kRgEarlier][tid], n) : -1;
            }
            __syncthreads();
            if (has_next) rg_prep(S, sF, tid, scale_log2, vl);
            if (use16) {
                // ---- F. epilogue: accumulate the round into O with the row's fixed shift
                const bool ok = tc::mbar_wait_bounded(&S.bar[1], ph1, kTcWaitNs, K_LSH_ATTN_TC, 4);
                if (__syncthreads_or(!ok)) {
                    tc::mbar_wait_bounded(&S.bar[1], ph1, kTcWaitNs, K_LSH_ATTN_TC, 5);   // let the MMA drain
                    failed = true;
                    break;
                }
                ph1 ^= 1u;
                tc::fence_after();
                uint32_t v[32];
                tc::tmem_ld32(trow + 128 + wg * 32, v);
                tc::tmem_ld_wait();
                const float L = S.rowsum[0][row] + S.rowsum[1][row];
                const bool acc_row = q.qvalid && L > 0.0f;
                const float f = 0x1p-15f;
                if (q.pos_i >= 0 && wg == 0) {
                    const size_t orow = (size_t)bh * n + q.pos_i;
                    if (acc_row) atomicAdd(acc_L + orow, L * f);
                    acc_M[orow] = bnd;
                }
                const uint32_t acc_mask = __ballot_sync(0xffffffffu, acc_row);
                if (acc_mask) {
                    unsigned char *tile = S.kv[sP][0] + warp * 4096;   // slot of chunk c-1: free now
#pragma unroll
                    for (int uu = 0; uu < 8; ++uu)
                        *reinterpret_cast<float4 *>(tile + tc::sw128(lane, uu)) =
                            make_float4(__uint_as_float(v[uu * 4 + 0]) * f, __uint_as_float(v[uu * 4 + 1]) * f,
                                        __uint_as_float(v[uu * 4 + 2]) * f, __uint_as_float(v[uu * 4 + 3]) * f);
                    __syncwarp();
#pragma unroll
                    for (int pp = 0; pp < 8; ++pp) {
                        const int rr = (lane >> 3) + 4 * pp, ch = lane & 7;
                        if ((acc_mask >> rr) & 1u) {
                            const float4 x = *reinterpret_cast<const float4 *>(tile + tc::sw128(rr, ch));
                            const int pos = MO.pos[quad * 32 + rr];
                            red_add_v4(acc_O + ((size_t)bh * n + pos) * kTcD + wg * 32 + ch * 4, x.x, x.y, x.z, x.w);
                        }
                    }
                }
            }
            // ---- G. rotate the ring: c's slot becomes the previous one, c-1's is free
            tc::fence_before();
            __syncthreads();
            tc::fence_after();
            const int t = sP;
            sP = sO;
            sO = sF;
            sF = t;
        }
        if (failed) break;
    }
    cp_async_wait<0>();
    tc::fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTcCols);
}

}  // namespace crs
