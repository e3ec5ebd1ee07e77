// Hierarchical lightning indexer (HISA) for decode rows, sm_100a.
//
// [P2] PaperTrace 2.2 "细粒度索引": the three cost-cutting directions (HISA
// scores block representatives, prunes blocks, and runs the original token
// indexer inside the kept blocks only, with the same top-k output), §2.2
// Eq.(7) (recall of the two levels multiplies), the HISA cost
// O(B d_c + k_b b d_r), and its update discussion in §2.2 (a block without a
// representative yet, the incomplete trailing one, is searched at token level).
//
// Steps per decode row (one query):
//   hisa_describe_kernel     rep_j = mean of block j's index keys (once per
//                            complete block, fp32)
//   hisa_coarse_kernel       c_j = sum_h w_h ReLU(q_h . rep_j), fp32
//   hisa_pick_blocks_kernel  the top_blocks blocks by (c desc, block asc),
//                            listed ascending
//   hisa_fine_kernel         r_s = sum_h w_h ReLU(q_h . k_s) for every key of
//                            the kept blocks and of the open block, in
//                            candidate order (= ascending position); a CTA
//                            takes 256 / b blocks
//   hisa_pick_tokens_kernel  the topk candidates by (r desc, position asc),
//                            ascending, -1 padded
// The two selections are exact; one 1024-thread CTA per row builds the k-th
// key bit by bit (CTA-wide counts) and lists the kept entries by CTA-wide
// prefix sums, as the block pick does.
#include "common.cuh"

namespace crs {

constexpr int kHd = 64;                 // index head dim
constexpr int kHMaxHeads = 8;
constexpr int kHDescWarps = 8;
constexpr int kHCoarseWarps = 8;
constexpr int kHMaxCand = 16384;        // kept-block keys + open block per row

struct HisaArgs {
    const __nv_bfloat16 *q;     // [rows, H, 64]
    const float *w;             // [rows, H]
    const __nv_bfloat16 *k;     // [keys, 64]
    const int64_t *k_off;       // [rows + 1]
    const int64_t *b_off;       // [rows + 1]
    float *rep;                 // [blocks, 64]
    float *coarse;              // [rows, max_keys / blk] (fixed row stride: bounded by max_keys)
    int32_t *blocks;            // [rows, top_blocks]
    int32_t *n_keep;            // [rows]
    float *fine;                // [rows, cand_cap]
    int32_t *out_idx;           // [rows, topk]
    int32_t *out_count;         // [rows]
    int n_rows, H, topk, blk, top_blocks, cand_cap, max_keys;
    int prefill;                // 1: row t is query t of one sequence (keys 0..t, shared reps)
};

// one warp per complete block: lane l averages dims 2l, 2l + 1 over the block
__global__ void __launch_bounds__(kHDescWarps * 32) hisa_describe_kernel(HisaArgs a) {
    const int row = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x * kHDescWarps + warp;
    const int64_t k0 = a.k_off[row];
    const int nb = (int)(min(a.k_off[row + 1] - k0, (int64_t)a.max_keys) / a.blk);
    if (j >= nb) return;
    const __nv_bfloat16 *src = a.k + (k0 + (int64_t)j * a.blk) * kHd + 2 * lane;
    float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 8
    for (int i = 0; i < a.blk; ++i) {
        const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(src + (size_t)i * kHd));
        s0 += v.x;
        s1 += v.y;
    }
    const float inv = 1.0f / (float)a.blk;
    *reinterpret_cast<float2 *>(a.rep + (a.b_off[row] + j) * kHd + 2 * lane) = make_float2(s0 * inv, s1 * inv);
}

// One warp scores 32 / HP blocks: lane l holds dims 2l, 2l + 1 of the HP
// (>= H, power of two) query heads; the partial dots (block i, head h) ->
// index i HP + h are reduce-scattered so lane v ends with index v; the HP
// lanes of a block then sum w_h ReLU(dot).
template <int HP>
__global__ void __launch_bounds__(kHCoarseWarps * 32) hisa_coarse_kernel(HisaArgs a) {
    constexpr int BPW = 32 / HP;
    const int row = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int nb;
    int64_t b0;
    if (a.prefill) {             // query row of one sequence: complete blocks below row + 1
        nb = (row + 1) / a.blk;
        b0 = 0;
        if (nb <= a.top_blocks) return;                      // every block is kept: no scores
    } else {
        const int64_t k0 = a.k_off[row];
        nb = (int)(min(a.k_off[row + 1] - k0, (int64_t)a.max_keys) / a.blk);
        b0 = a.b_off[row];
    }
    const int j0 = (blockIdx.x * kHCoarseWarps + warp) * BPW;
    if (j0 >= nb) return;                                    // warp-uniform
    float q[HP][2];
#pragma unroll
    for (int h = 0; h < HP; ++h) {
        float2 v = make_float2(0.0f, 0.0f);
        if (h < a.H)
            v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(a.q + ((size_t)row * a.H + h) * kHd + 2 * lane));
        q[h][0] = v.x;
        q[h][1] = v.y;
    }
    const float *rep = a.rep + b0 * kHd + 2 * lane;
    float v[32];
#pragma unroll
    for (int i = 0; i < BPW; ++i) {
        const float2 r = j0 + i < nb ? __ldcs(reinterpret_cast<const float2 *>(rep + (size_t)(j0 + i) * kHd))
                                     : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int h = 0; h < HP; ++h) v[i * HP + h] = fmaf(q[h][0], r.x, q[h][1] * r.y);
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
    const int h = lane % HP, i = lane / HP;
    float c = h < a.H ? a.w[(size_t)row * a.H + h] * fmaxf(v[0], 0.0f) : 0.0f;
    if (v[0] != v[0]) c = v[0];                              // a NaN dot stays NaN
#pragma unroll
    for (int o = 1; o < HP; o <<= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (h == 0 && j0 + i < nb) a.coarse[(size_t)row * (a.max_keys / a.blk) + j0 + i] = c;
}

// Exact top k of a CTA's KPT-per-thread keys (thread t owns entries
// [t KPT, t KPT + KPT)), ties to the smaller entry.  Returns per entry whether
// it is kept, the thread's first output slot and the number kept.
template <int KPT>
__device__ __forceinline__ void cta_topk(const uint32_t (&key)[KPT], const bool (&valid)[KPT], int k,
                                         bool (&take)[KPT], int &slot, int &n_sel, int2 *wtot) {
    int ph = 0;
    auto count_ge = [&](uint32_t c) -> int {
        int local = 0;
#pragma unroll
        for (int u = 0; u < KPT; ++u) local += (valid[u] && key[u] >= c) ? 1 : 0;
        if (KPT == 1) return __syncthreads_count(local);       // one barrier already
        return cta_count(local, ph);
    };
    uint32_t Tk = 0u;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t c = Tk | (1u << bit);
        if (count_ge(c) >= k) Tk = c;
    }
    const int need = k - (Tk == 0xffffffffu ? 0 : count_ge(Tk + 1u));
    int n_eq = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) n_eq += (valid[u] && key[u] == Tk) ? 1 : 0;
    int eq_before, dummy, t0, t1;
    cta_exscan2(n_eq, 0, eq_before, dummy, t0, t1, wtot);
    int n_take = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        const bool eq = valid[u] && key[u] == Tk;
        take[u] = (valid[u] && key[u] > Tk) || (eq && eq_before < need);
        eq_before += eq ? 1 : 0;
        n_take += take[u] ? 1 : 0;
    }
    int tok_dummy, tok_total;
    cta_exscan2(n_take, 0, slot, tok_dummy, n_sel, tok_total, wtot);
}

// one CTA per row: the kept blocks, ascending, -1 padded
template <int KPT>
__global__ void __launch_bounds__(kPickT) hisa_pick_blocks_kernel(HisaArgs a) {
    __shared__ int2 wtot[kPickT / 32 + 1];
    const int row = blockIdx.x, tid = threadIdx.x;
    const int64_t ctx = a.k_off[row + 1] - a.k_off[row];
    if (ctx > a.max_keys) {                  // the grids were sized by max_keys
        if (tid == 0) {
            raise_error(CRS_DEVERR_INDEX);
            a.n_keep[row] = 0;
        }
        for (int i = tid; i < a.top_blocks; i += kPickT) a.blocks[(size_t)row * a.top_blocks + i] = -1;
        return;
    }
    const int nb = (int)(ctx / a.blk);
    const float *c = a.coarse + (size_t)row * (a.max_keys / a.blk);
    uint32_t key[KPT];
    bool valid[KPT], take[KPT];
    bool nan = false;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        const int j = tid * KPT + u;
        valid[u] = j < nb;
        const float x = valid[u] ? c[j] : 0.0f;
        nan |= valid[u] && x != x;
        key[u] = valid[u] ? score_key(x) : 0u;
    }
    if (nan) raise_error(CRS_DEVERR_NONFINITE);
    const int k = min(a.top_blocks, nb);
    int slot = 0, n_sel = 0;
    if (k > 0) cta_topk<KPT>(key, valid, k, take, slot, n_sel, wtot);
    int32_t *out = a.blocks + (size_t)row * a.top_blocks;
    if (k > 0) {
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            if (take[u]) out[slot++] = tid * KPT + u;
    }
    for (int i = n_sel + tid; i < a.top_blocks; i += kPickT) out[i] = -1;
    if (tid == 0) a.n_keep[row] = n_sel;
}

// Prefill form, one warp per query row t: its complete blocks j < (t + 1) / blk
// sit KPL per lane (j = 32 u + lane), so word u of the row's kept-block bitmap is
// the warp's ballot for u.  The top_blocks blocks by (c desc, block asc): the k-th
// largest order-preserving key T bit by bit (warp counts), then every key > T and
// the first (in block order) of those equal to T.  Rows with at most top_blocks
// blocks keep them all.  Writes the bitmap [rows, keep_words] and the ascending
// list [rows, top_blocks] (-1 padded).
constexpr int kHPickWarps = 8;

template <int KPL>
__global__ void __launch_bounds__(kHPickWarps * 32) hisa_prefill_pick_kernel(HisaArgs a, uint32_t *keep,
                                                                           int keep_words) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kHPickWarps + warp;
    if (row >= a.n_rows) return;                             // warp-uniform
    const int nb = (row + 1) / a.blk;
    uint32_t *kw = keep + (size_t)row * keep_words;
    int32_t *out = a.blocks + (size_t)row * a.top_blocks;
    if (nb <= a.top_blocks) {
        for (int u = lane; u < keep_words; u += 32) {
            const int lo = 32 * u;
            kw[u] = nb >= lo + 32 ? 0xffffffffu : (nb <= lo ? 0u : ((1u << (nb - lo)) - 1u));
        }
        for (int i = lane; i < a.top_blocks; i += 32) out[i] = i < nb ? i : -1;
        return;
    }
    const float *c = a.coarse + (size_t)row * (a.max_keys / a.blk);
    uint32_t key[KPL];
    bool nan = false;
#pragma unroll
    for (int u = 0; u < KPL; ++u) {
        const int j = 32 * u + lane;
        const float x = j < nb ? c[j] : 0.0f;
        nan |= j < nb && x != x;
        key[u] = j < nb ? score_key(x) : 0u;
    }
    if (__any_sync(0xffffffffu, nan) && lane == 0) raise_error(CRS_DEVERR_NONFINITE);
    const int k = a.top_blocks;
    uint32_t T = 0u;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cnd = T | (1u << bit);
        int local = 0;
#pragma unroll
        for (int u = 0; u < KPL; ++u) local += (32 * u + lane < nb && key[u] >= cnd) ? 1 : 0;
        if ((int)__reduce_add_sync(0xffffffffu, (unsigned)local) >= k) T = cnd;
    }
    int gt = 0;
#pragma unroll
    for (int u = 0; u < KPL; ++u) gt += (32 * u + lane < nb && key[u] > T) ? 1 : 0;
    const int need = k - (int)__reduce_add_sync(0xffffffffu, (unsigned)gt);
    const uint32_t below = (1u << lane) - 1u;
    int eq_seen = 0, base = 0;
#pragma unroll
    for (int u = 0; u < KPL; ++u) {
        const bool in = 32 * u + lane < nb;
        const bool eq = in && key[u] == T;
        const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
        const bool tk = (in && key[u] > T) || (eq && eq_seen + __popc(eqm & below) < need);
        eq_seen += __popc(eqm);
        const uint32_t tm = __ballot_sync(0xffffffffu, tk);
        if (lane == 0 && u < keep_words) kw[u] = tm;
        if (tk) out[base + __popc(tm & below)] = 32 * u + lane;
        base += __popc(tm);
    }
    for (int u = KPL + lane; u < keep_words; u += 32) kw[u] = 0u;
    for (int i = base + lane; i < a.top_blocks; i += 32) out[i] = -1;
}

// grid (ceil((top_blocks + 1) / UP), rows), 256 threads: CTA x takes the UP =
// max(1, 256 / blk) units [x UP, x UP + UP); unit u < n_keep scores the keys
// of kept block u, unit top_blocks the open block; one key per thread and pass.
constexpr int kHFineThreads = 256;

__host__ __device__ inline int hisa_fine_units(int blk) { return blk >= kHFineThreads ? 1 : kHFineThreads / blk; }

__global__ void __launch_bounds__(kHFineThreads) hisa_fine_kernel(HisaArgs a) {
    __shared__ float sq[kHMaxHeads][kHd];
    __shared__ float sw[kHMaxHeads];
    const int row = blockIdx.y, t = threadIdx.x;
    const int64_t k0 = a.k_off[row];
    if (a.k_off[row + 1] - k0 > a.max_keys) return;
    const int ctx = (int)(a.k_off[row + 1] - k0);
    const int nb = ctx / a.blk;
    const int nkeep = a.n_keep[row];
    const int UP = hisa_fine_units(a.blk);
    const int u_first = blockIdx.x * UP;
    if (u_first >= nkeep && u_first + UP <= a.top_blocks) return;   // CTA-uniform: nothing kept here
    for (int e = t; e < a.H * kHd; e += kHFineThreads)
        sq[e / kHd][e % kHd] = __bfloat162float(a.q[(size_t)row * a.H * kHd + e]);
    if (t < a.H) sw[t] = a.w[(size_t)row * a.H + t];
    __syncthreads();
    for (int e = t; e < UP * a.blk; e += kHFineThreads) {
        const int u = u_first + e / a.blk, i = e % a.blk;
        int pos0, len, slot0;
        if (u < a.top_blocks) {
            if (u >= nkeep) continue;
            pos0 = a.blocks[(size_t)row * a.top_blocks + u] * a.blk;
            len = a.blk;
            slot0 = u * a.blk;
        } else if (u == a.top_blocks) {
            pos0 = nb * a.blk;
            len = ctx - pos0;
            slot0 = nkeep * a.blk;
        } else {
            continue;
        }
        if (i >= len) continue;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.k + (k0 + pos0 + i) * kHd);
        float dot[kHMaxHeads];
#pragma unroll
        for (int h = 0; h < kHMaxHeads; ++h) dot[h] = 0.0f;
#pragma unroll
        for (int c = 0; c < kHd / 8; ++c) {
            const uint4 raw = __ldg(src + c);
            const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 kv = __bfloat1622float2(p2[q]);
                const int d = c * 8 + 2 * q;
#pragma unroll
                for (int h = 0; h < kHMaxHeads; ++h)
                    if (h < a.H) dot[h] = fmaf(sq[h][d], kv.x, fmaf(sq[h][d + 1], kv.y, dot[h]));
            }
        }
        float r = 0.0f;
#pragma unroll
        for (int h = 0; h < kHMaxHeads; ++h)
            if (h < a.H) r += sw[h] * (dot[h] != dot[h] ? dot[h] : fmaxf(dot[h], 0.0f));
        a.fine[(size_t)row * a.cand_cap + slot0 + i] = r;
    }
}

// one CTA per row: the topk candidates (slot order = ascending position)
template <int KPT>
__global__ void __launch_bounds__(kPickT) hisa_pick_tokens_kernel(HisaArgs a) {
    __shared__ int2 wtot[kPickT / 32 + 1];
    const int row = blockIdx.x, tid = threadIdx.x;
    const int64_t ctx64 = a.k_off[row + 1] - a.k_off[row];
    const int ctx = ctx64 > a.max_keys ? 0 : (int)ctx64;    // an oversized row returns nothing
    const int nb = ctx / a.blk;
    const int nkeep = a.n_keep[row];
    const int n_cand = nkeep * a.blk + (ctx - nb * a.blk);
    const float *f = a.fine + (size_t)row * a.cand_cap;
    uint32_t key[KPT];
    bool valid[KPT], take[KPT];
    bool nan = false;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
        const int c = tid * KPT + u;
        valid[u] = c < n_cand;
        const float x = valid[u] ? f[c] : 0.0f;
        nan |= valid[u] && x != x;
        key[u] = valid[u] ? score_key(x) : 0u;
    }
    if (nan) raise_error(CRS_DEVERR_NONFINITE);
    const int k = min(a.topk, n_cand);
    int slot = 0, n_sel = 0;
    if (k > 0) cta_topk<KPT>(key, valid, k, take, slot, n_sel, wtot);
    int32_t *out = a.out_idx + (size_t)row * a.topk;
    if (k > 0) {
        const int32_t *blocks = a.blocks + (size_t)row * a.top_blocks;
#pragma unroll
        for (int u = 0; u < KPT; ++u)
            if (take[u]) {
                const int c = tid * KPT + u;
                const int b = c / a.blk;
                out[slot++] = b < nkeep ? blocks[b] * a.blk + (c - b * a.blk) : nb * a.blk + (c - nkeep * a.blk);
            }
    }
    for (int i = n_sel + tid; i < a.topk; i += kPickT) out[i] = -1;
    if (tid == 0) a.out_count[row] = n_sel;
}

struct HisaWs {
    float *coarse, *fine;
    int32_t *blocks, *n_keep;
    size_t total;
};

static int hisa_validate(const crs_hisa_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->n_rows < 1 || p->n_idx_heads < 1 || p->topk < 1 || p->blk < 1 || p->top_blocks < 1 ||
        p->max_keys < 0)
        return CRS_ERR_INVALID_ARG;
    if (p->d_idx != kHd || p->n_idx_heads > kHMaxHeads || p->blk > 256 || p->topk > 4096)
        return CRS_ERR_UNSUPPORTED;
    if ((long long)p->top_blocks * p->blk + p->blk > kHMaxCand) return CRS_ERR_UNSUPPORTED;
    if ((long long)p->max_keys / p->blk > 8LL * kPickT) return CRS_ERR_UNSUPPORTED;
    return CRS_OK;
}

static void hisa_ws_layout(const crs_hisa_params *p, HisaWs &w, char *base) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t max_blocks = (size_t)p->n_rows * (p->max_keys / p->blk);
    const size_t cand_cap = (size_t)p->top_blocks * p->blk + p->blk;
    size_t off = 0;
    auto take = [&](size_t bytes) { char *q = base ? base + off : nullptr; off += al(bytes); return q; };
    w.coarse = reinterpret_cast<float *>(take(max(size_t(1), max_blocks) * 4));
    w.fine = reinterpret_cast<float *>(take((size_t)p->n_rows * cand_cap * 4));
    w.blocks = reinterpret_cast<int32_t *>(take((size_t)p->n_rows * p->top_blocks * 4));
    w.n_keep = reinterpret_cast<int32_t *>(take((size_t)p->n_rows * 4));
    w.total = off;
}

static int hisa_kpt(int n) {
    return n <= kPickT ? 1 : n <= 2 * kPickT ? 2 : n <= 4 * kPickT ? 4 : n <= 8 * kPickT ? 8 : 16;
}

}  // namespace crs

using namespace crs;

extern "C" int crs_hisa_describe(const crs_hisa_params *p, const void *k_idx, const int64_t *k_offsets,
                                 const int64_t *blk_offsets, float *rep, void *stream) {
    int st = hisa_validate(p);
    if (st) return st;
    if (!k_idx || !k_offsets || !blk_offsets || !rep) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k_idx) & 3) || (reinterpret_cast<uintptr_t>(rep) & 7))
        return CRS_ERR_INVALID_ARG;
    const int max_blocks = p->max_keys / p->blk;
    if (max_blocks == 0) return CRS_OK;
    HisaArgs a{};
    a.k = static_cast<const __nv_bfloat16 *>(k_idx);
    a.k_off = k_offsets;
    a.b_off = blk_offsets;
    a.rep = rep;
    a.n_rows = p->n_rows;
    a.blk = p->blk;
    a.max_keys = p->max_keys;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        ProfScope _ps(K_HISA, s);
        hisa_describe_kernel<<<dim3(ceil_div(max_blocks, kHDescWarps), p->n_rows), kHDescWarps * 32, 0, s>>>(a);
    }
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

extern "C" size_t crs_hisa_topk_workspace_size(const crs_hisa_params *p) {
    if (hisa_validate(p)) return 0;
    HisaWs w;
    hisa_ws_layout(p, w, nullptr);
    return w.total;
}

extern "C" int crs_hisa_topk(const crs_hisa_params *p, const void *q_idx, const float *w, const void *k_idx,
                             const int64_t *k_offsets, const float *rep, const int64_t *blk_offsets,
                             int32_t *out_blocks, int32_t *out_idx, int32_t *out_count, void *ws,
                             size_t ws_bytes, void *stream) {
    int st = hisa_validate(p);
    if (st) return st;
    if (!q_idx || !w || !k_idx || !k_offsets || !rep || !blk_offsets || !out_idx || !out_count)
        return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q_idx) & 3) || (reinterpret_cast<uintptr_t>(k_idx) & 15) ||
        (reinterpret_cast<uintptr_t>(rep) & 7))
        return CRS_ERR_INVALID_ARG;
    const size_t need = crs_hisa_topk_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    HisaWs hw;
    hisa_ws_layout(p, hw, static_cast<char *>(ws));
    HisaArgs a{};
    a.q = static_cast<const __nv_bfloat16 *>(q_idx);
    a.w = w;
    a.k = static_cast<const __nv_bfloat16 *>(k_idx);
    a.k_off = k_offsets;
    a.b_off = blk_offsets;
    a.rep = const_cast<float *>(rep);
    a.coarse = hw.coarse;
    a.blocks = out_blocks ? out_blocks : hw.blocks;
    a.n_keep = hw.n_keep;
    a.fine = hw.fine;
    a.out_idx = out_idx;
    a.out_count = out_count;
    a.n_rows = p->n_rows;
    a.H = p->n_idx_heads;
    a.topk = p->topk;
    a.blk = p->blk;
    a.top_blocks = p->top_blocks;
    a.cand_cap = p->top_blocks * p->blk + p->blk;
    a.max_keys = p->max_keys;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int max_blocks = p->max_keys / p->blk;
    const int HP = p->n_idx_heads <= 1 ? 1 : p->n_idx_heads <= 2 ? 2 : p->n_idx_heads <= 4 ? 4 : 8;
    ProfScope _ps(K_HISA, s);
    if (max_blocks > 0) {
        const dim3 gc(ceil_div(max_blocks, kHCoarseWarps * (32 / HP)), p->n_rows);
        switch (HP) {
        case 1: hisa_coarse_kernel<1><<<gc, kHCoarseWarps * 32, 0, s>>>(a); break;
        case 2: hisa_coarse_kernel<2><<<gc, kHCoarseWarps * 32, 0, s>>>(a); break;
        case 4: hisa_coarse_kernel<4><<<gc, kHCoarseWarps * 32, 0, s>>>(a); break;
        default: hisa_coarse_kernel<8><<<gc, kHCoarseWarps * 32, 0, s>>>(a); break;
        }
    }
    switch (hisa_kpt(max_blocks)) {
    case 1: hisa_pick_blocks_kernel<1><<<p->n_rows, kPickT, 0, s>>>(a); break;
    case 2: hisa_pick_blocks_kernel<2><<<p->n_rows, kPickT, 0, s>>>(a); break;
    case 4: hisa_pick_blocks_kernel<4><<<p->n_rows, kPickT, 0, s>>>(a); break;
    default: hisa_pick_blocks_kernel<8><<<p->n_rows, kPickT, 0, s>>>(a); break;
    }
    hisa_fine_kernel<<<dim3(ceil_div(p->top_blocks + 1, hisa_fine_units(p->blk)), p->n_rows), kHFineThreads, 0, s>>>(a);
    switch (hisa_kpt(a.cand_cap)) {
    case 1: hisa_pick_tokens_kernel<1><<<p->n_rows, kPickT, 0, s>>>(a); break;
    case 2: hisa_pick_tokens_kernel<2><<<p->n_rows, kPickT, 0, s>>>(a); break;
    case 4: hisa_pick_tokens_kernel<4><<<p->n_rows, kPickT, 0, s>>>(a); break;
    case 8: hisa_pick_tokens_kernel<8><<<p->n_rows, kPickT, 0, s>>>(a); break;
    default: hisa_pick_tokens_kernel<16><<<p->n_rows, kPickT, 0, s>>>(a); break;
    }
    _ps.more(max_blocks > 0 ? 3 : 2);             // coarse, block pick, fine, token pick
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

// ------------------------------------------------------------ prefill form --
namespace crs {
constexpr int kHpBlk = 64;               // one block = one 64-key tile of the tensor-core indexer

static int hisa_prefill_validate(const crs_hisa_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->n_rows < 1 || p->n_idx_heads < 1 || p->topk < 1 || p->blk < 1 || p->top_blocks < 1)
        return CRS_ERR_INVALID_ARG;
    if (p->d_idx != kHd || p->n_idx_heads != 4 || p->blk != kHpBlk || p->topk > 2048)
        return CRS_ERR_UNSUPPORTED;
    if ((long long)p->top_blocks * p->blk < p->topk) return CRS_ERR_UNSUPPORTED;
    if (p->n_rows / p->blk > 1024 || p->n_rows > (1 << 19)) return CRS_ERR_UNSUPPORTED;
    return CRS_OK;
}

struct HisaPrefillWs {
    float *coarse;
    int32_t *blocks;
    uint32_t *keep;
    void *tc;
    int keep_words;
    size_t total;
};

static void hisa_prefill_layout(const crs_hisa_params *p, HisaPrefillWs &w, char *base) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const int n = p->n_rows, nbk = n / p->blk;
    w.keep_words = max(1, ceil_div(nbk, 32));
    size_t off = 0;
    auto take = [&](size_t bytes) { char *q = base ? base + off : nullptr; off += al(bytes); return q; };
    w.coarse = reinterpret_cast<float *>(take((size_t)n * max(nbk, 1) * 4));
    w.blocks = reinterpret_cast<int32_t *>(take((size_t)n * p->top_blocks * 4));
    w.keep = reinterpret_cast<uint32_t *>(take((size_t)n * w.keep_words * 4));
    crs_indexer_params ip{CRS_IDX_PREFILL, n, p->n_idx_heads, p->d_idx, p->topk, 0};
    w.tc = take(prefill_tc_workspace(&ip));
    w.total = off;
}
}  // namespace crs

extern "C" size_t crs_hisa_topk_prefill_workspace_size(const crs_hisa_params *p) {
    if (hisa_prefill_validate(p)) return 0;
    HisaPrefillWs w;
    hisa_prefill_layout(p, w, nullptr);
    return w.total;
}

extern "C" int crs_hisa_topk_prefill(const crs_hisa_params *p, const void *q_idx, const float *w, const void *k_idx,
                                     const float *rep, int32_t *out_blocks, int32_t *out_idx, int32_t *out_count,
                                     void *ws, size_t ws_bytes, void *stream) {
    int st = hisa_prefill_validate(p);
    if (st) return st;
    if (!q_idx || !w || !k_idx || !rep || !out_idx || !out_count) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q_idx) & 15) || (reinterpret_cast<uintptr_t>(k_idx) & 15) ||
        (reinterpret_cast<uintptr_t>(rep) & 7))
        return CRS_ERR_INVALID_ARG;
    const size_t need = crs_hisa_topk_prefill_workspace_size(p);
    if (!ws || ws_bytes < need) return CRS_ERR_WORKSPACE;
    HisaPrefillWs hw;
    hisa_prefill_layout(p, hw, static_cast<char *>(ws));
    const int n = p->n_rows, nbk = n / p->blk;
    HisaArgs a{};
    a.q = static_cast<const __nv_bfloat16 *>(q_idx);
    a.w = w;
    a.k = static_cast<const __nv_bfloat16 *>(k_idx);
    a.rep = const_cast<float *>(rep);
    a.coarse = hw.coarse;
    a.blocks = out_blocks ? out_blocks : hw.blocks;
    a.n_rows = n;
    a.H = p->n_idx_heads;
    a.topk = p->topk;
    a.blk = p->blk;
    a.top_blocks = p->top_blocks;
    a.max_keys = n;
    a.prefill = 1;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        ProfScope _ps(K_HISA, s);
        if (nbk > p->top_blocks) {
            const dim3 gc(ceil_div(nbk, kHCoarseWarps * (32 / 4)), n);
            hisa_coarse_kernel<4><<<gc, kHCoarseWarps * 32, 0, s>>>(a);
            _ps.more(1);
        }
        const int kpl = ceil_div(max(nbk, 1), 32);
        const unsigned gp = (unsigned)ceil_div(n, kHPickWarps);
        if (kpl <= 1) hisa_prefill_pick_kernel<1><<<gp, kHPickWarps * 32, 0, s>>>(a, hw.keep, hw.keep_words);
        else if (kpl <= 2) hisa_prefill_pick_kernel<2><<<gp, kHPickWarps * 32, 0, s>>>(a, hw.keep, hw.keep_words);
        else if (kpl <= 4) hisa_prefill_pick_kernel<4><<<gp, kHPickWarps * 32, 0, s>>>(a, hw.keep, hw.keep_words);
        else if (kpl <= 8) hisa_prefill_pick_kernel<8><<<gp, kHPickWarps * 32, 0, s>>>(a, hw.keep, hw.keep_words);
        else if (kpl <= 16) hisa_prefill_pick_kernel<16><<<gp, kHPickWarps * 32, 0, s>>>(a, hw.keep, hw.keep_words);
        else hisa_prefill_pick_kernel<32><<<gp, kHPickWarps * 32, 0, s>>>(a, hw.keep, hw.keep_words);
    }
    CRS_CHECK_LAUNCH();
    // the token level: the tensor-core prefill indexer with every row's kept blocks
    const crs_indexer_params ip{CRS_IDX_PREFILL, n, p->n_idx_heads, p->d_idx, p->topk, 0};
    return launch_prefill_tc(&ip, q_idx, w, k_idx, out_idx, out_count, hw.tc, s, hw.keep, hw.keep_words,
                             p->top_blocks);
}
