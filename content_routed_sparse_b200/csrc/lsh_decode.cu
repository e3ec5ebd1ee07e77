// LSH attention in decode: fixed hash, growable bucket lists, paged KV, sm_100a.
//
// [P1] PaperTrace 2.1.1 §5.2 "Prefill、Decode 与 KV 状态": with the hash fixed, a
// new key gets its bucket ids in O(d R) and is appended to the bucket lists;
// the query computes its own bucket ids and reads those lists; each list needs
// a growable page table, a length and a capacity; the KV itself stays paged by
// time and the lists hold logical positions, so K/V are gathered through the
// block table.  [P2] PaperTrace 2.2 (block_table maps logical positions to
// physical pages).  The neighbourhood of the newest token t is every earlier
// token sharing a bucket in some round, counted once (pairs met in an earlier
// round are skipped), without t itself when no_self; keys are the shared-QK
// vectors normalised (key_norm), as in the prefill path.
//
// State (all caller-owned device memory, layouts in include/crs.h):
//   K_pool, V_pool [pages, P, H, d] bf16 + block_table [S, max_pages]
//   bucket_store [S, H, R, max_len] u8      bucket of every token and round
//   list_table [S, H, R, b, list_pages]     page ids of each bucket list
//   list_len [S, H, R, b], list_pool [n_list_pages, Lp], alloc (pages used)
//   seq_len [S]                             tokens already in each row
// Kernels:
//   lsd_hash_kernel        one warp per (row, head, token, round): u = x R_{h,r}
//                          (fp32 FMA chain in index order, as the prefill hash),
//                          bucket = argmax [u; -u], ties to the lower index
//   lsd_store_kv_kernel    normalised key and value rows into their pages
//   lsd_append_kernel      one warp per (row, head, round): tokens in position
//                          order, lanes grouped by bucket (match_any), one
//                          length update and page allocation per group
//   lsd_attend_kernel      one CTA per (row, head): the lists' kept entries are
//                          compacted into shared memory, then 8-lane groups
//                          score and accumulate them (online softmax), groups
//                          merged in order
//   lsd_advance_kernel     seq_len += tokens appended
#include "common.cuh"

namespace crs {

constexpr int kLdD = 64;                  // head dim
constexpr int kLdMaxRounds = 8;

struct LdState {
    __nv_bfloat16 *K, *V;
    const int32_t *block_table;
    uint8_t *bucket;
    int32_t *list_table, *list_len, *list_pool, *alloc, *seq_len;
};

struct LdArgs {
    LdState st;
    const __nv_bfloat16 *X;   // new tokens [S, n_new, H, d]
    const __nv_bfloat16 *Vn;  // new values [S, n_new, H, d]
    const float *rot;         // [H, R, d, b/2]
    float *O, *lse;           // [S, H, d], [S, H]
    int32_t *count;           // [S, H]
    int S, H, n_new, b, R, P, max_pages, Lp, list_pages, n_list_pages, max_len, no_self, key_norm;
    float scale;
};

__device__ __forceinline__ size_t ld_list_id(const LdArgs &a, int s, int h, int r, int bucket) {
    return (((size_t)s * a.H + h) * a.R + r) * a.b + bucket;
}

// grid (S * H, n_new * R / 8): warp w handles token tok = w / R, round r = w % R
__global__ void __launch_bounds__(256) lsd_hash_kernel(LdArgs a) {
    const int sh = blockIdx.x, s = sh / a.H, h = sh - s * a.H;
    const int w = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= a.n_new * a.R) return;
    const int tok = w / a.R, r = w - tok * a.R;
    const int t = a.st.seq_len[s] + tok;
    if (t >= a.max_len) return;                              // flagged by lsd_append_kernel
    const __nv_bfloat16 *x = a.X + (((size_t)s * a.n_new + tok) * a.H + h) * kLdD;
    const int half = a.b / 2;
    const float *R = a.rot + ((size_t)h * a.R + r) * kLdD * half;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    // the row in registers (two values per lane, broadcast by shuffles); the chain
    // itself stays one FMA per term in index order
    const float2 xl = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162 *>(x)[lane]);
    for (int k0 = 0; k0 < half; k0 += 32) {             // same trip count in every lane
        const int k = k0 + lane;
        const bool kv = k < half;
        float u = 0.0f;
#pragma unroll
        for (int i = 0; i < kLdD; ++i) {
            const float xi = __shfl_sync(0xffffffffu, (i & 1) ? xl.y : xl.x, i >> 1);
            u = fmaf(xi, kv ? __ldg(R + (size_t)i * half + k) : 0.0f, u);
        }
        if (kv) {
            if (u > best || (u == best && k < bi)) { best = u; bi = k; }
            if (-u > best || (-u == best && k + half < bi)) { best = -u; bi = k + half; }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    if (bi >= a.b) {                                         // every u NaN: no maximum
        bi = 0;
        if (lane == 0) raise_error(CRS_DEVERR_NONFINITE);
    }
    if (lane == 0) a.st.bucket[(((size_t)s * a.H + h) * a.R + r) * a.max_len + t] = (uint8_t)bi;
}

// one warp per (row, token, head): the key (normalised) and value rows into their page
__global__ void __launch_bounds__(256) lsd_store_kv_kernel(LdArgs a) {
    const int s = blockIdx.y, w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= a.n_new * a.H) return;
    const int tok = w / a.H, h = w - tok * a.H;
    const int t = a.st.seq_len[s] + tok;
    if (t >= a.max_len || t / a.P >= a.max_pages) return;    // flagged by lsd_append_kernel
    const size_t src = (((size_t)s * a.n_new + tok) * a.H + h) * kLdD + 2 * lane;
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(a.X + src));
    float sc = 1.0f;
    if (a.key_norm) {
        const float n2 = warp_sum(x.x * x.x + x.y * x.y);
        sc = n2 > 0.0f ? rsqrtf(n2) : 0.0f;
    }
    const int page = a.st.block_table[(size_t)s * a.max_pages + t / a.P];
    const size_t dst = (((size_t)page * a.P + t % a.P) * a.H + h) * kLdD + 2 * lane;
    *reinterpret_cast<__nv_bfloat162 *>(a.st.K + dst) = __floats2bfloat162_rn(x.x * sc, x.y * sc);
    *reinterpret_cast<__nv_bfloat162 *>(a.st.V + dst) = *reinterpret_cast<const __nv_bfloat162 *>(a.Vn + src);
}

// one warp per (row, head, round): append the new tokens in position order
__global__ void __launch_bounds__(256) lsd_append_kernel(LdArgs a) {
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= a.S * a.H * a.R) return;
    const int r = w % a.R, sh = w / a.R, s = sh / a.H, h = sh - s * a.H;
    const int t0 = a.st.seq_len[s];
    const uint8_t *bk = a.st.bucket + (((size_t)s * a.H + h) * a.R + r) * a.max_len;
    const int cap = a.list_pages * a.Lp;
    for (int c = 0; c < a.n_new; c += 32) {
        const int tok = c + lane;
        const int t = t0 + tok;
        bool live = tok < a.n_new;
        if (live && (t >= a.max_len || t / a.P >= a.max_pages)) {
            raise_error(CRS_DEVERR_CAPACITY);               // no room for the token itself
            live = false;
        }
        const int bucket = live ? (int)bk[t] : -1 - lane;
        const unsigned grp = __match_any_sync(0xffffffffu, bucket);
        const int leader = __ffs(grp) - 1;
        const int rank = __popc(grp & ((1u << lane) - 1u));
        const int n_grp = __popc(grp);
        const size_t lid = live ? ld_list_id(a, s, h, r, bucket) : 0;
        int L = 0;
        if (live && lane == leader) {
            L = a.st.list_len[lid];
            const int L1 = min(cap, L + n_grp);
            // pages this group starts: those holding entries L .. L1-1 that do not exist yet
            const int have = (L + a.Lp - 1) / a.Lp, need = (L1 + a.Lp - 1) / a.Lp;
            if (need > have) {
                const int pg = atomicAdd(a.st.alloc, need - have);
                for (int q = have; q < need; ++q)
                    a.st.list_table[lid * a.list_pages + q] =
                        pg + (q - have) < a.n_list_pages ? pg + (q - have) : -1;
            }
            if (L + n_grp > cap) raise_error(CRS_DEVERR_CAPACITY);
            a.st.list_len[lid] = L1;
        }
        L = __shfl_sync(0xffffffffu, L, leader);
        __syncwarp();
        if (live) {
            const int e = L + rank;
            if (e < cap) {
                const int pg = a.st.list_table[lid * a.list_pages + e / a.Lp];
                if (pg >= 0) a.st.list_pool[(size_t)pg * a.Lp + e % a.Lp] = t;
                else raise_error(CRS_DEVERR_CAPACITY);       // the page pool ran out
            }
        }
        __syncwarp();
    }
}

// One CTA per (row, head): the newest token t attends to its buckets' lists.
// Candidates are taken round by round; entry j of round r is skipped when j > t,
// when j == t (no_self) or when j shares an earlier round's bucket with t
// (already met).
//   1. the 256 threads walk the rounds' lists as one sequence (round by round,
//      entries in order), two entries each per pass (list page -> entry ->
//      earlier buckets and block table), and the kept
//      candidates' K/V row indices are compacted into shared memory in that order
//      (warp ballots, warp offsets), up to kLdCap at a time;
//   2. 32 groups of 8 lanes take the candidates in turn: lane g of a group loads
//      16 bytes (columns [8g, 8g + 8)) of the K and the V row, three shuffles
//      give the score, and the group keeps an online softmax (m, l, 8 outputs);
//   3. the 32 group states are merged in group order.
constexpr int kLdAttThreads = 256;
constexpr int kLdCap = 2048;               // candidate rows held in shared memory
constexpr int kLdGroups = kLdAttThreads / 8;

struct LdGroup {
    float m, l, acc[8];
    int cnt;
};

// Scores and accumulates the candidates c = G, G + 32, ... < nc of the buffer,
// four per pass (their K and V loads in flight together), in that order.  The
// loop runs the same number of times in every lane (the score shuffles need the
// whole warp); a group past the end loads nothing and keeps its state.
constexpr int kLdUnroll = 4;

__device__ __forceinline__ void lsd_consume(const LdArgs &a, const uint32_t *crow, int nc, int G, int g,
                                            const float (&qv)[8], LdGroup &st) {
    for (int c0 = 0; c0 < nc; c0 += kLdUnroll * kLdGroups) {
        uint4 kraw[kLdUnroll], vraw[kLdUnroll];
        bool valid[kLdUnroll];
#pragma unroll
        for (int u = 0; u < kLdUnroll; ++u) {
            const int c = c0 + u * kLdGroups + G;
            valid[u] = c < nc;
            kraw[u] = vraw[u] = make_uint4(0u, 0u, 0u, 0u);
            if (valid[u]) {
                const size_t row = (size_t)crow[c] * kLdD + 8 * g;
                kraw[u] = __ldg(reinterpret_cast<const uint4 *>(a.st.K + row));
                vraw[u] = __ldg(reinterpret_cast<const uint4 *>(a.st.V + row));
            }
        }
#pragma unroll
        for (int u = 0; u < kLdUnroll; ++u) {
            const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kraw[u]);
            float dot = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 kv = __bfloat1622float2(k2[e]);
                dot = fmaf(qv[2 * e], kv.x, fmaf(qv[2 * e + 1], kv.y, dot));
            }
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            dot += __shfl_xor_sync(0xffffffffu, dot, 4);
            if (valid[u]) {
                const float mn = fmaxf(st.m, dot);
                const float corr = __expf(st.m - mn), p = __expf(dot - mn);
                st.l = st.l * corr + p;
                const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vraw[u]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 vv = __bfloat1622float2(v2[e]);
                    st.acc[2 * e] = fmaf(p, vv.x, st.acc[2 * e] * corr);
                    st.acc[2 * e + 1] = fmaf(p, vv.y, st.acc[2 * e + 1] * corr);
                }
                st.m = mn;
                ++st.cnt;
            }
        }
    }
}

__global__ void __launch_bounds__(kLdAttThreads, 4) lsd_attend_kernel(LdArgs a) {
    __shared__ uint32_t crow[kLdCap];
    __shared__ int wcount[kLdAttThreads / 32];
    __shared__ float gm[kLdGroups], gl[kLdGroups];
    __shared__ int gc[kLdGroups];
    __shared__ float go[kLdGroups][kLdD];
    const int sh = blockIdx.x, s = sh / a.H, h = sh - s * a.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = tid >> 3, g = tid & 7;
    const int t = a.st.seq_len[s];                           // the newest token
    if (t >= a.max_len) {                                    // no room: flagged by the append
        if (tid < kLdD) a.O[((size_t)s * a.H + h) * kLdD + tid] = 0.0f;
        if (tid == 0) {
            a.lse[(size_t)s * a.H + h] = -INFINITY;
            if (a.count) a.count[(size_t)s * a.H + h] = 0;
        }
        return;
    }
    float qv[8];
    {
        const size_t q_off = ((size_t)s * a.n_new * a.H + h) * kLdD + 8 * g;   // token 0 of the step
        const uint4 raw = *reinterpret_cast<const uint4 *>(a.X + q_off);
        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 f = __bfloat1622float2(p2[u]);
            qv[2 * u] = a.scale * f.x;
            qv[2 * u + 1] = a.scale * f.y;
        }
    }
    uint8_t tb[kLdMaxRounds];
    const uint8_t *bk = a.st.bucket + ((size_t)s * a.H + h) * a.R * a.max_len;
#pragma unroll
    for (int r = 0; r < kLdMaxRounds; ++r) tb[r] = r < a.R ? bk[(size_t)r * a.max_len + t] : 0;
    LdGroup st;
    st.m = -INFINITY;
    st.l = 0.0f;
    st.cnt = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) st.acc[c] = 0.0f;
    // the rounds' entries as one sequence, round by round (cum = start of each round)
    int cum[kLdMaxRounds + 1];
    cum[0] = 0;
#pragma unroll
    for (int r = 0; r < kLdMaxRounds; ++r)
        cum[r + 1] = cum[r] + (r < a.R ? min(a.st.list_len[ld_list_id(a, s, h, r, tb[r])], a.list_pages * a.Lp) : 0);
    const int total_entries = cum[kLdMaxRounds];
    int nc = 0;                                              // candidates buffered (CTA-uniform)
    for (int base = 0; base < total_entries; base += 2 * kLdAttThreads) {
        bool keep[2];
        uint32_t row[2];
        int pg[2], j[2], rr[2], e[2];
        size_t lid[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int f = base + u * kLdAttThreads + tid;
            int r = 0;
#pragma unroll
            for (int q = 1; q < kLdMaxRounds; ++q) r += (q < a.R && f >= cum[q]) ? 1 : 0;
            rr[u] = r;
            e[u] = f - cum[r];
            lid[u] = ld_list_id(a, s, h, r, tb[r]);
            pg[u] = f < total_entries ? a.st.list_table[lid[u] * a.list_pages + e[u] / a.Lp] : -1;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) j[u] = pg[u] >= 0 ? a.st.list_pool[(size_t)pg[u] * a.Lp + e[u] % a.Lp] : -1;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            keep[u] = j[u] >= 0 && j[u] <= t && !(a.no_self && j[u] == t);
            row[u] = 0u;
            if (keep[u] && j[u] / a.P >= a.max_pages) {         // no page-table slot for it
                raise_error(CRS_DEVERR_INDEX);
                keep[u] = false;
            }
            if (keep[u]) {
                bool met = false;
                for (int r2 = 0; r2 < rr[u]; ++r2) met |= bk[(size_t)r2 * a.max_len + j[u]] == tb[r2];
                const int page = a.st.block_table[(size_t)s * a.max_pages + j[u] / a.P];
                keep[u] = !met;
                row[u] = (uint32_t)(((size_t)page * a.P + j[u] % a.P) * a.H + h);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            // compact in entry order: warp ballot, then the earlier warps' counts
            const uint32_t bal = __ballot_sync(0xffffffffu, keep[u]);
            if (lane == 0) wcount[warp] = __popc(bal);
            __syncthreads();
            int off = nc, total = 0;
#pragma unroll
            for (int w = 0; w < kLdAttThreads / 32; ++w) {
                const int cw = wcount[w];
                if (w < warp) off += cw;
                total += cw;
            }
            if (keep[u]) crow[off + __popc(bal & ((1u << lane) - 1u))] = row[u];
            nc += total;
            __syncthreads();
            if (nc > kLdCap - kLdAttThreads) {               // room for one more pass of 256
                lsd_consume(a, crow, nc, G, g, qv, st);
                nc = 0;
                __syncthreads();
            }
        }
    }
    lsd_consume(a, crow, nc, G, g, qv, st);
    // merge the 32 group states in group order
    if (g == 0) {
        gm[G] = st.m;
        gl[G] = st.l;
        gc[G] = st.cnt;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) go[G][8 * g + c] = st.acc[c];
    __syncthreads();
    if (tid < kLdD) {
        float M = -INFINITY;
        int C = 0;
        for (int w = 0; w < kLdGroups; ++w) {
            M = fmaxf(M, gm[w]);
            C += gc[w];
        }
        float L = 0.0f, acc = 0.0f;
        for (int w = 0; w < kLdGroups; ++w) {
            const float f = gc[w] > 0 ? __expf(gm[w] - M) : 0.0f;
            L += gl[w] * f;
            acc += go[w][tid] * f;
        }
        a.O[((size_t)s * a.H + h) * kLdD + tid] = C > 0 ? acc / L : 0.0f;
        if (tid == 0) {
            a.lse[(size_t)s * a.H + h] = C > 0 ? M + logf(L) : -INFINITY;
            if (a.count) a.count[(size_t)s * a.H + h] = C;
        }
    }
}

__global__ void lsd_advance_kernel(int32_t *seq_len, int S, int n_new, int max_len) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s < S) seq_len[s] = min(max_len, seq_len[s] + n_new);
}

static int ld_validate(const crs_lsh_decode_params *p) {
    if (!p) return CRS_ERR_INVALID_ARG;
    if (p->n_seq < 1 || p->n_heads < 1 || p->n_buckets < 2 || (p->n_buckets & 1) || p->n_rounds < 1 ||
        p->page_size < 1 || p->max_pages < 1 || p->list_page < 1 || p->list_pages < 1 || p->n_list_pages < 1 ||
        p->max_len < 1)
        return CRS_ERR_INVALID_ARG;
    if (p->d != kLdD || p->n_buckets > 256 || p->n_rounds > kLdMaxRounds) return CRS_ERR_UNSUPPORTED;
    return CRS_OK;
}

static LdArgs ld_args(const crs_lsh_decode_params *p, const crs_lsh_decode_state *st) {
    LdArgs a{};
    a.st.K = static_cast<__nv_bfloat16 *>(st->k_pool);
    a.st.V = static_cast<__nv_bfloat16 *>(st->v_pool);
    a.st.block_table = st->block_table;
    a.st.bucket = st->bucket_store;
    a.st.list_table = st->list_table;
    a.st.list_len = st->list_len;
    a.st.list_pool = st->list_pool;
    a.st.alloc = st->alloc;
    a.st.seq_len = st->seq_len;
    a.S = p->n_seq;
    a.H = p->n_heads;
    a.b = p->n_buckets;
    a.R = p->n_rounds;
    a.P = p->page_size;
    a.max_pages = p->max_pages;
    a.Lp = p->list_page;
    a.list_pages = p->list_pages;
    a.n_list_pages = p->n_list_pages;
    a.max_len = p->max_len;
    a.no_self = p->no_self;
    a.key_norm = p->key_norm;
    a.scale = p->scale;
    return a;
}

static bool ld_state_ok(const crs_lsh_decode_state *st) {
    return st && st->k_pool && st->v_pool && st->block_table && st->bucket_store && st->list_table &&
           st->list_len && st->list_pool && st->alloc && st->seq_len &&
           !((reinterpret_cast<uintptr_t>(st->k_pool) | reinterpret_cast<uintptr_t>(st->v_pool)) & 15);
}

// hash + store + append + (optionally) attend + advance for n_new tokens per row
static int ld_run(const crs_lsh_decode_params *p, const crs_lsh_decode_state *st, const void *x, const void *v,
                  const float *rot, int n_new, float *O, float *lse, int32_t *count, cudaStream_t s) {
    LdArgs a = ld_args(p, st);
    a.X = static_cast<const __nv_bfloat16 *>(x);
    a.Vn = static_cast<const __nv_bfloat16 *>(v);
    a.rot = rot;
    a.n_new = n_new;
    a.O = O;
    a.lse = lse;
    a.count = count;
    ProfScope _ps(K_LSH_DECODE, s);
    lsd_hash_kernel<<<dim3(p->n_seq * p->n_heads, ceil_div(n_new * p->n_rounds, 8)), 256, 0, s>>>(a);
    lsd_store_kv_kernel<<<dim3(ceil_div(n_new * p->n_heads, 8), p->n_seq), 256, 0, s>>>(a);
    lsd_append_kernel<<<ceil_div(p->n_seq * p->n_heads * p->n_rounds, 8), 256, 0, s>>>(a);
    if (O) lsd_attend_kernel<<<p->n_seq * p->n_heads, kLdAttThreads, 0, s>>>(a);
    lsd_advance_kernel<<<ceil_div(p->n_seq, 128), 128, 0, s>>>(st->seq_len, p->n_seq, n_new, p->max_len);
    _ps.more(O ? 4 : 3);                          // hash, store, append, (attend,) advance
    CRS_CHECK_LAUNCH();
    return CRS_OK;
}

}  // namespace crs

using namespace crs;

extern "C" int crs_lsh_decode_prefill(const crs_lsh_decode_params *p, const crs_lsh_decode_state *st,
                                      const void *x, const void *v, const float *rot, int n_tokens, void *stream) {
    int e = ld_validate(p);
    if (e) return e;
    if (!ld_state_ok(st) || !x || !v || !rot || n_tokens < 0) return CRS_ERR_INVALID_ARG;
    if ((long long)n_tokens * p->n_rounds > 8LL * 65535) return CRS_ERR_UNSUPPORTED;   // append in pieces
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(v)) & 3) return CRS_ERR_INVALID_ARG;
    if (n_tokens == 0) return CRS_OK;
    return ld_run(p, st, x, v, rot, n_tokens, nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

extern "C" int crs_lsh_decode_step(const crs_lsh_decode_params *p, const crs_lsh_decode_state *st, const void *x,
                                   const void *v, const float *rot, float *O, float *lse, int32_t *count,
                                   void *stream) {
    int e = ld_validate(p);
    if (e) return e;
    if (!ld_state_ok(st) || !x || !v || !rot || !O || !lse) return CRS_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(v)) & 3) return CRS_ERR_INVALID_ARG;
    return ld_run(p, st, x, v, rot, 1, O, lse, count, static_cast<cudaStream_t>(stream));
}
