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
//   lsd_attend_kernel      one CTA per (row, head): each lane takes a candidate
//                          (online softmax in registers), lanes and warps merged
//                          in shared memory
//   lsd_advance_kernel     seq_len += tokens appended
#include "common.cuh"

namespace crs {

constexpr int kLdD = 64;                  // head dim
constexpr int kLdMaxRounds = 8;
constexpr int kLdAttWarps = 4;

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
    for (int k = lane; k < half; k += 32) {
        float u = 0.0f;
        for (int i = 0; i < kLdD; ++i) u = fmaf(__bfloat162float(x[i]), R[(size_t)i * half + k], u);
        if (u > best || (u == best && k < bi)) { best = u; bi = k; }
        if (-u > best || (-u == best && k + half < bi)) { best = -u; bi = k + half; }
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
// Candidates are taken round by round; entry j of round r is skipped when j == t
// (no_self) or when j shares an earlier round's bucket with t (already met).
// Lane = candidate: dot with q (registers), online softmax and a 64-wide value
// accumulator per lane; lanes then warps are merged through shared memory.
__global__ void __launch_bounds__(kLdAttWarps * 32) lsd_attend_kernel(LdArgs a) {
    __shared__ float sq[kLdD];
    __shared__ float sm[kLdAttWarps * 32], sl[kLdAttWarps * 32];
    __shared__ float so[kLdAttWarps][kLdD];
    __shared__ int scnt[kLdAttWarps];
    const int sh = blockIdx.x, s = sh / a.H, h = sh - s * a.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = a.st.seq_len[s];                           // the newest token
    const int nt = kLdAttWarps * 32;
    if (t >= a.max_len) {                                    // no room: flagged by the append
        if (tid < kLdD) a.O[((size_t)s * a.H + h) * kLdD + tid] = 0.0f;
        if (tid == 0) {
            a.lse[(size_t)s * a.H + h] = -INFINITY;
            if (a.count) a.count[(size_t)s * a.H + h] = 0;
        }
        return;
    }
    const size_t q_off = ((size_t)s * a.n_new * a.H + h) * kLdD;   // token 0 of the step
    if (tid < kLdD) sq[tid] = a.scale * __bfloat162float(a.X[q_off + tid]);
    __syncthreads();
    uint8_t tb[kLdMaxRounds];
    const uint8_t *bk = a.st.bucket + ((size_t)s * a.H + h) * a.R * a.max_len;
#pragma unroll
    for (int r = 0; r < kLdMaxRounds; ++r) tb[r] = r < a.R ? bk[(size_t)r * a.max_len + t] : 0;
    float m = -INFINITY, l = 0.0f, o[kLdD];
#pragma unroll
    for (int c = 0; c < kLdD; ++c) o[c] = 0.0f;
    int cnt = 0;
    for (int r = 0; r < a.R; ++r) {
        const size_t lid = ld_list_id(a, s, h, r, tb[r]);
        const int len = min(a.st.list_len[lid], a.list_pages * a.Lp);
        for (int e = tid; e < len; e += nt) {
            const int pg = a.st.list_table[lid * a.list_pages + e / a.Lp];
            if (pg < 0) continue;
            const int j = a.st.list_pool[(size_t)pg * a.Lp + e % a.Lp];
            if (j > t || (a.no_self && j == t)) continue;
            bool met = false;
            for (int r2 = 0; r2 < r; ++r2) met |= bk[(size_t)r2 * a.max_len + j] == tb[r2];
            if (met) continue;
            const int page = a.st.block_table[(size_t)s * a.max_pages + j / a.P];
            const size_t row = (((size_t)page * a.P + j % a.P) * a.H + h) * kLdD;
            const uint4 *kr = reinterpret_cast<const uint4 *>(a.st.K + row);
            float dot = 0.0f;
#pragma unroll
            for (int c = 0; c < kLdD / 8; ++c) {
                const uint4 raw = __ldg(kr + c);
                const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 kv = __bfloat1622float2(p2[u]);
                    dot = fmaf(sq[c * 8 + 2 * u], kv.x, fmaf(sq[c * 8 + 2 * u + 1], kv.y, dot));
                }
            }
            const float mn = fmaxf(m, dot);
            const float corr = __expf(m - mn), p = __expf(dot - mn);
            l = l * corr + p;
            const uint4 *vr = reinterpret_cast<const uint4 *>(a.st.V + row);
#pragma unroll
            for (int c = 0; c < kLdD / 8; ++c) {
                const uint4 raw = __ldg(vr + c);
                const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 vv = __bfloat1622float2(p2[u]);
                    o[c * 8 + 2 * u] = fmaf(p, vv.x, o[c * 8 + 2 * u] * corr);
                    o[c * 8 + 2 * u + 1] = fmaf(p, vv.y, o[c * 8 + 2 * u + 1] * corr);
                }
            }
            m = mn;
            ++cnt;
        }
    }
    // merge: the CTA maximum, then each lane's rescaled (l, o) summed per warp, then per CTA
    sm[tid] = m;
    __syncthreads();
    float M = -INFINITY;
    for (int i = 0; i < nt; ++i) M = fmaxf(M, sm[i]);
    const float f = m == -INFINITY ? 0.0f : __expf(m - M);
    float lw = warp_sum(l * f);
    const int cw = warp_sum_int(cnt);
#pragma unroll
    for (int c = 0; c < kLdD; ++c) {
        const float v = warp_sum(o[c] * f);
        if (lane == 0) so[warp][c] = v;
    }
    if (lane == 0) {
        sl[warp] = lw;
        scnt[warp] = cw;
    }
    __syncthreads();
    if (tid < kLdD) {
        float L = 0.0f, acc = 0.0f;
        int C = 0;
        for (int w = 0; w < kLdAttWarps; ++w) {
            L += sl[w];
            acc += so[w][tid];
            C += scnt[w];
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
    if (O) lsd_attend_kernel<<<p->n_seq * p->n_heads, kLdAttWarps * 32, 0, s>>>(a);
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
