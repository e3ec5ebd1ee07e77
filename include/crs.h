/*
 * crs.h -- C ABI of libcrs, content-routed sparse attention on NVIDIA B200 (sm_100a).
 *
 * A selector computes, for every query, a candidate set of key positions; exact
 * softmax attention then runs over the gathered K/V only.  Three selectors:
 *   - Reformer-style LSH routing (crs_lsh_route + crs_lsh_attn),
 *   - a DSA-style lightning indexer with token top-k (crs_indexer_topk),
 *   - a COBS-style block-mass selector (crs_block_describe + crs_block_select),
 * and one attention kernel over explicit index lists (crs_sparse_attn).
 *
 * Pages cited:
 *   [P1] PaperTrace 2.1.1 "哈希与聚类: 用内容建立稀疏注意力邻域"
 *   [P2] PaperTrace 2.2 "细粒度索引: 用轻量 selector 召回关键 token"
 *   [P4] Understanding LLMs ch. 26 "高效、稀疏与替代架构地图"
 *   [P5] "COBS 阅读笔记: 块稀疏注意力的选择器到底漏掉了什么"
 *
 * Conventions (all entry points):
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; libcrs
 *     never allocates, frees or keeps a pointer after the call returns.
 *     Tensors are dense, row-major (C order), in the layouts stated below.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are asynchronous on that stream.
 *   - Scratch memory comes from the caller: `ws`/`ws_bytes`, sized by the
 *     matching *_workspace_size() call.  A short workspace returns
 *     CRS_ERR_WORKSPACE with nothing launched.
 *   - Host-side validation errors return immediately with nothing launched.
 *     A failed launch returns CRS_ERR_CUDA.
 *   - Problems a kernel detects in the data (a non-finite indexer score, an
 *     index out of range, a bounded wait that ran out) are OR-ed into a
 *     per-device error word; crs_get_device_error() reads and clears it.
 *   - Index lists hold int32 positions within their sequence, ascending;
 *     -1 marks an unused slot.
 *   - bf16 means IEEE bfloat16 stored in 16 bits; f32 means IEEE binary32.
 */
#ifndef CRS_H
#define CRS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status -- */
typedef enum {
    CRS_OK = 0,
    CRS_ERR_INVALID_ARG = 1,  /* a size, pointer or parameter is out of range     */
    CRS_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels implement   */
    CRS_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed          */
    CRS_ERR_NONFINITE = 4,    /* (device word bit) NaN/Inf met where not allowed */
    CRS_ERR_TIMEOUT = 5,      /* (device word bit) a bounded wait ran out        */
    CRS_ERR_WORKSPACE = 6,    /* ws is NULL or shorter than required             */
    CRS_ERR_INDEX = 7         /* (device word bit) an index list entry is out of range */
} crs_status;

typedef enum { CRS_F32 = 0, CRS_BF16 = 1 } crs_dtype;

/* Bits of the device error word. */
#define CRS_DEVERR_NONFINITE 0x1u
#define CRS_DEVERR_TIMEOUT   0x2u
#define CRS_DEVERR_INDEX     0x4u
#define CRS_DEVERR_CAPACITY  0x8u   /* a bounded structure was full: an entry was dropped */

/* Human-readable name of a crs_status value (static string, never NULL). */
const char *crs_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int crs_version(void);

/* Synchronizes `stream`, then reads and clears the error word of the current
 * device.  *flags receives the CRS_DEVERR_* bits set since the last call
 * (0 = none).  Returns CRS_ERR_CUDA if the synchronization fails. */
int crs_get_device_error(void *stream, uint32_t *flags);

/* Diagnostic record of the first failure a kernel reported about itself
 * since the last call (a bounded wait that gave up, an operand check):
 * out[0] = kernel id + 1 (0 = none), out[1] = site within the kernel,
 * out[2..4] = the CTA's blockIdx, out[5..15] = kernel-specific values.
 * Synchronizes `stream`, copies min(n, 16) words and clears the record. */
int crs_get_device_diag(void *stream, uint32_t *out, int n);

/* Test switch for the failure path of the bounded waits (the pages have no
 * counterpart: it exists to exercise this library's own fault handling).  While
 * on (on != 0, current device), the first mbarrier wait of the tensor-core LSH
 * kernels (the hash of crs_lsh_route and the chunk attention of crs_lsh_attn)
 * gives up at once, as a wait that ran out would: the kernel sets
 * CRS_DEVERR_TIMEOUT, records (kernel id, site 1) in the diagnostic record,
 * waits for the tensor-core work it issued, frees its tensor memory and
 * returns without writing its outputs (bucket ids, attention sums).  Turn it
 * off (on = 0) before using the results of later calls.  Returns CRS_ERR_CUDA
 * if the device global cannot be written. */
int crs_debug_force_wait_timeout(int on);

/* Measurement aid (no counterpart in the pages): the L2 read ceiling of row
 * gathers, against which the gather attention over an L2-resident K/V set is
 * reported.  Reads the `n_idx` rows idx[0 .. n_idx) (each 0 <= idx[i] < rows)
 * of `table` (device, rows x 512 bytes, 16-byte aligned), one 512-byte row per
 * warp load instruction (32 lanes x 16 bytes, L1 bypassed), from 8 CTAs of 512
 * threads per SM; a warp writes the XOR of what it read to `sink` (device,
 * 16 bytes) only when that XOR equals a fixed constant, which keeps the loads.  The caller times the launch on `stream`
 * (a table of 16 MiB stays in L2).  CRS_ERR_INVALID_ARG for null pointers,
 * rows < 1 or n_idx < 1; index values are the caller's to keep in range. */
int crs_probe_l2_gather(const void *table, int64_t rows, const int32_t *idx, int64_t n_idx, void *sink,
                        void *stream);

/* Launch tracing.  [P1] "一个可复现的评测矩阵" and [P2] §1.1 "性能轴" ask for the
 * time of every stage (routing, sort, selection, gather, attention) reported
 * separately; this is how the library provides it.  Every kernel
 * launch is counted.  While enabled, each launch is also bracketed by two
 * CUDA events recorded on the launch's own stream.
 * crs_profile_collect() synchronizes on those events, writes one record per
 * kernel that launched since the previous collect (up to max_out records;
 * *n_out receives how many kernels there were) and resets the counters. */
typedef struct {
    char name[32];           /* kernel family, e.g. "lsh_chunk_attn"            */
    int64_t launches;        /* launches since the previous collect             */
    int64_t timed_launches;  /* of those, launches made while tracing was on    */
    double total_ms;         /* summed device time of the timed launches        */
} crs_kernel_stat;

int crs_profile_set(int enabled);
int crs_profile_collect(crs_kernel_stat *out, int max_out, int *n_out);

/* ====================================================================== *
 * LSH routing.  [P1] §2.1 Eq.(4): per head h and round r, u = x R_{h,r} with
 * R_{h,r} in R^{d x b/2}; bucket = argmax_j [u ; -u]_j (0-based, lowest
 * index on ties).  [P1] §2.1-2.2: tokens are stably sorted on the bucket id
 * (sort key = bucket * n + position); perm maps a sorted slot to its
 * original position, inv_perm maps a position to its slot.
 * The projection is evaluated in fp32 as one fused multiply-add per term in
 * increasing index order starting from 0, so the bucket ids are reproducible
 * bit for bit.
 * ====================================================================== */
typedef struct {
    int B;          /* batch                                                    */
    int H;          /* heads                                                    */
    int n;          /* tokens per sequence, >= 1                                */
    int d;          /* head dim, multiple of 8, <= 128                          */
    int n_buckets;  /* b, even, 2..1024                                         */
    int n_rounds;   /* independent hash rounds, 1..8                            */
    int chunk;      /* m, slots per chunk (used by crs_lsh_attn), 1..128       */
    int dtype;      /* crs_dtype of X / QK / V / O                              */
} crs_lsh_params;

/* X: [B,H,n,d] (dtype); R: [H,n_rounds,d,n_buckets/2] f32.
 * Outputs (int32, [B,H,n_rounds,n]): bucket, perm (slot -> position),
 * inv_perm (position -> slot).  Needs no workspace (ws may be NULL). */
size_t crs_lsh_route_workspace_size(const crs_lsh_params *p);
int crs_lsh_route(const crs_lsh_params *p, const void *X, const float *R, int32_t *bucket,
                  int32_t *perm, int32_t *inv_perm, void *ws, size_t ws_bytes, void *stream);

/* ====================================================================== *
 * LSH attention.  [P1] §2.2: each round's sorted array is cut into chunks of
 * m slots; a query chunk attends to itself and the previous chunk (chunk 0
 * has none).  A pair (i, j) is an edge of round r iff bucket_r(j) ==
 * bucket_r(i), j <= i when causal, j != i when no_self, j < valid_len[b]
 * ([P1] §1.1 Eq.(2); causality on ORIGINAL positions, [P1] §"8.2").  Shared
 * QK ([P1] §2): keys are q_j/|q_j| when key_norm != 0 (a zero vector stays
 * zero), logits scale * q_i . k_j.  Rounds are merged by their log-sum-exp
 * weights with each pair counted only in the first round it appears in
 * ([P1] "重复候选和归一化"), which equals one softmax over the union of the
 * rounds' candidates.  A query with no edge, and every padded query
 * (i >= valid_len[b]), gets O = 0 and lse = -inf.
 * ====================================================================== */
typedef struct {
    crs_lsh_params p;
    int causal;     /* 1: j <= i                                              */
    int no_self;    /* 1: j != i                                              */
    int key_norm;   /* 1: k_j = q_j / |q_j| (Reformer shared-QK), 0: k_j = q_j */
    float scale;    /* logit scale, typically 1/sqrt(d)                       */
} crs_lsh_attn_params;

/* QK, V: [B,H,n,d] (p.dtype); bucket/perm/inv_perm: [B,H,n_rounds,n] from
 * crs_lsh_route; valid_len: [B] int32 (NULL = n for all).
 * O: [B,H,n,d] f32, written in original token order (f32 whatever p.dtype:
 * the 2e-3 output tolerance for bf16 inputs is below bf16's unit roundoff
 * 2^-8, so the result keeps the fp32 accumulator's precision);
 * lse: [B,H,n] f32 natural-log normaliser of the merged softmax, or NULL.
 * O must start on a 16-byte boundary (rows are written as 16-byte vectors;
 * else CRS_ERR_INVALID_ARG).  The tensor-core kernels also read QK and V rows
 * as 16-byte pieces: with either not 16-byte aligned the call takes the
 * CUDA-core kernel instead. */
size_t crs_lsh_attn_workspace_size(const crs_lsh_attn_params *p);
int crs_lsh_attn(const crs_lsh_attn_params *p, const void *QK, const void *V,
                 const int32_t *bucket, const int32_t *perm, const int32_t *inv_perm,
                 const int32_t *valid_len, void *O, float *lse, void *ws, size_t ws_bytes,
                 void *stream);

/* The candidate sets U(i) of crs_lsh_attn as an explicit CSR matrix, an
 * inspection export for small inputs ([P1] §4: the index tensors row_ptr /
 * col_idx, perm, inverse_perm; §2.1-2.2 and §1.1 Eq.(2) define the set: the
 * keys j of i's chunk and the chunk before it, in some round, with i's bucket,
 * j <= i when causal, j != i when no_self, j < valid_len[b]; each key once).
 * A padded query (i >= valid_len[b]) gets its set like any other row
 * (crs_lsh_attn gives such a row O = 0).  Rows are ordered (b, h, i).
 *   row_ptr: [B*H*n + 1] int64; col_idx: [row_ptr[B*H*n]] int32, each row's
 *   keys ascending.
 * Two calls: with col_idx == NULL the call writes row_ptr (counts, then their
 * prefix sum; read row_ptr[B*H*n] to size col_idx); with col_idx it fills the
 * rows, reading row_ptr as the first call left it (same inputs).  Only the
 * routing fields of p (B, H, n, n_rounds, chunk), causal and no_self are used.
 * n <= 65536 and B*H*n <= 2^22 (else CRS_ERR_UNSUPPORTED); a permutation
 * entry outside [0, n) sets CRS_DEVERR_INDEX and is skipped. */
int crs_lsh_candidates_csr(const crs_lsh_attn_params *p, const int32_t *bucket, const int32_t *perm,
                           const int32_t *inv_perm, const int32_t *valid_len, int64_t *row_ptr,
                           int32_t *col_idx, void *stream);

/* ====================================================================== *
 * LSH attention in decode.  [P1] §5.2 "Prefill、Decode 与 KV 状态": the hash is
 * fixed (R as crs_lsh_route); each new token's bucket ids (one per round, O(d R))
 * are appended to that (row, head, round, bucket)'s list of logical positions;
 * K/V stay paged by time behind a block table ([P2] §2.1 "主 KV gather 的物理代价").
 * The newest token t of a row attends to every token j <= t sharing a bucket
 * with it in some round, each once, without t itself when no_self; keys are
 * the shared-QK vectors normalised when key_norm (stored normalised in bf16),
 * logits scale * q . k, fp32 softmax; an empty set gives O = 0, lse = -inf.
 * State (caller-owned, zero-initialised except k/v pools and block_table):
 *   k_pool, v_pool [n_pages, page_size, n_heads, d] bf16 (16-byte aligned);
 *   block_table [n_seq, max_pages] int32 (logical page -> physical page);
 *   bucket_store [n_seq, n_heads, n_rounds, max_len] uint8;
 *   list_table [n_seq, n_heads, n_rounds, n_buckets, list_pages] int32,
 *   list_len [n_seq, n_heads, n_rounds, n_buckets] int32,
 *   list_pool [n_list_pages, list_page] int32, alloc [1] int32 (pages used);
 *   seq_len [n_seq] int32 (tokens already in each row).
 * A list holds at most list_pages * list_page entries; a full list, an
 * exhausted list pool, or a row beyond max_len / max_pages * page_size sets
 * CRS_DEVERR_CAPACITY and drops the entry.  d = 64, n_buckets even <= 256,
 * n_rounds <= 8 (else CRS_ERR_UNSUPPORTED).
 * crs_lsh_decode_prefill appends n_tokens tokens per row (x, v [n_seq,
 * n_tokens, n_heads, d] bf16) in position order; crs_lsh_decode_step appends
 * one token per row (x, v [n_seq, 1, n_heads, d]) and attends with it:
 * O [n_seq, n_heads, d] f32, lse [n_seq, n_heads] f32 (natural log), count
 * [n_seq, n_heads] int32 (candidates, may be NULL).  Both advance seq_len.
 * ====================================================================== */
typedef struct {
    int n_seq, n_heads, d, n_buckets, n_rounds;
    int page_size;     /* tokens per KV page                                   */
    int max_pages;     /* block_table row length                               */
    int list_page;     /* positions per bucket-list page                       */
    int list_pages;    /* page-table length of one bucket list                 */
    int n_list_pages;  /* pages in list_pool                                   */
    int max_len;       /* tokens per row at most (bucket_store row length)     */
    int no_self, key_norm;
    float scale;
} crs_lsh_decode_params;

typedef struct {
    void *k_pool, *v_pool;
    const int32_t *block_table;
    uint8_t *bucket_store;
    int32_t *list_table, *list_len, *list_pool, *alloc, *seq_len;
} crs_lsh_decode_state;

int crs_lsh_decode_prefill(const crs_lsh_decode_params *p, const crs_lsh_decode_state *st, const void *x,
                           const void *v, const float *rot, int n_tokens, void *stream);
int crs_lsh_decode_step(const crs_lsh_decode_params *p, const crs_lsh_decode_state *st, const void *x,
                        const void *v, const float *rot, float *O, float *lse, int32_t *count, void *stream);

/* ====================================================================== *
 * Routing (k-means) attention with quota execution.  [P1] §3.1: frozen
 * centres M [H, C, d] f32; routing scores S_Q = Q M^T, S_K = K M^T, each an
 * integer decision taken in fp32 as one FMA per term in increasing index order
 * from 0; centre c keeps its m best queries J_c^Q and m best keys J_c^K
 * (score desc, index asc), returned ascending in JQ, JK [B, H, C, m] (-1 past
 * n).  Query i attends to the union of J_c^K over the centres with i in J_c^Q,
 * each key once, j <= i when causal, j != i when no_self; logits scale * q.k;
 * fp32 softmax; an empty set gives O = 0, lse = -inf.
 * Q, K, V: [B, H, n, d] bf16 (16-byte aligned); O [B, H, n, d] f32; lse [B, H, n]
 * f32 (natural log); count [B, H, n] int32 (keys attended, may be NULL).
 * d = 64, C <= 256, m <= 256, n <= 16384 (else CRS_ERR_UNSUPPORTED).
 * ====================================================================== */
typedef struct {
    int B, H, n, d;
    int C;            /* centres per head                                     */
    int m;            /* quota: queries and keys kept per centre              */
    int causal, no_self;
    float scale;
} crs_route_params;

size_t crs_route_attn_workspace_size(const crs_route_params *p);
int crs_route_attn(const crs_route_params *p, const void *Q, const void *K, const void *V, const float *M,
                   int32_t *JQ, int32_t *JK, float *O, float *lse, int32_t *count, void *ws, size_t ws_bytes,
                   void *stream);

/* ====================================================================== *
 * Lightning indexer + token top-k.  [P2] §1.1 / §2.1 Eq.(2)-(4):
 *   r_{t,s} = sum_h w_{t,h} ReLU(q_{t,h} . k_s)   (no extra scale)
 * S_t = the topk positions with the largest r_{t,s}, ties to the smaller
 * position ([P2] §3.1 "多卡一致性"), returned ascending; a row with fewer
 * than topk visible keys returns all of them and -1 in the other slots
 * ([P2] §2.1).  The score matrix is never stored whole ([P2] §2.1).
 * Modes:
 *   CRS_IDX_PREFILL: one causal sequence of n_rows tokens; row t sees keys
 *                    0..t; k_offsets is ignored.
 *   CRS_IDX_DECODE:  n_rows sequences, one query each; row s sees the keys
 *                    k_idx[k_offsets[s] .. k_offsets[s+1]) (int64 offsets,
 *                    [n_rows+1]); positions are relative to k_offsets[s].
 * A NaN score sets CRS_DEVERR_NONFINITE and ranks below every number.
 * ====================================================================== */
enum { CRS_IDX_PREFILL = 0, CRS_IDX_DECODE = 1 };

typedef struct {
    int mode;         /* CRS_IDX_PREFILL or CRS_IDX_DECODE                      */
    int n_rows;       /* queries                                                */
    int n_idx_heads;  /* index heads, 1..8                                      */
    int d_idx;        /* index head dim, 64                                     */
    int topk;         /* 1..4096                                                */
    int max_keys;     /* DECODE: an upper bound of the longest row (sizes ws)   */
} crs_indexer_params;

/* q_idx: [n_rows, n_idx_heads, d_idx] bf16; w: [n_rows, n_idx_heads] f32;
 * k_idx: [keys, d_idx] bf16; out_idx: [n_rows, topk] int32; out_count:
 * [n_rows] int32 (number of valid entries). */
size_t crs_indexer_topk_workspace_size(const crs_indexer_params *p);
int crs_indexer_topk(const crs_indexer_params *p, const void *q_idx, const float *w,
                     const void *k_idx, const int64_t *k_offsets, int32_t *out_idx,
                     int32_t *out_count, void *ws, size_t ws_bytes, void *stream);

/* ====================================================================== *
 * Hierarchical indexer (HISA) for decode rows.  [P2] "索引器的三种降本方向",
 * §2.2 Eq.(7): each complete block of `blk` keys of a row has a representative
 * rep_j (the mean of its index keys, f32, from crs_hisa_describe, once per
 * filled block); the row scores c_j = sum_h w_h ReLU(q_h . rep_j), keeps the
 * top_blocks blocks by (c desc, block asc), and runs the token indexer of
 * crs_indexer_topk (same score, ties, ascending -1-padded output) on the kept
 * blocks' keys plus the open trailing block only.  out_blocks (optional,
 * [n_rows, top_blocks], ascending, -1 padded) returns the kept blocks: the
 * pages keep each level's candidates to locate a miss.
 * k_offsets: [n_rows + 1] int64, row s owns keys k_offsets[s]..k_offsets[s+1]
 * (at most max_keys, else CRS_DEVERR_INDEX and an empty row); blk_offsets:
 * [n_rows + 1] int64, blk_offsets[s+1] - blk_offsets[s] = floor(keys_s / blk);
 * rep: [blk_offsets[n_rows], 64] f32.  d_idx = 64, n_idx_heads <= 8,
 * blk <= 256, top_blocks * blk + blk <= 16384, max_keys / blk <= 8192
 * (else CRS_ERR_UNSUPPORTED); k_idx 16-byte aligned.
 * ====================================================================== */
typedef struct {
    int n_rows;       /* decode rows, one query each                            */
    int n_idx_heads;  /* index heads, 1..8                                      */
    int d_idx;        /* 64                                                     */
    int topk;         /* tokens returned, 1..4096                               */
    int blk;          /* keys per block                                         */
    int top_blocks;   /* blocks kept by the coarse level                        */
    int max_keys;     /* an upper bound of the longest row                      */
} crs_hisa_params;

int crs_hisa_describe(const crs_hisa_params *p, const void *k_idx, const int64_t *k_offsets,
                      const int64_t *blk_offsets, float *rep, void *stream);
size_t crs_hisa_topk_workspace_size(const crs_hisa_params *p);
int crs_hisa_topk(const crs_hisa_params *p, const void *q_idx, const float *w, const void *k_idx,
                  const int64_t *k_offsets, const float *rep, const int64_t *blk_offsets,
                  int32_t *out_blocks, int32_t *out_idx, int32_t *out_count, void *ws, size_t ws_bytes,
                  void *stream);

/* HISA prefill (causal) form.  [P2] "索引器的三种降本方向", §2.1 Eq.(4) and §2.2
 * Eq.(7): the n queries of one sequence; query t sees keys 0..t as the flat
 * prefill indexer's rows do; its complete blocks are the sequence's blocks
 * j < (t + 1) / blk, whose representatives rep_j do not depend on the query
 * (crs_hisa_describe with n_rows = 1, k_offsets = {0, n}, blk_offsets = {0, n / blk});
 * then the decode row rule with ctx = t + 1: the top_blocks blocks by
 * (c desc, block asc) (all of them when there are at most top_blocks), and the
 * token top-k (same score, ties, ascending, -1-padded output) over the kept
 * blocks' keys and the open block (keys (t + 1) / blk * blk .. t).
 * p: n_rows = n (queries = keys), n_idx_heads = 4, d_idx = 64, blk = 64,
 * topk <= 2048, top_blocks * blk >= topk, n / blk <= 1024, n <= 2^19 (else
 * CRS_ERR_UNSUPPORTED); max_keys is not used.
 * q_idx [n, 4, 64] bf16, w [n, 4] f32, k_idx [n, 64] bf16 (16-byte aligned);
 * rep [n / blk, 64] f32; out_blocks (optional) [n, top_blocks] int32; out_idx
 * [n, topk] int32; out_count [n] int32.  The token level runs on the tensor
 * cores (one 64-key block = one key tile; a row's unkept complete blocks are
 * masked), with the exact selection of crs_indexer_topk. */
size_t crs_hisa_topk_prefill_workspace_size(const crs_hisa_params *p);
int crs_hisa_topk_prefill(const crs_hisa_params *p, const void *q_idx, const float *w, const void *k_idx,
                          const float *rep, int32_t *out_blocks, int32_t *out_idx, int32_t *out_count,
                          void *ws, size_t ws_bytes, void *stream);

/* ====================================================================== *
 * Block descriptors.  [P5] Eq.(11), (16), (20) and Algorithm 2: for each
 * complete block of L consecutive keys of one (sequence, KV head):
 *   mu = mean key; Kt = K - mu; G = Kt Kt^T / L (L x L);
 *   (lambda_i, w_i) = the `rank` largest eigenpairs of G;
 *   xi_i = Kt^T w_i / sqrt(L)   (= sqrt(lambda_i) u_i, sign arbitrary).
 * The descriptor depends on the block alone and is computed once, when the
 * block is full ([P5] "可缓存性约束").  Blocks [blk_begin, blk_end) are
 * (re)computed; others are left untouched.
 * ====================================================================== */
typedef struct {
    int n_seq;      /* sequences                                             */
    int n_kv;       /* KV heads                                              */
    int T;          /* tokens per sequence in the cache                      */
    int D;          /* head dim, 128                                         */
    int L;          /* block size, 32                                        */
    int rank;       /* kept eigen-directions, 1..8                           */
    int blk_begin;  /* first block to compute                                */
    int blk_end;    /* one past the last block to compute, <= T / L          */
} crs_block_params;

/* K: [n_seq, T, n_kv, D] bf16.  mu: [n_seq, n_kv, T/L, D] f32;
 * xi: [n_seq, n_kv, T/L, rank, D] f32. */
int crs_block_describe(const crs_block_params *p, const void *K, float *mu, float *xi,
                       void *stream);

/* ====================================================================== *
 * Block selection.  [P5] Eq.(14)/(19): s_{g,b} = qt . mu_b + 1/2 sum_i (xi_i . qt)^2
 * with qt = scale * q_g (the ln L constant cancels); [P5] Eq.(15)/(6): KV head
 * h scores block b by sum over its query-head group g of softmax_b(s_{g,.});
 * the top_blocks complete blocks by (score desc, block asc) are kept; the
 * token list is their positions united with the window [T-window, T),
 * without duplicates, ascending.  Query heads [h*G, (h+1)*G) share KV head h
 * ([P4] §26.2).
 * ====================================================================== */
typedef struct {
    crs_block_params b;  /* n_seq, n_kv, T, D, L, rank (blk_* ignored)       */
    int n_q;             /* query heads, multiple of n_kv, G = n_q/n_kv <= 16 */
    int top_blocks;      /* kept blocks, 1..T/L                              */
    int window;          /* trailing window, 0..T                            */
    float scale;         /* typically 1/sqrt(D)                              */
} crs_block_sel_params;

/* Q: [n_seq, n_q, D] bf16; mu, xi from crs_block_describe.
 * tok_idx: [n_seq, n_kv, top_blocks*L + window] int32; tok_count: [n_seq, n_kv].
 * rank 0 is the mean-pool selector of [P5] Table 1 (s_{g,b} = qt . mu_b, the
 * first-order term alone): xi may then be NULL; Q 8-byte and mu 16-byte aligned. */
size_t crs_block_select_workspace_size(const crs_block_sel_params *p);
int crs_block_select(const crs_block_sel_params *p, const void *Q, const float *mu,
                     const float *xi, int32_t *tok_idx, int32_t *tok_count, void *ws,
                     size_t ws_bytes, void *stream);

/* Allocation-free variant of crs_block_select.  The pages have no counterpart
 * of this call; it exists for callers that cannot allocate device memory when
 * they call the library (an engine whose pool owns all device memory and
 * refuses allocations after start-up, a plugin host that passes only input
 * and output buffers, a latency-bound loop that must not pay for cudaMalloc /
 * cudaFree or their implicit synchronization).  Same parameters, inputs,
 * outputs and result as crs_block_select, but no workspace argument: the
 * scratch is a static device array of CRS_NOALLOC_SCRATCH_BYTES inside the
 * library, which every GPU that loads libcrs holds until the process exits.
 *   - Limit: crs_block_select_workspace_size(p) (n_seq * n_q * (T/L) * 4
 *     bytes) must not exceed CRS_NOALLOC_SCRATCH_BYTES, i.e. at most 4,194,304
 *     (sequence, query head, block) scores; larger problems return
 *     CRS_ERR_WORKSPACE with nothing launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it with the
 *     device's current context; a call under another context (after a
 *     cudaDeviceReset, say) looks it up again.  Make the first call on a
 *     device, and the first call after a reset, before any stream capture.
 *   - Every call, on any stream, shares the one array and it keeps the last
 *     call's contents: calls that overlap on the GPU (concurrent streams)
 *     race on it and must be serialized by the caller.  Nothing needs
 *     clearing between calls: the kernels write every scratch entry they read.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine. */
#define CRS_NOALLOC_SCRATCH_BYTES (16u << 20)
int crs_block_select_noalloc(const crs_block_sel_params *p, const void *Q, const float *mu,
                             const float *xi, int32_t *tok_idx, int32_t *tok_count, void *stream);

/* Deployed descriptor compression.  [P5] §5.5 ("量化：对存储的特征向量做
 * FP4") and Algorithm 2 steps 7-8: the block mean is stored in bf16 and each
 * scaled eigenvector in E2M1 FP4 with one fp32 scale per vector.
 *   mu, xi:   from crs_block_describe (fp32, [n_seq, n_kv, T/L, D] and
 *             [n_seq, n_kv, T/L, rank, D]).
 *   mu16:     [n_seq, n_kv, T/L, D] bf16 (round to nearest even).
 *   xi4:      [n_seq, n_kv, T/L, rank, D/2] bytes: two 4-bit codes per byte,
 *             the even element in the low nibble; code bit 3 = sign, bits 0-2
 *             index {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *   xi_scale: [n_seq, n_kv, T/L, rank] fp32, = max |xi| / 6 of the vector; an
 *             element is ~ sign * value(code) * scale.
 * Rounding (the page leaves it open): the nearest value of xi / scale, a tie
 * going to the zero-mantissa code, decided in fp32.  At r = 4, D = 128 the
 * factors take 272 bytes per block instead of 1024 in bf16 ([P5] §5.5); with
 * the mean, 528 bytes instead of 2560 in fp32.  All pointers 16-byte aligned
 * (else CRS_ERR_INVALID_ARG); blk_begin / blk_end are ignored. */
int crs_block_quantize(const crs_block_params *p, const float *mu, const float *xi, void *mu16,
                       uint8_t *xi4, float *xi_scale, void *stream);

/* crs_block_select on compressed descriptors (same selection rule, outputs and
 * workspace as crs_block_select; the score uses the dequantised mean and
 * eigenvectors).  Supported: up to 16 query heads per KV head (a divisor of
 * 16, as for crs_block_select), rank 1..4 (else CRS_ERR_UNSUPPORTED); Q,
 * mu16 and xi4 16-byte aligned (else CRS_ERR_INVALID_ARG).  The products
 * Q . mu and Q . code are formed on the tensor cores from the bf16 query and
 * the codes widened to bf16 (both exact), accumulated in fp32; the softmax
 * scale and the per-vector FP4 scale are applied afterwards. */
int crs_block_select_fp4(const crs_block_sel_params *p, const void *Q, const void *mu16,
                         const uint8_t *xi4, const float *xi_scale, int32_t *tok_idx,
                         int32_t *tok_count, void *ws, size_t ws_bytes, void *stream);

/* ====================================================================== *
 * Query-subspace descriptors ([P5] "子空间方法", Eq.(17)-(18)).  U: [D, sd] f32
 * (row-major), orthonormal columns spanning the query subspace (the top sd
 * eigenvectors of the queries' second moment, computed offline; an input).
 * crs_block_describe_ss: mu as crs_block_describe; xi_ss [n_seq, n_kv, T/L,
 * rank, sd] f32 = the rank scaled eigenvectors of B_b = U^T Sigma_b U, formed
 * by the Gram route on the projected centred keys Y = Kt U (1 <= sd <= D).
 * crs_block_select_ss: the crs_block_select rule with the quadratic term
 * (xi_i . U^T qt)^2 ([P5] Eq.(18)); workspace from
 * crs_block_select_ss_workspace_size (scores + projected queries).
 * ====================================================================== */
int crs_block_describe_ss(const crs_block_params *p, const void *K, const float *U, int sd, float *mu,
                          float *xi_ss, void *stream);
size_t crs_block_select_ss_workspace_size(const crs_block_sel_params *p, int sd);
int crs_block_select_ss(const crs_block_sel_params *p, const void *Q, const float *U, int sd,
                        const float *mu, const float *xi_ss, int32_t *tok_idx, int32_t *tok_count,
                        void *ws, size_t ws_bytes, void *stream);

/* The pages' deployed descriptor ([P5] "子空间方法" Eq.(17)-(18) with §5.5
 * "量化" and the delivered row of Table 3: s ~ 85, r = 4, FP4): the block mean
 * in bf16 (full space) and the r scaled eigenvectors of U^T Sigma_b U in E2M1
 * FP4 with one fp32 scale each, scored with the projected query.
 * crs_block_quantize_ss: mu [n_seq, n_kv, T/L, D] f32 and xi_ss [n_seq, n_kv,
 *   T/L, rank, sd] f32 (from crs_block_describe_ss) -> mu16 (bf16, round to
 *   nearest even), xi4 [n_seq, n_kv, T/L, rank, 48] bytes (codes of dims
 *   0..95, two per byte, the even dim in the low nibble, dims >= sd zero; the
 *   code and scale rule of crs_block_quantize), xi_scale [.., rank] f32.
 *   sd <= 96 (else CRS_ERR_UNSUPPORTED); mu, mu16, xi4 16-byte aligned.
 * crs_block_select_fp4_ss: the crs_block_select rule with
 *   s_{g,b} = qt . mu16_b + 1/2 sum_i (sigma_i code_i . U^T qt)^2, qt = scale q_g;
 *   U [D, sd] f32 row-major.  The products run on the tensor cores: Q . mu16
 *   (both exact in bf16) and code_i . p_g with p_g = U^T q_g (fp32, one FMA per
 *   term in dim order) split into a bf16 value and a bf16 residual (two query
 *   columns each), accumulated in fp32.  G = n_q / n_kv <= 8, rank <= 4 (else
 *   CRS_ERR_UNSUPPORTED); Q, mu16, xi4 16-byte aligned.  Workspace:
 *   crs_block_select_fp4_ss_workspace_size (scores + projected queries). */
int crs_block_quantize_ss(const crs_block_params *p, const float *mu, const float *xi_ss, int sd, void *mu16,
                          uint8_t *xi4, float *xi_scale, void *stream);
size_t crs_block_select_fp4_ss_workspace_size(const crs_block_sel_params *p, int sd);
int crs_block_select_fp4_ss(const crs_block_sel_params *p, const void *Q, const float *U, int sd, const void *mu16,
                            const uint8_t *xi4, const float *xi_scale, int32_t *tok_idx, int32_t *tok_count,
                            void *ws, size_t ws_bytes, void *stream);

/* ====================================================================== *
 * Quest box selector ([P5] Quest section, Eq.(23)-(24), Table 1).
 * crs_block_quest_describe: per complete block b of L keys and KV head h the
 * element-wise minimum and maximum of its keys, kmin_b, kmax_b (the keys'
 * own bf16 values: exact).  Blocks [blk_begin, blk_end) of every (sequence,
 * KV head) are written; p->rank is ignored.
 *   K: [n_seq, T, n_kv, D] bf16; kmin, kmax: [n_seq, n_kv, T/L, D] bf16.
 * crs_block_select_quest: the block selection rule of crs_block_select with
 * the box score s_{g,b} = sum_t max(qt_t kmin_{b,t}, qt_t kmax_{b,t}),
 * qt = scale * q_g, the largest inner product a point of the box reaches.
 * kmin <= kmax element-wise (as crs_block_quest_describe writes them); same
 * workspace size as crs_block_select; Q, kmin, kmax 8-byte aligned (else
 * CRS_ERR_INVALID_ARG); D = 128, G <= 16 dividing 16 (else CRS_ERR_UNSUPPORTED).
 * ====================================================================== */
int crs_block_quest_describe(const crs_block_params *p, const void *K, void *kmin, void *kmax,
                             void *stream);
int crs_block_select_quest(const crs_block_sel_params *p, const void *Q, const void *kmin,
                           const void *kmax, int32_t *tok_idx, int32_t *tok_count, void *ws,
                           size_t ws_bytes, void *stream);

/* ====================================================================== *
 * Attention over explicit index lists.  [P1] §1.1 Eq.(1) restricted to the
 * candidate set, with the allowed set P(i) of Eq.(2) cut by the causal and the
 * padding mask; [P2] §1.1 (one selected set shared by the main heads);
 * [P4] §26.2 (query heads [h*G, (h+1)*G) share KV head h):
 *   O_{t,g} = sum_{j in I} softmax_j(scale * q_{t,g} . k_{j,h}) v_{j,h},  h = g / G,
 * over the entries j of the row's list with j >= 0, j <= q_pos[t] and
 * key_valid[kv_base[t] + j] != 0.  An empty set gives O = 0 and lse = -inf.
 * Duplicated entries are a caller error.
 * ====================================================================== */
typedef struct {
    int n_rows;     /* queries                                               */
    int n_q;        /* query heads per row                                   */
    int n_kv;       /* KV heads; G = n_q / n_kv <= 16                        */
    int D;          /* head dim, 128                                         */
    int max_idx;    /* slots per index list                                  */
    int n_lists;    /* 1: one list per row shared by all KV heads;
                       n_kv: one list per (row, KV head)                     */
    int n_keys;     /* tokens held by K and V (their first dimension), >= 1:
                       an entry j of row t with kv_base[t] + j >= n_keys, or
                       j < -1, sets CRS_DEVERR_INDEX and is skipped, so no
                       entry can reach outside K/V                          */
    float scale;    /* typically 1/sqrt(D)                                   */
} crs_attn_params;

/* Q: [n_rows, n_q, D] bf16.  K, V: [n_keys, n_kv, D] bf16, token j of row t
 * and KV head h at element ((kv_base[t] + j) * n_kv + h) * D (kv_base:
 * [n_rows] int64, NULL = 0).  I: [n_rows, n_lists, max_idx] int32.
 * Masks (either may be NULL = no mask):
 *   key_valid: [n_keys] uint8, 0 marks a padding key never attended;
 *   q_pos:     [n_rows] int32, the causal limit: entries j > q_pos[t] are
 *              skipped (for a decode row of a sequence with c keys, c - 1).
 * O: [n_rows, n_q, D] f32 (the fp32 accumulator's precision; P.V runs on bf16
 * tensor cores with P split into a bf16 value and a bf16 residual);
 * lse: [n_rows, n_q] f32 or NULL.
 * Q, K, V and the workspace must start on 16-byte boundaries (rows are read as
 * 16-byte pieces; else CRS_ERR_INVALID_ARG).
 * Workspace: crs_sparse_attn_workspace_size(p), queried with the same device
 * current as the call (the split count depends on the device's SM count). */
size_t crs_sparse_attn_workspace_size(const crs_attn_params *p);
int crs_sparse_attn(const crs_attn_params *p, const void *Q, const void *K, const void *V,
                    const int64_t *kv_base, const int32_t *I, const uint8_t *key_valid,
                    const int32_t *q_pos, void *O, float *lse, void *ws, size_t ws_bytes,
                    void *stream);

#ifdef __cplusplus
}
#endif
#endif /* CRS_H */
