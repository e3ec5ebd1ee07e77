/*
 * CPU oracle for content-routed sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg load this library.  It shares no code, header, table or
 * helper with the CUDA path: every function below is the plain definition of
 * one step, written out in loops, in fp64 unless a step's integer decision is
 * taken in fp32 (the LSH bucket, see oracle_lsh_hash).  OpenMP only splits
 * independent rows across cores; it never changes an operation order.
 *
 * Pages cited:
 *   [P1] PaperTrace 2.1.1 "哈希与聚类: 用内容建立稀疏注意力邻域"
 *   [P2] PaperTrace 2.2 "细粒度索引: 用轻量 selector 召回关键 token"
 *   [P4] Understanding LLMs ch. 26 "高效、稀疏与替代架构地图"
 *   [P5] "COBS 阅读笔记: 块稀疏注意力的选择器到底漏掉了什么"
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OAPI __attribute__((visibility("default")))

/* Threads used by later calls (rows are split across them; no operation order
 * depends on the count), and the current count. */
OAPI void oracle_set_num_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
OAPI int oracle_max_threads(void) { return omp_get_max_threads(); }

/* ======================================================================
 * O1  LSH bucket id.  [P1] §2.1 Eq.(4): u = x R with R in R^{d x b/2};
 * the bucket is the argmax of the concatenation [u ; -u] over b entries.
 * The argmax is an integer decided by floating point, so it is taken in the
 * precision of the kernel: each u_k is one fp32 fused multiply-add per term,
 * terms in increasing index order starting from 0.  Ties go to the lowest
 * index (the first maximum met scanning j = 0..b-1).
 * Layout: X [B,H,n,d] fp32, R [H,rounds,d,b/2] fp32, bucket [B,H,rounds,n].
 * ====================================================================== */
OAPI void oracle_lsh_hash(int B, int H, int n, int d, int n_buckets, int n_rounds,
                          const float *X, const float *R, int32_t *bucket)
{
    const int half = n_buckets / 2;
    const long nbh = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < nbh; ++bh) {
        const int h = (int)(bh % H);
        for (int i = 0; i < n; ++i) {
            const float *x = X + (bh * n + i) * (long)d;
            for (int r = 0; r < n_rounds; ++r) {
                const float *Rr = R + ((long)h * n_rounds + r) * (long)d * half;
                int arg = 0;
                float best = 0.0f;
                for (int j = 0; j < n_buckets; ++j) {
                    const int k = (j < half) ? j : j - half;
                    float u = 0.0f;
                    for (int t = 0; t < d; ++t)
                        u = fmaf(x[t], Rr[(long)t * half + k], u);
                    const float c = (j < half) ? u : -u;
                    if (j == 0 || c > best) {
                        best = c;
                        arg = j;
                    }
                }
                bucket[(bh * n_rounds + r) * (long)n + i] = arg;
            }
        }
    }
}

/* fp64 companion of O1: the gap between the largest and second largest entry
 * of [u ; -u] computed in fp64, per (b,h,r,i).  Reported by tests as the
 * distance of each bucket decision from a tie. */
OAPI void oracle_lsh_margin(int B, int H, int n, int d, int n_buckets, int n_rounds,
                            const float *X, const float *R, double *margin)
{
    const int half = n_buckets / 2;
    const long nbh = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < nbh; ++bh) {
        const int h = (int)(bh % H);
        for (int i = 0; i < n; ++i) {
            const float *x = X + (bh * n + i) * (long)d;
            for (int r = 0; r < n_rounds; ++r) {
                const float *Rr = R + ((long)h * n_rounds + r) * (long)d * half;
                double b1 = -INFINITY, b2 = -INFINITY;
                for (int j = 0; j < n_buckets; ++j) {
                    const int k = (j < half) ? j : j - half;
                    double u = 0.0;
                    for (int t = 0; t < d; ++t)
                        u += (double)x[t] * (double)Rr[(long)t * half + k];
                    const double c = (j < half) ? u : -u;
                    if (c > b1) {
                        b2 = b1;
                        b1 = c;
                    } else if (c > b2) {
                        b2 = c;
                    }
                }
                margin[(bh * n_rounds + r) * (long)n + i] = b1 - b2;
            }
        }
    }
}

/* ======================================================================
 * O1  Sort.  [P1] §2.1 (last paragraph) and §2.2: the sort key combines the
 * bucket id and the position; sorting tokens by it gives the permutation pi
 * (slot -> original position); pi^{-1} maps a position back to its slot.
 * Key = bucket * n + pos, ascending.  Keys are unique, so this equals a
 * stable sort on the bucket id.
 * ====================================================================== */
static int cmp_i64(const void *a, const void *b)
{
    const int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

OAPI void oracle_lsh_sort(int n_segments, int n, const int32_t *bucket,
                          int32_t *perm, int32_t *inv_perm)
{
#pragma omp parallel for schedule(static)
    for (long sg = 0; sg < n_segments; ++sg) {
        int64_t *key = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        const int32_t *bk = bucket + sg * (long)n;
        for (int p = 0; p < n; ++p)
            key[p] = (int64_t)bk[p] * n + p;
        qsort(key, (size_t)n, sizeof(int64_t), cmp_i64);
        for (int s = 0; s < n; ++s) {
            const int p = (int)(key[s] % n);
            perm[sg * (long)n + s] = p;
            inv_perm[sg * (long)n + p] = s;
        }
        free(key);
    }
}

/* ======================================================================
 * O2  Candidate set of query i in one (batch, head).
 * [P1] §2.1-2.2: after sorting, the sorted array is cut into chunks of m
 * slots; a query's chunk attends to itself and to the previous chunk (chunk 0
 * has none); a legal edge still needs the same bucket id and is judged on the
 * original positions.  [P1] §1.1 Eq.(2): N(i) = B(i) ∩ C(i) ∩ P(i): content,
 * causal (j <= i) and valid (j < valid_len); optionally no self (j != i).
 * Several rounds: the union over rounds, a set ([P1] "重复候选和归一化":
 * duplicates are removed before the softmax).
 * Arrays bucket/perm/inv_perm point at this (b,h): [rounds, n].
 * Returns |U(i)|; cand[] receives U(i) in ascending order.  mark[] is n bytes
 * of zeroed scratch and is left zeroed.
 * ====================================================================== */
static int cmp_i32(const void *a, const void *b)
{
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

OAPI int oracle_lsh_candidates(int n, int n_rounds, int m, int causal, int no_self,
                               int valid_len, const int32_t *bucket, const int32_t *perm,
                               const int32_t *inv_perm, int i, int32_t *cand, uint8_t *mark)
{
    int cnt = 0;
    for (int r = 0; r < n_rounds; ++r) {
        const int32_t *bk = bucket + (long)r * n;
        const int32_t *pm = perm + (long)r * n;
        const int32_t *ip = inv_perm + (long)r * n;
        const int c = ip[i] / m;
        for (int cc = c - 1; cc <= c; ++cc) {
            if (cc < 0)
                continue;
            const int s0 = cc * m;
            const int s1 = (s0 + m < n) ? s0 + m : n;
            for (int s = s0; s < s1; ++s) {
                const int j = pm[s];
                if (bk[j] != bk[i]) continue;
                if (causal && j > i) continue;
                if (no_self && j == i) continue;
                if (j >= valid_len) continue;
                if (!mark[j]) {
                    mark[j] = 1;
                    cand[cnt++] = j;
                }
            }
        }
    }
    for (int t = 0; t < cnt; ++t)
        mark[cand[t]] = 0;
    qsort(cand, (size_t)cnt, sizeof(int32_t), cmp_i32);
    return cnt;
}

/* ======================================================================
 * O3  LSH attention.  [P1] §1.1 Eq.(1): O_i = sum_{j in N(i)} softmax_j(s_ij) v_j,
 * with the shared-QK key k_j = q_j / |q_j| ([P1] §2, Reformer: the query
 * keeps its norm) when key_norm != 0, k_j = q_j otherwise; s_ij = scale * q_i.k_j.
 * Computed directly over the union set U(i): no per-round merge.  A query
 * with an empty set, and every padded query (i >= valid_len), gets O_i = 0
 * and lse = -inf.  A zero-norm key is the zero vector.
 * Layout: QK, V [B,H,n,d] fp64; bucket/perm/inv_perm [B,H,rounds,n];
 * valid_len [B]; rows: the query positions to compute (NULL = all n), the
 * outputs O [B,H,n_rows,d], lse [B,H,n_rows], count [B,H,n_rows].
 * ====================================================================== */
OAPI void oracle_lsh_attn(int B, int H, int n, int d, int n_rounds, int m, int causal,
                          int no_self, int key_norm, double scale, const double *QK,
                          const double *V, const int32_t *bucket, const int32_t *perm,
                          const int32_t *inv_perm, const int32_t *valid_len,
                          const int32_t *rows, int n_rows, double *O, double *lse,
                          int32_t *count)
{
    const long nbh = (long)B * H;
    const int nr = rows ? n_rows : n;
#pragma omp parallel
    {
        int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        uint8_t *mark = (uint8_t *)calloc((size_t)n, 1);
        double *logit = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (long bh = 0; bh < nbh; ++bh) {
            for (int t = 0; t < nr; ++t) {
                const int b = (int)(bh / H);
                const int i = rows ? rows[t] : t;
                const long seg = bh * (long)n_rounds * n;
                const double *Qb = QK + bh * (long)n * d;
                const double *Vb = V + bh * (long)n * d;
                double *o = O + (bh * nr + t) * (long)d;
                for (int k = 0; k < d; ++k)
                    o[k] = 0.0;
                double l = -INFINITY;
                int cnt = 0;
                if (i < valid_len[b]) {
                    cnt = oracle_lsh_candidates(n, n_rounds, m, causal, no_self, valid_len[b],
                                                bucket + seg, perm + seg, inv_perm + seg, i,
                                                cand, mark);
                    if (cnt > 0) {
                        const double *qi = Qb + (long)i * d;
                        double mx = -INFINITY;
                        for (int c = 0; c < cnt; ++c) {
                            const double *qj = Qb + (long)cand[c] * d;
                            double dot = 0.0, nn = 0.0;
                            for (int k = 0; k < d; ++k) {
                                dot += qi[k] * qj[k];
                                nn += qj[k] * qj[k];
                            }
                            double s;
                            if (key_norm)
                                s = (nn > 0.0) ? scale * dot / sqrt(nn) : 0.0;
                            else
                                s = scale * dot;
                            logit[c] = s;
                            if (s > mx) mx = s;
                        }
                        double z = 0.0;
                        for (int c = 0; c < cnt; ++c)
                            z += exp(logit[c] - mx);
                        for (int c = 0; c < cnt; ++c) {
                            const double p = exp(logit[c] - mx) / z;
                            const double *vj = Vb + (long)cand[c] * d;
                            for (int k = 0; k < d; ++k)
                                o[k] += p * vj[k];
                        }
                        l = mx + log(z);
                    }
                }
                lse[bh * nr + t] = l;
                count[bh * nr + t] = cnt;
            }
        }
        free(cand);
        free(mark);
        free(logit);
    }
}

/* ======================================================================
 * O3d  LSH decode step.  [P1] §5.2 "Prefill、Decode 与 KV 状态": with the hash
 * fixed, a new key's bucket ids are computed once and appended to the bucket
 * lists; the new query reads the lists of its own buckets.  Reading: the
 * newest token t = len-1 of a row attends to
 *   U(t) = { j <= t : bucket_r(j) == bucket_r(t) for some round r },
 * without j == t when no_self, each j once (pairs counted once across rounds,
 * as O3), with no chunk window (the whole bucket is the neighbourhood in
 * decode); keys, scale, the empty set and lse as O3.
 * Layout: X, V [S, H, n_max, d] fp64; bucket [S, H, rounds, n_max] (from O1
 * on the fp32 vectors); len [S] = tokens of row s including the new one;
 * outputs O [S, H, d], lse [S, H], count [S, H].
 * ====================================================================== */
OAPI void oracle_lsh_decode(int S, int H, int n_max, int d, int n_rounds, int no_self, int key_norm,
                            double scale, const double *X, const double *V, const int32_t *bucket,
                            const int32_t *len, double *O, double *lse, int32_t *count)
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < S; ++s)
        for (int h = 0; h < H; ++h) {
            const long sh = (long)s * H + h;
            const int t = len[s] - 1;
            const double *x = X + sh * n_max * d, *v = V + sh * n_max * d;
            const int32_t *bk = bucket + sh * (long)n_rounds * n_max;
            double *o = O + sh * d;
            double mx = -INFINITY;
            int cnt = 0;
            for (int pass = 0; pass < 2; ++pass) {          /* 0: max logit, 1: accumulate */
                double z = 0.0;
                if (pass == 1)
                    for (int c = 0; c < d; ++c)
                        o[c] = 0.0;
                for (int j = 0; j <= t; ++j) {
                    if (no_self && j == t) continue;
                    int hit = 0;
                    for (int r = 0; r < n_rounds && !hit; ++r)
                        hit = bk[(long)r * n_max + j] == bk[(long)r * n_max + t];
                    if (!hit) continue;
                    double nrm = 1.0;
                    if (key_norm) {
                        nrm = 0.0;
                        for (int c = 0; c < d; ++c)
                            nrm += x[(long)j * d + c] * x[(long)j * d + c];
                        nrm = sqrt(nrm);
                    }
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c)
                        dot += x[(long)t * d + c] * x[(long)j * d + c];
                    const double lg = nrm > 0.0 ? scale * dot / nrm : 0.0;
                    if (pass == 0) {
                        if (lg > mx) mx = lg;
                        ++cnt;
                    } else {
                        const double e = exp(lg - mx);
                        z += e;
                        for (int c = 0; c < d; ++c)
                            o[c] += e * v[(long)j * d + c];
                    }
                }
                if (pass == 1) {
                    if (cnt == 0) {
                        lse[sh] = -INFINITY;
                    } else {
                        for (int c = 0; c < d; ++c)
                            o[c] /= z;
                        lse[sh] = mx + log(z);
                    }
                }
            }
            count[sh] = cnt;
        }
}

/* ======================================================================
 * O4  Lightning-indexer score and token top-k.
 * [P2] §1.1 and §2.1 Eq.(3)-(4): r_{t,s} = sum_h w_{t,h} ReLU(q_{t,h} . k_s)
 * over the index heads, no extra scale; S_t = Select(r_{t,0:t}, k) keeps the k
 * largest.  [P2] §2.1 "Select 不等于一次普通 top-k": a row with fewer than k
 * visible keys returns them all and marks the other slots invalid (-1);
 * [P2] §3.1 "多卡一致性": ties are broken lexicographically on (score, index),
 * i.e. equal scores prefer the smaller index.  Output ascending by position.
 * Layout: q [rows, heads, d]; w [rows, heads]; K: keys of row t are
 * K[(key_base[t] + s) * d + .] for s < n_visible[t].
 * ====================================================================== */
OAPI void oracle_indexer_score(int n_heads, int d, const double *q, const double *w,
                               const double *K, long n_keys, double *out)
{
    for (long s = 0; s < n_keys; ++s) {
        const double *k = K + s * d;
        double r = 0.0;
        for (int h = 0; h < n_heads; ++h) {
            double dot = 0.0;
            for (int t = 0; t < d; ++t)
                dot += q[h * d + t] * k[t];
            r += w[h] * (dot > 0.0 ? dot : 0.0);
        }
        out[s] = r;
    }
}

typedef struct {
    double s;
    int32_t i;
} scored_t;

static int cmp_score_desc_idx_asc(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i > y->i) - (x->i < y->i);
}

OAPI void oracle_indexer_topk(int n_rows, int n_heads, int d, int topk, const double *q,
                              const double *w, const double *K, const int64_t *key_base,
                              const int32_t *n_visible, int32_t *out_idx, int32_t *out_count,
                              double *out_cutoff, double *out_next)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < n_rows; ++t) {
        const int nv = n_visible[t];
        scored_t *sc = (scored_t *)malloc(sizeof(scored_t) * (size_t)(nv > 0 ? nv : 1));
        double *tmp = (double *)malloc(sizeof(double) * (size_t)(nv > 0 ? nv : 1));
        oracle_indexer_score(n_heads, d, q + t * (long)n_heads * d, w + t * (long)n_heads,
                             K + key_base[t] * (long)d, nv, tmp);
        for (int s = 0; s < nv; ++s) {
            sc[s].s = tmp[s];
            sc[s].i = s;
        }
        qsort(sc, (size_t)nv, sizeof(scored_t), cmp_score_desc_idx_asc);
        const int kk = nv < topk ? nv : topk;
        int32_t *o = out_idx + t * (long)topk;
        for (int c = 0; c < kk; ++c)
            o[c] = sc[c].i;
        qsort(o, (size_t)kk, sizeof(int32_t), cmp_i32);
        for (int c = kk; c < topk; ++c)
            o[c] = -1;
        out_count[t] = kk;
        out_cutoff[t] = kk > 0 ? sc[kk - 1].s : -INFINITY;
        out_next[t] = nv > kk ? sc[kk].s : -INFINITY;
        free(sc);
        free(tmp);
    }
}

/* ======================================================================
 * O3k  Routing (k-means) attention with quota execution.  [P1] §3.1: with the
 * centres M frozen (inference), the routing scores are S_Q = Q M^T and
 * S_K = K M^T; each centre c takes its m best queries and m best keys,
 *   J_c^Q = Top_m(S_Q[:, c]),  J_c^K = Top_m(S_K[:, c]),
 * a token may belong to several centres, and each query's outputs over its
 * centres must be combined at its original index ("定额执行").  The score is
 * an integer decision taken in fp32 as O1: one fused multiply-add per term in
 * increasing index order from 0; Top_m keeps (score desc, index asc).
 * Reading: query i attends to the union U(i) of J_c^K over the centres c with
 * i in J_c^Q, each key once (pairs counted once, as O3), restricted to j <= i
 * when causal and to j != i when no_self; logits scale * q_i . k_j (separate
 * Q and K, no normalisation); an empty set gives O = 0, lse = -inf.
 * Layout: Qf, Kf [B,H,n,d] fp32 (for the scores), Q, K, V [B,H,n,d] fp64,
 * M [H, C, d] fp32; outputs JQ, JK [B,H,C,m] (ascending), O [B,H,n,d],
 * lse [B,H,n], count [B,H,n].
 * ====================================================================== */
static float route_score(const float *x, const float *mu, int d)
{
    float acc = 0.0f;
    for (int t = 0; t < d; ++t)
        acc = fmaf(x[t], mu[t], acc);
    return acc;
}

OAPI void oracle_kmeans_route(int B, int H, int n, int d, int C, int m, int causal, int no_self, double scale,
                              const float *Qf, const float *Kf, const float *M, const double *Q,
                              const double *K, const double *V, int32_t *JQ, int32_t *JK, double *O,
                              double *lse, int32_t *count)
{
    const int mm = m < n ? m : n;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const long bh = (long)b * H + h;
            scored_t *sc = (scored_t *)malloc(sizeof(scored_t) * (size_t)n);
            uint8_t *inq = (uint8_t *)calloc((size_t)n * C, 1);   /* [i][c]: i in J_c^Q */
            uint8_t *ink = (uint8_t *)calloc((size_t)n * C, 1);
            for (int role = 0; role < 2; ++role) {
                const float *X = (role == 0 ? Qf : Kf) + bh * (long)n * d;
                int32_t *J = (role == 0 ? JQ : JK) + bh * (long)C * m;
                uint8_t *in = role == 0 ? inq : ink;
                for (int c = 0; c < C; ++c) {
                    const float *mu = M + ((long)h * C + c) * d;
                    for (int i = 0; i < n; ++i) {
                        sc[i].s = (double)route_score(X + (long)i * d, mu, d);
                        sc[i].i = i;
                    }
                    qsort(sc, (size_t)n, sizeof(scored_t), cmp_score_desc_idx_asc);
                    int32_t *Jc = J + (long)c * m;
                    for (int k = 0; k < mm; ++k)
                        Jc[k] = sc[k].i;
                    qsort(Jc, (size_t)mm, sizeof(int32_t), cmp_i32);
                    for (int k = mm; k < m; ++k)
                        Jc[k] = -1;
                    for (int k = 0; k < mm; ++k)
                        in[(long)Jc[k] * C + c] = 1;
                }
            }
            const double *q = Q + bh * (long)n * d, *k = K + bh * (long)n * d, *v = V + bh * (long)n * d;
            for (int i = 0; i < n; ++i) {
                double *o = O + (bh * n + i) * d;
                for (int t = 0; t < d; ++t)
                    o[t] = 0.0;
                double mx = -INFINITY, z = 0.0;
                int cnt = 0;
                for (int pass = 0; pass < 2; ++pass)
                    for (int j = 0; j < n; ++j) {
                        if (causal && j > i) continue;
                        if (no_self && j == i) continue;
                        int hit = 0;
                        for (int c = 0; c < C && !hit; ++c)
                            hit = inq[(long)i * C + c] && ink[(long)j * C + c];
                        if (!hit) continue;
                        double dot = 0.0;
                        for (int t = 0; t < d; ++t)
                            dot += q[(long)i * d + t] * k[(long)j * d + t];
                        const double lg = scale * dot;
                        if (pass == 0) {
                            if (lg > mx) mx = lg;
                            ++cnt;
                        } else {
                            const double e = exp(lg - mx);
                            z += e;
                            for (int t = 0; t < d; ++t)
                                o[t] += e * v[(long)j * d + t];
                        }
                    }
                if (cnt > 0) {
                    for (int t = 0; t < d; ++t)
                        o[t] /= z;
                    lse[bh * n + i] = mx + log(z);
                } else {
                    lse[bh * n + i] = -INFINITY;
                }
                count[bh * n + i] = cnt;
            }
            free(sc);
            free(inq);
            free(ink);
        }
}

/* ======================================================================
 * O4h  Hierarchical indexer (HISA), decode rows.  [P2] "索引器的三种降本方向"
 * and §2.2 Eq.(7): the history of a row is cut into blocks of `blk` keys;
 * each complete block has a representative (reading: the mean of its index
 * keys, d_c = d) scored with the indexer's own formula,
 *   c_j = sum_h w_h ReLU(q_h . rep_j);
 * the top_blocks blocks by (c desc, block asc) are kept (all of them when the
 * row has fewer); the original token indexer then runs only on the kept
 * blocks' keys and on the open (incomplete) trailing block ([P2] "未满块由局部
 * 或单独 open-block 路径处理"), and returns the same top-k interface as O4
 * (ties to the smaller position, ascending, -1 padded).  The kept blocks are
 * returned too (ascending, -1 padded): the pages keep each level's candidates
 * to locate a miss ([P2] "失败样本怎样定位到具体层级").
 * Layout: keys of row s are K[k_offsets[s] .. k_offsets[s+1]); block j of row s
 * has rep[(blk_offsets[s] + j) * d + .], j < (k_offsets[s+1]-k_offsets[s])/blk.
 * given_blocks (optional, [n_rows, top_blocks], -1 padded) replaces the
 * coarse selection: the fine stage on a given candidate set.
 * ====================================================================== */
OAPI void oracle_hisa_describe(int n_rows, int d, int blk, const double *K, const int64_t *k_offsets,
                               const int64_t *blk_offsets, double *rep)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < n_rows; ++t) {
        const long ctx = (long)(k_offsets[t + 1] - k_offsets[t]);
        const long nb = ctx / blk;
        for (long j = 0; j < nb; ++j) {
            double *r = rep + (blk_offsets[t] + j) * d;
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int i = 0; i < blk; ++i)
                    acc += K[(k_offsets[t] + j * blk + i) * d + c];
                r[c] = acc / blk;
            }
        }
    }
}

/* One row: query qt / weights wt, its keys Kr[0 .. ctx), the representatives
 * rep_r of its ctx / blk complete blocks; given (or NULL) replaces the coarse
 * selection; coarse_r (or NULL) receives the coarse scores. */
static void hisa_row(int n_heads, int d, int topk, int blk, int top_blocks, const double *qt,
                     const double *wt, const double *Kr, long ctx, const double *rep_r,
                     const int32_t *given, int32_t *ob, int32_t *o, int32_t *count, double *coarse_r)
{
    const int nb = (int)(ctx / blk);
    int nkeep = 0;
    if (given) {
        for (int c = 0; c < top_blocks; ++c)
            if (given[c] >= 0)
                ob[nkeep++] = given[c];
    } else {
        scored_t *sc = (scored_t *)malloc(sizeof(scored_t) * (size_t)(nb > 0 ? nb : 1));
        double *cs = (double *)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
        oracle_indexer_score(n_heads, d, qt, wt, rep_r, nb, cs);
        for (int j = 0; j < nb; ++j) {
            sc[j].s = cs[j];
            sc[j].i = j;
            if (coarse_r) coarse_r[j] = cs[j];
        }
        qsort(sc, (size_t)nb, sizeof(scored_t), cmp_score_desc_idx_asc);
        nkeep = nb < top_blocks ? nb : top_blocks;
        for (int c = 0; c < nkeep; ++c)
            ob[c] = sc[c].i;
        free(sc);
        free(cs);
    }
    qsort(ob, (size_t)nkeep, sizeof(int32_t), cmp_i32);
    for (int c = nkeep; c < top_blocks; ++c)
        ob[c] = -1;
    /* candidates: the kept blocks' keys, then the open block's */
    const long open0 = (long)nb * blk;
    const long ncand = (long)nkeep * blk + (ctx - open0);
    scored_t *sc = (scored_t *)malloc(sizeof(scored_t) * (size_t)(ncand > 0 ? ncand : 1));
    double one;
    long c = 0;
    for (int b = 0; b < nkeep; ++b)
        for (int i = 0; i < blk; ++i, ++c) {
            const long pos = (long)ob[b] * blk + i;
            oracle_indexer_score(n_heads, d, qt, wt, Kr + pos * d, 1, &one);
            sc[c].s = one;
            sc[c].i = (int32_t)pos;
        }
    for (long pos = open0; pos < ctx; ++pos, ++c) {
        oracle_indexer_score(n_heads, d, qt, wt, Kr + pos * d, 1, &one);
        sc[c].s = one;
        sc[c].i = (int32_t)pos;
    }
    qsort(sc, (size_t)ncand, sizeof(scored_t), cmp_score_desc_idx_asc);
    const int kk = ncand < topk ? (int)ncand : topk;
    for (int i = 0; i < kk; ++i)
        o[i] = sc[i].i;
    qsort(o, (size_t)kk, sizeof(int32_t), cmp_i32);
    for (int i = kk; i < topk; ++i)
        o[i] = -1;
    *count = kk;
    free(sc);
}

OAPI void oracle_hisa_topk(int n_rows, int n_heads, int d, int topk, int blk, int top_blocks,
                           const double *q, const double *w, const double *K, const int64_t *k_offsets,
                           const double *rep, const int64_t *blk_offsets, const int32_t *given_blocks,
                           int32_t *out_blocks, int32_t *out_idx, int32_t *out_count,
                           double *coarse_score)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < n_rows; ++t)
        hisa_row(n_heads, d, topk, blk, top_blocks, q + t * (long)n_heads * d, w + t * (long)n_heads,
                 K + k_offsets[t] * (long)d, (long)(k_offsets[t + 1] - k_offsets[t]),
                 rep + blk_offsets[t] * (long)d, given_blocks ? given_blocks + t * (long)top_blocks : NULL,
                 out_blocks + t * (long)top_blocks, out_idx + t * (long)topk, out_count + t,
                 coarse_score ? coarse_score + blk_offsets[t] : NULL);
}

/* O4h, prefill (causal) form: the n queries of one sequence, query i seeing
 * keys 0..i as the flat indexer's prefill rows do ([P2] §2.1 Eq.(4), S_t over
 * r_{t,0:t}).  Its complete blocks are the sequence's blocks j < (i + 1) / blk,
 * whose representatives (rep, computed once for the sequence) do not depend on
 * the query; the rest is the row rule above with ctx = i + 1.  Layout: q [n,
 * heads, d]; w [n, heads]; K [n, d]; rep [n / blk, d]; outputs per query. */
OAPI void oracle_hisa_topk_prefill(int n, int n_heads, int d, int topk, int blk, int top_blocks,
                                   const double *q, const double *w, const double *K, const double *rep,
                                   int32_t *out_blocks, int32_t *out_idx, int32_t *out_count)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (long i = 0; i < n; ++i)
        hisa_row(n_heads, d, topk, blk, top_blocks, q + i * (long)n_heads * d, w + i * (long)n_heads, K,
                 i + 1, rep, NULL, out_blocks + i * (long)top_blocks, out_idx + i * (long)topk, out_count + i,
                 NULL);
}

/* ======================================================================
 * O5  Block descriptor.  [P5] Eq.(11): mean key and population covariance
 * Sigma_b = (1/L) sum (k_r - kbar)(k_r - kbar)^T; Eq.(16): keep the r largest
 * eigen-directions, xi_i = sqrt(lambda_i) u_i; Eq.(20) / Algorithm 2 (Gram
 * route): eigen-decompose G = (1/L) Kt Kt^T (L x L) and map back with
 * xi_i = Kt^T w_i / sqrt(L).  A partial block uses its own count L' for L.
 * The eigen-decomposition is the cyclic Jacobi method (Jacobi 1846; as in
 * Golub & Van Loan, "Matrix Computations", symmetric Schur 2x2 rotations),
 * swept until the off-diagonal mass is below 1e-30 of the total.
 * Layout: K [n_blocks, L_cap, D] fp64 (rows >= L_eff[b] ignored); outputs
 * mu [n_blocks, D], xi [n_blocks, rank, D], lam [n_blocks, rank] (descending).
 * ====================================================================== */
static void jacobi_eig(int n, double *A, double *Vm)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j)
            Vm[i * n + j] = (i == j) ? 1.0 : 0.0;
    double total = 0.0;
    for (int i = 0; i < n * n; ++i)
        total += A[i] * A[i];
    for (int sweep = 0; sweep < 100; ++sweep) {
        double off = 0.0;
        for (int p = 0; p < n; ++p)
            for (int q = 0; q < n; ++q)
                if (p != q) off += A[p * n + q] * A[p * n + q];
        if (off <= 1e-30 * total || off == 0.0)
            break;
        for (int p = 0; p < n - 1; ++p) {
            for (int q = p + 1; q < n; ++q) {
                const double apq = A[p * n + q];
                if (apq == 0.0) continue;
                const double theta = (A[q * n + q] - A[p * n + p]) / (2.0 * apq);
                const double t = (theta >= 0.0 ? 1.0 : -1.0) /
                                 (fabs(theta) + sqrt(theta * theta + 1.0));
                const double c = 1.0 / sqrt(t * t + 1.0);
                const double s = t * c;
                /* A <- J^T A J with J the rotation in the (p,q) plane */
                for (int k = 0; k < n; ++k) {
                    const double akp = A[k * n + p], akq = A[k * n + q];
                    A[k * n + p] = c * akp - s * akq;
                    A[k * n + q] = s * akp + c * akq;
                }
                for (int k = 0; k < n; ++k) {
                    const double apk = A[p * n + k], aqk = A[q * n + k];
                    A[p * n + k] = c * apk - s * aqk;
                    A[q * n + k] = s * apk + c * aqk;
                }
                for (int k = 0; k < n; ++k) {
                    const double vkp = Vm[k * n + p], vkq = Vm[k * n + q];
                    Vm[k * n + p] = c * vkp - s * vkq;
                    Vm[k * n + q] = s * vkp + c * vkq;
                }
            }
        }
    }
}

/* U == NULL: the descriptors of the full key space (Y = Kt, sd = D).  Else
 * U [D, sd] (row-major) spans the query subspace and the eigenvectors are
 * taken of the projected covariance B = U^T Sigma U, [P5] Eq.(17), by the
 * same Gram route on Y = Kt U: G = Y Y^T / L, xi_i = Y^T w_i / sqrt(L) in R^sd. */
static void block_describe_core(int n_blocks, int L_cap, int D, int rank, const double *K,
                                const int32_t *L_eff, const double *U, int sd, double *mu, double *xi,
                                double *lam)
{
#pragma omp parallel
    {
        double *Kt = (double *)malloc(sizeof(double) * (size_t)L_cap * D);
        double *Y = (double *)malloc(sizeof(double) * (size_t)L_cap * sd);
        double *G = (double *)malloc(sizeof(double) * (size_t)L_cap * L_cap);
        double *W = (double *)malloc(sizeof(double) * (size_t)L_cap * L_cap);
        int *order = (int *)malloc(sizeof(int) * (size_t)L_cap);
#pragma omp for schedule(dynamic, 8)
        for (long b = 0; b < n_blocks; ++b) {
            const int L = L_eff ? L_eff[b] : L_cap;
            const double *Kb = K + b * (long)L_cap * D;
            double *m = mu + b * (long)D;
            for (int t = 0; t < D; ++t) {
                double acc = 0.0;
                for (int r = 0; r < L; ++r)
                    acc += Kb[(long)r * D + t];
                m[t] = (L > 0) ? acc / L : 0.0;
            }
            for (int r = 0; r < L; ++r)
                for (int t = 0; t < D; ++t)
                    Kt[(long)r * D + t] = Kb[(long)r * D + t] - m[t];
            for (int r = 0; r < L; ++r)
                for (int j = 0; j < sd; ++j) {
                    if (!U) {
                        Y[(long)r * sd + j] = Kt[(long)r * D + j];
                        continue;
                    }
                    double acc = 0.0;
                    for (int t = 0; t < D; ++t)
                        acc += Kt[(long)r * D + t] * U[(long)t * sd + j];
                    Y[(long)r * sd + j] = acc;
                }
            for (int i = 0; i < L; ++i)
                for (int j = 0; j < L; ++j) {
                    double acc = 0.0;
                    for (int t = 0; t < sd; ++t)
                        acc += Y[(long)i * sd + t] * Y[(long)j * sd + t];
                    G[i * L + j] = acc / L;
                }
            if (L > 0)
                jacobi_eig(L, G, W);
            /* order eigenpairs by eigenvalue, descending (selection sort, ties by index) */
            for (int i = 0; i < L; ++i)
                order[i] = i;
            for (int i = 0; i < L; ++i) {
                int best = i;
                for (int j = i + 1; j < L; ++j)
                    if (G[order[j] * L + order[j]] > G[order[best] * L + order[best]])
                        best = j;
                const int tmp = order[i];
                order[i] = order[best];
                order[best] = tmp;
            }
            for (int e = 0; e < rank; ++e) {
                double *x = xi + (b * (long)rank + e) * sd;
                if (e >= L) {
                    for (int t = 0; t < sd; ++t)
                        x[t] = 0.0;
                    lam[b * (long)rank + e] = 0.0;
                    continue;
                }
                const int col = order[e];
                lam[b * (long)rank + e] = G[col * L + col];
                for (int t = 0; t < sd; ++t) {
                    double acc = 0.0;
                    for (int r = 0; r < L; ++r)
                        acc += Y[(long)r * sd + t] * W[r * L + col];
                    x[t] = acc / sqrt((double)L);
                }
            }
        }
        free(Kt);
        free(Y);
        free(G);
        free(W);
        free(order);
    }
}

OAPI void oracle_block_describe(int n_blocks, int L_cap, int D, int rank, const double *K,
                                const int32_t *L_eff, double *mu, double *xi, double *lam)
{
    block_describe_core(n_blocks, L_cap, D, rank, K, L_eff, NULL, D, mu, xi, lam);
}

/* O5s  Subspace descriptors ([P5] "子空间方法", Eq.(17)-(18)): U [D, sd] holds
 * the query-subspace basis (orthonormal columns, computed offline from the
 * queries' second moment); xi [n_blocks, rank, sd] are the scaled top-rank
 * eigenvectors of U^T Sigma_b U; mu as in O5. */
OAPI void oracle_block_describe_ss(int n_blocks, int L_cap, int D, int sd, int rank, const double *K,
                                   const double *U, double *mu, double *xi, double *lam)
{
    block_describe_core(n_blocks, L_cap, D, rank, K, NULL, U, sd, mu, xi, lam);
}

/* Exact block log-mass, [P5] Eq.(1): ln m_b = ln sum_{r in b} exp(q . k_r).
 * Used by tests as the OSA reference ([P5] Algorithm 1) and for the toy
 * example of [P5] Eq.(P4)-(P5). */
OAPI double oracle_block_log_mass(int L, int D, const double *q, const double *Kb)
{
    double mx = -INFINITY;
    for (int r = 0; r < L; ++r) {
        double s = 0.0;
        for (int t = 0; t < D; ++t)
            s += q[t] * Kb[(long)r * D + t];
        if (s > mx) mx = s;
    }
    double z = 0.0;
    for (int r = 0; r < L; ++r) {
        double s = 0.0;
        for (int t = 0; t < D; ++t)
            s += q[t] * Kb[(long)r * D + t];
        z += exp(s - mx);
    }
    return mx + log(z);
}

/* ======================================================================
 * O6  Block selection.  [P5] Eq.(14)/(19): the second-order log-mass
 * estimate, without the ln L constant that cancels in the ranking,
 *   s_{g,b} = qt . mu_b + 1/2 sum_i (xi_i . qt)^2,  qt = scale * q_g;
 * [P5] Eq.(15)/(6): for KV head h the block score is the sum over its
 * query-head group of each head's softmax over blocks,
 *   score_b = sum_{g in group(h)} exp(s_{g,b}) / sum_{b'} exp(s_{g,b'});
 * keep the top_blocks blocks by (score desc, block asc) among the
 * n_full = floor(T / L) complete blocks; the token set is the union of the
 * kept blocks' positions and the window [T - window, T), without duplicates,
 * ascending.  Query heads of group h are [h*G, (h+1)*G) ([P4] §26.2).
 * Layout: Q [n_seq, n_q, D]; mu [n_seq, n_kv, n_full, D];
 * xi [n_seq, n_kv, n_full, rank, D]; outputs tok [n_seq, n_kv, cap] (-1 pad),
 * tok_count [n_seq, n_kv], blk [n_seq, n_kv, top_blocks] (ascending),
 * blk_score [n_seq, n_kv, n_full].
 * ====================================================================== */
enum { SEL_COBS = 0, SEL_QUEST = 1, SEL_SUBSPACE = 2 };

/* One query head's block score s_{g,b} for selector `kind`:
 *   SEL_COBS:  qt . A_b + 1/2 sum_i (B_{b,i} . qt)^2      (A = mu, B = xi, [P5] Eq.(14)/(19);
 *              rank 0 is the mean-pool selector qt . kbar_b, [P5] Table 1)
 *   SEL_QUEST: sum_t max(qt_t A_{b,t}, qt_t B_{b,t})       (A = kmin, B = kmax, [P5] Eq.(24))
 *   SEL_SUBSPACE: qt . A_b + 1/2 sum_i (B_{b,i} . qs)^2    (B = xi in R^sd, qs = U^T qt,
 *              [P5] Eq.(18): q^T Sigma q ~ qs^T B_b qs) */
static double head_block_score(int kind, int D, int rank, int sd, const double *qt, const double *qs,
                               const double *A, const double *B)
{
    double v = 0.0;
    if (kind == SEL_QUEST) {
        for (int t = 0; t < D; ++t) {
            const double lo = qt[t] * A[t], hi = qt[t] * B[t];
            v += lo > hi ? lo : hi;
        }
        return v;
    }
    for (int t = 0; t < D; ++t)
        v += qt[t] * A[t];
    const double *qq = kind == SEL_SUBSPACE ? qs : qt;
    const int n = kind == SEL_SUBSPACE ? sd : D;
    double quad = 0.0;
    for (int e = 0; e < rank; ++e) {
        const double *x = B + (long)e * n;
        double p = 0.0;
        for (int t = 0; t < n; ++t)
            p += x[t] * qq[t];
        quad += p * p;
    }
    return v + 0.5 * quad;
}

static void block_select_run(int kind, int n_seq, int n_kv, int n_q, int D, int rank, int sd,
                             const double *U, int n_full, int L, int T, int top_blocks, int window,
                             double scale, const double *Q, const double *Ab, const double *Bb, int cap,
                             int32_t *tok, int32_t *tok_count, int32_t *blk, double *blk_score)
{
    const int G = n_q / n_kv;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)n_full);
        double *qt = (double *)malloc(sizeof(double) * (size_t)D);
        double *qs = (double *)malloc(sizeof(double) * (size_t)(sd > 0 ? sd : 1));
        scored_t *sc = (scored_t *)malloc(sizeof(scored_t) * (size_t)(n_full > 0 ? n_full : 1));
        uint8_t *mark = (uint8_t *)malloc((size_t)(T > 0 ? T : 1));
#pragma omp for collapse(2) schedule(dynamic, 1)
        for (int sq = 0; sq < n_seq; ++sq) {
            for (int h = 0; h < n_kv; ++h) {
                const long sh = (long)sq * n_kv + h;
                double *score = blk_score + sh * n_full;
                for (int b = 0; b < n_full; ++b)
                    score[b] = 0.0;
                for (int g = h * G; g < (h + 1) * G; ++g) {
                    const double *q = Q + ((long)sq * n_q + g) * D;
                    for (int t = 0; t < D; ++t)
                        qt[t] = scale * q[t];
                    if (kind == SEL_SUBSPACE)
                        for (int j = 0; j < sd; ++j) {
                            double acc = 0.0;
                            for (int t = 0; t < D; ++t)
                                acc += U[(long)t * sd + j] * qt[t];
                            qs[j] = acc;
                        }
                    double mx = -INFINITY;
                    for (int b = 0; b < n_full; ++b) {
                        const long blkid = sh * n_full + b;
                        const double *a = Ab + blkid * (long)D;
                        const double *bb = kind == SEL_QUEST      ? Bb + blkid * (long)D
                                           : kind == SEL_SUBSPACE ? Bb + blkid * (long)rank * sd
                                                                  : Bb + blkid * (long)rank * D;
                        s[b] = head_block_score(kind, D, rank, sd, qt, qs, a, bb);
                        if (s[b] > mx) mx = s[b];
                    }
                    double z = 0.0;
                    for (int b = 0; b < n_full; ++b)
                        z += exp(s[b] - mx);
                    for (int b = 0; b < n_full; ++b)
                        score[b] += exp(s[b] - mx) / z;
                }
                for (int b = 0; b < n_full; ++b) {
                    sc[b].s = score[b];
                    sc[b].i = b;
                }
                qsort(sc, (size_t)n_full, sizeof(scored_t), cmp_score_desc_idx_asc);
                const int nk = top_blocks < n_full ? top_blocks : n_full;
                int32_t *bo = blk + sh * top_blocks;
                for (int c = 0; c < nk; ++c)
                    bo[c] = sc[c].i;
                qsort(bo, (size_t)nk, sizeof(int32_t), cmp_i32);
                for (int c = nk; c < top_blocks; ++c)
                    bo[c] = -1;
                memset(mark, 0, (size_t)T);
                for (int c = 0; c < nk; ++c)
                    for (int r = 0; r < L; ++r)
                        mark[bo[c] * L + r] = 1;
                for (int p = (T - window > 0 ? T - window : 0); p < T; ++p)
                    mark[p] = 1;
                int cnt = 0;
                int32_t *to = tok + sh * cap;
                for (int p = 0; p < T; ++p)
                    if (mark[p]) {
                        if (cnt < cap) to[cnt] = p;
                        ++cnt;
                    }
                for (int c = cnt; c < cap; ++c)
                    to[c] = -1;
                tok_count[sh] = cnt;
            }
        }
        free(s);
        free(qt);
        free(qs);
        free(sc);
        free(mark);
    }
}


OAPI void oracle_block_select(int n_seq, int n_kv, int n_q, int D, int rank, int n_full, int L,
                              int T, int top_blocks, int window, double scale, const double *Q,
                              const double *mu, const double *xi, int cap, int32_t *tok,
                              int32_t *tok_count, int32_t *blk, double *blk_score)
{
    block_select_run(SEL_COBS, n_seq, n_kv, n_q, D, rank, D, NULL, n_full, L, T, top_blocks, window,
                     scale, Q, mu, xi, cap, tok, tok_count, blk, blk_score);
}

/* O6s  Subspace block selection: O6 with the quadratic term of [P5] Eq.(18),
 * (xi_i . U^T qt)^2 with xi in R^sd (from O5s).  U [D, sd]; xi [n_seq, n_kv,
 * n_full, rank, sd]; other layouts as O6. */
OAPI void oracle_block_select_ss(int n_seq, int n_kv, int n_q, int D, int sd, int rank, int n_full,
                                 int L, int T, int top_blocks, int window, double scale, const double *Q,
                                 const double *U, const double *mu, const double *xi, int cap,
                                 int32_t *tok, int32_t *tok_count, int32_t *blk, double *blk_score)
{
    block_select_run(SEL_SUBSPACE, n_seq, n_kv, n_q, D, rank, sd, U, n_full, L, T, top_blocks, window,
                     scale, Q, mu, xi, cap, tok, tok_count, blk, blk_score);
}

/* ======================================================================
 * O6q  Quest selection.  [P5] Eq.(23): per block the element-wise minimum
 * and maximum of its keys (an axis-aligned box); Eq.(24): the block's score
 * for a query is the largest inner product any point of the box reaches,
 *   s_{g,b} = sum_t max(qt_t kmin_{b,t}, qt_t kmax_{b,t}),  qt = scale * q_g.
 * Reading: the same group aggregation, top-k and window rule as O6 (the
 * pages compare the selectors inside one block-sparse pipeline, [P5] Table 1).
 * Layout: K [n_seq, T, n_kv, D]; kmin, kmax [n_seq, n_kv, n_full, D].
 * ====================================================================== */
OAPI void oracle_quest_describe(int n_seq, int T, int n_kv, int D, int L, const double *K,
                                double *kmin, double *kmax)
{
    const int n_full = T / L;
#pragma omp parallel for collapse(2) schedule(static)
    for (int sq = 0; sq < n_seq; ++sq)
        for (int h = 0; h < n_kv; ++h)
            for (int b = 0; b < n_full; ++b) {
                double *lo = kmin + (((long)sq * n_kv + h) * n_full + b) * D;
                double *hi = kmax + (((long)sq * n_kv + h) * n_full + b) * D;
                for (int t = 0; t < D; ++t) {
                    lo[t] = INFINITY;
                    hi[t] = -INFINITY;
                }
                for (int r = 0; r < L; ++r) {
                    const double *k = K + (((long)sq * T + (long)b * L + r) * n_kv + h) * D;
                    for (int t = 0; t < D; ++t) {
                        if (k[t] < lo[t]) lo[t] = k[t];
                        if (k[t] > hi[t]) hi[t] = k[t];
                    }
                }
            }
}

OAPI void oracle_quest_select(int n_seq, int n_kv, int n_q, int D, int n_full, int L, int T,
                              int top_blocks, int window, double scale, const double *Q,
                              const double *kmin, const double *kmax, int cap, int32_t *tok,
                              int32_t *tok_count, int32_t *blk, double *blk_score)
{
    block_select_run(SEL_QUEST, n_seq, n_kv, n_q, D, 0, D, NULL, n_full, L, T, top_blocks, window,
                     scale, Q, kmin, kmax, cap, tok, tok_count, blk, blk_score);
}

/* ======================================================================
 * O7  Attention over a given index set.  [P1] §1.1 Eq.(1) restricted to the
 * candidate set; [P2] §1 (the selected positions are shared by the main
 * heads); [P4] §26.2 Table 26.1 (query heads [h*G, (h+1)*G) share KV head h).
 *   O_{t,g} = sum_{j in I} softmax_j(scale * q_{t,g} . k_{j,kv(g)}) v_{j,kv(g)}
 * over the valid (>= 0) entries of the index list; an empty list gives 0 and
 * lse = -inf.  Duplicated entries are a caller error and are counted as given.
 * Masks ([P1] §1.1 Eq.(2): the allowed set P(i) is cut by the causal and the
 * padding mask before the softmax): an entry j of row t takes part only when
 * j <= q_pos[t] (q_pos NULL: no causal limit) and key_valid[kv_base[t] + j]
 * is non-zero (key_valid NULL: every key valid).
 * Layout: Q [rows, n_q, D]; K, V: token j of row t, head h at
 * ((kv_base[t] + j) * n_kv + h) * D; I [rows, n_lists, max_idx] where
 * n_lists = n_kv (a list per KV head) or 1 (one list shared by all heads).
 * ====================================================================== */
static int oracle_entry_allowed(int32_t j, long t, const int64_t *kv_base,
                                const uint8_t *key_valid, const int32_t *q_pos)
{
    if (j < 0) return 0;
    if (q_pos && j > q_pos[t]) return 0;
    if (key_valid && !key_valid[kv_base[t] + j]) return 0;
    return 1;
}

OAPI void oracle_sparse_attn(int n_rows, int n_q, int n_kv, int D, double scale, const double *Q,
                             const double *K, const double *V, const int64_t *kv_base,
                             const int32_t *I, int n_lists, int max_idx, const uint8_t *key_valid,
                             const int32_t *q_pos, double *O, double *lse)
{
    const int G = n_q / n_kv;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)(max_idx > 0 ? max_idx : 1));
#pragma omp for collapse(2) schedule(dynamic, 4)
        for (long t = 0; t < n_rows; ++t) {
            for (int g = 0; g < n_q; ++g) {
                const int h = g / G;
                const int32_t *idx = I + (t * n_lists + (n_lists == 1 ? 0 : h)) * (long)max_idx;
                const double *q = Q + (t * n_q + g) * (long)D;
                double *o = O + (t * n_q + g) * (long)D;
                for (int k = 0; k < D; ++k)
                    o[k] = 0.0;
                double mx = -INFINITY;
                for (int c = 0; c < max_idx; ++c) {
                    if (!oracle_entry_allowed(idx[c], t, kv_base, key_valid, q_pos)) continue;
                    const double *kj = K + ((kv_base[t] + idx[c]) * n_kv + h) * (long)D;
                    double dot = 0.0;
                    for (int k = 0; k < D; ++k)
                        dot += q[k] * kj[k];
                    logit[c] = scale * dot;
                    if (logit[c] > mx) mx = logit[c];
                }
                if (mx == -INFINITY) {
                    lse[t * n_q + g] = -INFINITY;
                    continue;
                }
                double z = 0.0;
                for (int c = 0; c < max_idx; ++c)
                    if (oracle_entry_allowed(idx[c], t, kv_base, key_valid, q_pos)) z += exp(logit[c] - mx);
                for (int c = 0; c < max_idx; ++c) {
                    if (!oracle_entry_allowed(idx[c], t, kv_base, key_valid, q_pos)) continue;
                    const double p = exp(logit[c] - mx) / z;
                    const double *vj = V + ((kv_base[t] + idx[c]) * n_kv + h) * (long)D;
                    for (int k = 0; k < D; ++k)
                        o[k] += p * vj[k];
                }
                lse[t * n_q + g] = mx + log(z);
            }
        }
        free(logit);
    }
}

/* ======================================================================
 * f1  Deployed descriptor compression.  [P5] §5.5 "量化：对存储的特征向量做
 * FP4": each scaled eigenvector xi_i is stored in E2M1 FP4 (2 exponent bits,
 * 1 mantissa bit) with one fp32 scale per vector; the block mean is stored
 * in bf16 (Algorithm 2 steps 7-8).  The page fixes the format but not the
 * scale rule or the rounding; the reading taken here: scale = max_d |xi_d| / 6
 * (6 is the largest E2M1 magnitude), each element x / scale rounded to the
 * nearest E2M1 value {0, 0.5, 1, 1.5, 2, 3, 4, 6}, a tie going to the value
 * with a zero mantissa bit (the even code), a zero vector getting scale 0.
 * The codes are integers decided by floating point, so the division and the
 * comparisons are taken in fp32, the kernel's precision.
 * Code: bit 3 = sign, bits 0-2 = magnitude index into the list above; two
 * codes per byte, the even element in the low nibble.
 * Layout: xi [n_vec, D] fp32 -> codes [n_vec, D/2] bytes, scale [n_vec].
 * ====================================================================== */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

static int e2m1_index(float a)   /* a = |x / scale| in fp32 */
{
    int best = 0;
    for (int i = 1; i < 8; ++i) {
        const float d_new = fabsf(a - kE2M1[i]);
        const float d_best = fabsf(a - kE2M1[best]);
        /* strictly closer wins; an exact tie goes to the even index */
        if (d_new < d_best || (d_new == d_best && (i & 1) == 0)) best = i;
    }
    return best;
}

OAPI void oracle_fp4_quantize(int n_vec, int D, const float *xi, uint8_t *codes, float *scale)
{
    for (int v = 0; v < n_vec; ++v) {
        const float *x = xi + (size_t)v * D;
        float amax = 0.0f;
        for (int d = 0; d < D; ++d) amax = fmaxf(amax, fabsf(x[d]));
        const float s = amax / 6.0f;
        scale[v] = s;
        for (int d = 0; d < D; d += 2) {
            uint8_t c[2] = {0, 0};
            for (int e = 0; e < 2; ++e) {
                if (s > 0.0f) {
                    const float y = x[d + e] / s;
                    const int idx = e2m1_index(fabsf(y));
                    c[e] = (uint8_t)(((y < 0.0f && idx != 0) ? 8 : 0) | idx);
                }
            }
            codes[(size_t)v * (D / 2) + d / 2] = (uint8_t)(c[0] | (c[1] << 4));
        }
    }
}

OAPI void oracle_fp4_dequantize(int n_vec, int D, const uint8_t *codes, const float *scale,
                                double *out)
{
    for (int v = 0; v < n_vec; ++v)
        for (int d = 0; d < D; ++d) {
            const uint8_t byte = codes[(size_t)v * (D / 2) + d / 2];
            const int c = (d & 1) ? (byte >> 4) : (byte & 15);
            const double mag = (double)kE2M1[c & 7] * (double)scale[v];
            out[(size_t)v * D + d] = (c & 8) ? -mag : mag;
        }
}
