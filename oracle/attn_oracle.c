/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for exact scaled-dot-product
 * attention, its variable-length form, the paged-KV gather and single-token
 * paged decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links or calls this
 * file; only the tests, the package smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (the plain definition, no tiling, no online update):
 *
 *   Standard attention as described on the page "Flash Attention 是什么：
 *   2026 最新原理、架构演进与实战详解" (ai.lansai.wang), section
 *   "核心工作机制": scores S = Q K^T, a softmax over each row of S, then the
 *   product with V.  The same page, section "常见误解澄清" (misconception 1),
 *   states that the fused method reaches exactly this result up to rounding,
 *   so this definition is what the GPU path is compared with.
 *
 *   For every query row i and its admissible key set A_i:
 *     s_ij  = scale * sum_k q_ik k_jk          (j in A_i)
 *     m_i   = max_j s_ij
 *     l_i   = sum_j exp(s_ij - m_i)
 *     o_i   = sum_j (exp(s_ij - m_i) / l_i) v_j
 *     lse_i = m_i + ln l_i
 *   A_i is every key (non-causal) or keys j <= i (causal, top-left aligned;
 *   the causal switch is the flash_attn_causal knob on the page
 *   "为什么“Flash”突然成了AI圈的高频词" (lqnn.cn), section 3.3).  An empty
 *   A_i gives o_i = 0 and lse_i = -inf.
 *
 * Each row of S is materialised in full (a plain array of its scores) before
 * its max, sum and output are taken; oracle_attention_probs materialises the
 * whole N x N probability matrix of one head for the small pin tests.
 *
 * Paged decode follows the page "“Flash”不是那个被时代淘汰的插件"
 * (0539edu.com), section 2: the KV cache is a pool of fixed-size pages
 * (256 tokens by default), each page a contiguous K (or V) slice, and a
 * sequence owns a list of pages.  The oracle first gathers a sequence's
 * pages back into a contiguous [len, d] array per head, then applies the
 * definition above with a single query row and no mask.  A sequence's page
 * list is read either from a packed table (sequences' lists back to back) or
 * from its own fixed-width row of a block table.
 *
 * Parallelism: OpenMP over independent output rows.  Each row is computed by
 * one thread in a fixed order, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* One output row of the definition.
 *   q      : the query row, d values
 *   kbase  : key row j (d values) starts at kbase + j * kstride
 *   vbase  : value row j (dv values) starts at vbase + j * vstride
 *   nkeys  : keys 0 .. nkeys-1 are admissible
 *   srow   : scratch for the materialised score row, >= nkeys doubles
 *   o      : dv outputs;  *lse : the row's log-sum-exp
 */
static void attention_row(const double *q, const double *kbase, int64_t kstride,
                          const double *vbase, int64_t vstride, int64_t nkeys,
                          int64_t d, int64_t dv, double scale, double *srow,
                          double *o, double *lse) {
    int64_t j, c;
    for (c = 0; c < dv; ++c) o[c] = 0.0;
    if (nkeys <= 0) {
        *lse = -INFINITY;
        return;
    }
    /* pass 1: the full score row */
    for (j = 0; j < nkeys; ++j) {
        const double *kj = kbase + j * kstride;
        double dot = 0.0;
        for (c = 0; c < d; ++c) dot += q[c] * kj[c];
        srow[j] = scale * dot;
    }
    /* pass 2: row max and normaliser */
    double m = srow[0];
    for (j = 1; j < nkeys; ++j)
        if (srow[j] > m) m = srow[j];
    double l = 0.0;
    for (j = 0; j < nkeys; ++j) l += exp(srow[j] - m);
    /* pass 3: probabilities times V */
    for (j = 0; j < nkeys; ++j) {
        const double p = exp(srow[j] - m) / l;
        const double *vj = vbase + j * vstride;
        for (c = 0; c < dv; ++c) o[c] += p * vj[c];
    }
    *lse = m + log(l);
}

/* Fixed-length attention.  q,k are [B,H,N,d] and v,o [B,H,N,dv], contiguous
 * (the layout the page "为什么“Flash”突然成了AI圈的高频词", section 2.1,
 * prints as [1, 32, 16384, 128]); lse is [B,H,N].
 * rows: optional list of nrows flat row ids r = (b*H + h)*N + i; when rows is
 * NULL every row is computed (nrows ignored).  Outputs for row r go to
 * o[r*dv ...] and lse[r] in both cases. */
int oracle_attention(const double *q, const double *k, const double *v,
                     double *o, double *lse, int64_t B, int64_t H, int64_t N,
                     int64_t d, int64_t dv, int causal, double scale,
                     const int64_t *rows, int64_t nrows) {
    if (B < 0 || H < 0 || N < 0 || d <= 0 || dv <= 0) return -1;
    const int64_t total = rows ? nrows : B * H * N;
    int failed = 0;
#pragma omp parallel
    {
        double *srow = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!srow) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < total; ++t) {
                const int64_t r = rows ? rows[t] : t;
                const int64_t bh = r / N, i = r % N;
                const double *kb = k + bh * N * d;
                const double *vb = v + bh * N * dv;
                const int64_t nk = causal ? (i + 1) : N;
                attention_row(q + r * d, kb, d, vb, dv, nk, d, dv, scale, srow,
                              o + r * dv, lse + r);
            }
            free(srow);
        }
    }
    return failed ? -2 : 0;
}

/* The full probability matrix P = softmax(scale * Q K^T) of one head, with
 * the causal mask applied (masked entries are exactly 0).  q,k are [N,d];
 * p is [N,N].  Small inputs only (pin tests). */
int oracle_attention_probs(const double *q, const double *k, double *p,
                           int64_t N, int64_t d, int causal, double scale) {
    int64_t i, j, c;
    for (i = 0; i < N; ++i) {
        double *prow = p + i * N;
        const int64_t nk = causal ? i + 1 : N;
        for (j = 0; j < N; ++j) prow[j] = 0.0;
        if (nk == 0) continue;
        for (j = 0; j < nk; ++j) {
            double dot = 0.0;
            for (c = 0; c < d; ++c) dot += q[i * d + c] * k[j * d + c];
            prow[j] = scale * dot;
        }
        double m = prow[0];
        for (j = 1; j < nk; ++j)
            if (prow[j] > m) m = prow[j];
        double l = 0.0;
        for (j = 0; j < nk; ++j) l += exp(prow[j] - m);
        for (j = 0; j < nk; ++j) prow[j] = exp(prow[j] - m) / l;
    }
    return 0;
}

/* Variable-length attention over sequences packed back to back.
 * q,k,v,o are [total,H,d] (row t of sequence b is token cu_seqlens[b] + t);
 * lse is [H,total].  Attention never crosses a sequence boundary; with
 * causal set, token t of a sequence sees tokens 0..t of the same sequence.
 * rows: optional list of flat ids r = h*total + g (g a packed token index);
 * NULL computes everything. */
int oracle_attention_varlen(const double *q, const double *k, const double *v,
                            double *o, double *lse, const int64_t *cu_seqlens,
                            int64_t B, int64_t H, int64_t d, int causal,
                            double scale, const int64_t *rows, int64_t nrows) {
    if (B < 0 || H < 0 || d <= 0) return -1;
    const int64_t totaltok = cu_seqlens[B];
    int64_t maxlen = 0;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t len = cu_seqlens[b + 1] - cu_seqlens[b];
        if (len < 0) return -1;
        if (len > maxlen) maxlen = len;
    }
    const int64_t total = rows ? nrows : H * totaltok;
    const int64_t rs = H * d; /* stride between consecutive tokens */
    int failed = 0;
#pragma omp parallel
    {
        double *srow = (double *)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);
        if (!srow || !orow) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < total; ++t) {
                const int64_t r = rows ? rows[t] : t;
                const int64_t h = r / totaltok, g = r % totaltok;
                /* the sequence that owns packed token g */
                int64_t b = 0;
                while (b + 1 <= B && cu_seqlens[b + 1] <= g) ++b;
                const int64_t start = cu_seqlens[b];
                const int64_t len = cu_seqlens[b + 1] - start;
                const int64_t i = g - start;
                const int64_t nk = causal ? i + 1 : len;
                double l;
                attention_row(q + g * rs + h * d, k + start * rs + h * d, rs,
                              v + start * rs + h * d, rs, nk, d, d, scale, srow,
                              orow, &l);
                for (int64_t c = 0; c < d; ++c) o[g * rs + h * d + c] = orow[c];
                lse[h * totaltok + g] = l;
            }
        }
        free(srow);
        free(orow);
    }
    return failed ? -2 : 0;
}

/* Gather of a paged KV cache back into contiguous rows.
 *   pages      : [P_pool, H, page_size, d]  (one contiguous slice per page
 *                and head)
 *   page_table : the pages of every sequence, packed: sequence b's pages are
 *                entries off_b .. off_b + npages_b - 1, where npages_b is the
 *                number of page_size-token pages its seq_lens[b] tokens
 *                occupy and off_b is the sum of npages over earlier
 *                sequences
 *   out        : [sum_b seq_lens[b], H, d], sequence b starting at row
 *                sum_{b'<b} seq_lens[b']
 * Token t of sequence b lives in page table entry off_b + floor(t/page_size),
 * at slot t mod page_size of that page. */
int oracle_gather_paged(const double *pages, const int64_t *page_table,
                        const int64_t *seq_lens, double *out, int64_t B,
                        int64_t H, int64_t d, int64_t page_size) {
    if (page_size <= 0 || d <= 0 || H < 0 || B < 0) return -1;
    int64_t off = 0, row = 0;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t len = seq_lens[b];
        if (len < 0) return -1;
        for (int64_t t = 0; t < len; ++t) {
            const int64_t page = page_table[off + t / page_size];
            const int64_t slot = t % page_size;
            for (int64_t h = 0; h < H; ++h) {
                const double *src = pages + ((page * H + h) * page_size + slot) * d;
                double *dst = out + ((row + t) * H + h) * d;
                for (int64_t c = 0; c < d; ++c) dst[c] = src[c];
            }
        }
        off += (len + page_size - 1) / page_size;
        row += len;
    }
    return 0;
}

/* Single-token decode over the paged cache: for each sequence b and head h,
 * the query q[b,h,:] attends (no mask) to all seq_lens[b] cached tokens.
 * q, o are [B,H,d]; lse (optional, may be NULL) is [B,H]. */
int oracle_decode_paged(const double *q, const double *k_pages,
                        const double *v_pages, const int64_t *page_table,
                        const int64_t *seq_lens, double *o, double *lse,
                        int64_t B, int64_t H, int64_t d, int64_t page_size) {
    if (page_size <= 0 || d <= 0 || H < 0 || B < 0) return -1;
    int64_t off = 0;
    int rc = 0;
    for (int64_t b = 0; b < B && rc == 0; ++b) {
        const int64_t len = seq_lens[b];
        if (len < 0) return -1;
        const int64_t np = (len + page_size - 1) / page_size;
        double *kc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * H * d));
        double *vc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * H * d));
        if (!kc || !vc) {
            free(kc);
            free(vc);
            return -2;
        }
        /* this sequence alone, as a one-sequence packed table */
        oracle_gather_paged(k_pages, page_table + off, &len, kc, 1, H, d, page_size);
        oracle_gather_paged(v_pages, page_table + off, &len, vc, 1, H, d, page_size);
        int failed = 0;
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
            if (!srow) {
#pragma omp atomic write
                failed = 1;
            } else {
#pragma omp for schedule(static)
                for (int64_t h = 0; h < H; ++h) {
                    double l;
                    attention_row(q + (b * H + h) * d, kc + h * d, H * d, vc + h * d,
                                  H * d, len, d, d, 1.0 / sqrt((double)d), srow,
                                  o + (b * H + h) * d, &l);
                    if (lse) lse[b * H + h] = l;
                }
                free(srow);
            }
        }
        if (failed) rc = -2;
        free(kc);
        free(vc);
        off += np;
    }
    return rc;
}

/* Grouped-query attention (multi-query when Hkv = 1): H query heads share
 * Hkv key/value heads, query head h reading K/V head h / (H / Hkv) (integer
 * division), the variant the page "Flash Attention 是什么" names in its
 * section 进阶学习路径 (item 4).  q is [B,H,N,d], k is [B,Hkv,N,d], v is
 * [B,Hkv,N,dv], o is [B,H,N,dv], lse is [B,H,N]; the definition per row is
 * the one above.  rows: optional flat query row ids (b*H + h)*N + i. */
int oracle_attention_gqa(const double *q, const double *k, const double *v,
                         double *o, double *lse, int64_t B, int64_t H, int64_t Hkv,
                         int64_t N, int64_t d, int64_t dv, int causal, double scale,
                         const int64_t *rows, int64_t nrows) {
    if (B < 0 || H < 0 || N < 0 || d <= 0 || dv <= 0 || Hkv <= 0 || H % Hkv != 0) return -1;
    const int64_t group = H / Hkv;
    const int64_t total = rows ? nrows : B * H * N;
    int failed = 0;
#pragma omp parallel
    {
        double *srow = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!srow) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < total; ++t) {
                const int64_t r = rows ? rows[t] : t;
                const int64_t bh = r / N, i = r % N;
                const int64_t b = bh / H, h = bh % H;
                const int64_t g = h / group;
                const double *kb = k + (b * Hkv + g) * N * d;
                const double *vb = v + (b * Hkv + g) * N * dv;
                const int64_t nk = causal ? (i + 1) : N;
                attention_row(q + r * d, kb, d, vb, dv, nk, d, dv, scale, srow,
                              o + r * dv, lse + r);
            }
            free(srow);
        }
    }
    return failed ? -2 : 0;
}

/* Single-token decode with grouped K/V heads: q, o are [B,H,d]; the pages
 * are [P_pool, Hkv, page_size, d]; query head h of sequence b attends to K/V
 * head h / (H / Hkv) of its cached tokens.  lse (optional) is [B,H]. */
int oracle_decode_paged_gqa(const double *q, const double *k_pages,
                            const double *v_pages, const int64_t *page_table,
                            const int64_t *seq_lens, double *o, double *lse,
                            int64_t B, int64_t H, int64_t Hkv, int64_t d,
                            int64_t page_size) {
    if (page_size <= 0 || d <= 0 || H < 0 || B < 0 || Hkv <= 0 || H % Hkv != 0) return -1;
    const int64_t group = H / Hkv;
    int64_t off = 0;
    int rc = 0;
    for (int64_t b = 0; b < B && rc == 0; ++b) {
        const int64_t len = seq_lens[b];
        if (len < 0) return -1;
        const int64_t np = (len + page_size - 1) / page_size;
        double *kc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * Hkv * d));
        double *vc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * Hkv * d));
        if (!kc || !vc) {
            free(kc);
            free(vc);
            return -2;
        }
        oracle_gather_paged(k_pages, page_table + off, &len, kc, 1, Hkv, d, page_size);
        oracle_gather_paged(v_pages, page_table + off, &len, vc, 1, Hkv, d, page_size);
        int failed = 0;
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
            if (!srow) {
#pragma omp atomic write
                failed = 1;
            } else {
#pragma omp for schedule(static)
                for (int64_t h = 0; h < H; ++h) {
                    const int64_t g = h / group;
                    double l;
                    attention_row(q + (b * H + h) * d, kc + g * d, Hkv * d, vc + g * d,
                                  Hkv * d, len, d, d, 1.0 / sqrt((double)d), srow,
                                  o + (b * H + h) * d, &l);
                    if (lse) lse[b * H + h] = l;
                }
                free(srow);
            }
        }
        if (failed) rc = -2;
        free(kc);
        free(vc);
        off += np;
    }
    return rc;
}

/* Single-token decode through a block table: one row of max_pages entries
 * per sequence, sequence b's k-th page being block_table[b * max_pages + k]
 * (the "page table per sequence" of the paged cache on the page
 * "“Flash”不是那个被时代淘汰的插件", 0539edu.com, section 2, kept as a
 * fixed-width row; entries past a sequence's pages are not read).  q, o are
 * [B,H,d], the pages [P_pool, Hkv, page_size, d]; query head h of sequence b
 * attends to K/V head h / (H / Hkv) of its seq_lens[b] cached tokens, which
 * must fit its row (seq_lens[b] <= max_pages * page_size).  lse (optional)
 * is [B,H]. */
int oracle_decode_paged_strided(const double *q, const double *k_pages,
                                const double *v_pages, const int64_t *block_table,
                                int64_t max_pages, const int64_t *seq_lens, double *o,
                                double *lse, int64_t B, int64_t H, int64_t Hkv, int64_t d,
                                int64_t page_size) {
    if (page_size <= 0 || d <= 0 || H < 0 || B < 0 || Hkv <= 0 || H % Hkv != 0 ||
        max_pages < 0)
        return -1;
    const int64_t group = H / Hkv;
    int rc = 0;
    for (int64_t b = 0; b < B && rc == 0; ++b) {
        const int64_t len = seq_lens[b];
        if (len < 0 || len > max_pages * page_size) return -1;
        double *kc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * Hkv * d));
        double *vc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * Hkv * d));
        if (!kc || !vc) {
            free(kc);
            free(vc);
            return -2;
        }
        /* the sequence's row is a one-sequence packed table */
        oracle_gather_paged(k_pages, block_table + b * max_pages, &len, kc, 1, Hkv, d, page_size);
        oracle_gather_paged(v_pages, block_table + b * max_pages, &len, vc, 1, Hkv, d, page_size);
        int failed = 0;
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
            if (!srow) {
#pragma omp atomic write
                failed = 1;
            } else {
#pragma omp for schedule(static)
                for (int64_t h = 0; h < H; ++h) {
                    const int64_t g = h / group;
                    double l;
                    attention_row(q + (b * H + h) * d, kc + g * d, Hkv * d, vc + g * d,
                                  Hkv * d, len, d, d, 1.0 / sqrt((double)d), srow,
                                  o + (b * H + h) * d, &l);
                    if (lse) lse[b * H + h] = l;
                }
                free(srow);
            }
        }
        if (failed) rc = -2;
        free(kc);
        free(vc);
    }
    return rc;
}

/* Appending new tokens to the paged cache, the step before decode in the
 * serving loop of the page "“Flash”不是那个被时代淘汰的插件" (0539edu.com),
 * section 2: a new token's K (or V) row is written into the page that holds
 * its position.  Sequence b holds seq_lens[b] tokens AFTER the append; its
 * n_b = cu_new[b+1] - cu_new[b] new tokens are its last n_b positions
 * (pos = seq_lens[b] - n_b + i for new token i), and the packed page table
 * already lists every page those positions need.  pages is [P, Hkv, page_size,
 * d] and is updated in place; new_rows is [cu_new[B], Hkv, d]. */
int oracle_append_paged(double *pages, const int64_t *page_table, const int64_t *seq_lens,
                        const double *new_rows, const int64_t *cu_new, int64_t B,
                        int64_t Hkv, int64_t d, int64_t page_size) {
    if (page_size <= 0 || d <= 0 || Hkv <= 0 || B < 0) return -1;
    int64_t off = 0;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t len = seq_lens[b];
        const int64_t n = cu_new[b + 1] - cu_new[b];
        if (len < 0 || n < 0 || n > len) return -1;
        for (int64_t i = 0; i < n; ++i) {
            const int64_t pos = len - n + i;
            const int64_t page = page_table[off + pos / page_size];
            const int64_t slot = pos % page_size;
            for (int64_t h = 0; h < Hkv; ++h) {
                const double *src = new_rows + ((cu_new[b] + i) * Hkv + h) * d;
                double *dst = pages + ((page * Hkv + h) * page_size + slot) * d;
                for (int64_t c = 0; c < d; ++c) dst[c] = src[c];
            }
        }
        off += (len + page_size - 1) / page_size;
    }
    return 0;
}

/* Prefill over the paged cache (decode with several query tokens): sequence
 * b caches seq_lens[b] tokens, the last q_b = cu_q[b+1] - cu_q[b] of which are
 * its new query tokens.  Query i of sequence b sits at position
 * seq_lens[b] - q_b + i and, with causal set, sees the keys at positions up to
 * its own (the mask aligned to the end of the sequence); without it, all
 * seq_lens[b] keys.  q, o are [cu_q[B], H, d]; lse is [H, cu_q[B]]; the pages
 * are [P, Hkv, page_size, d] with query head h reading K/V head h / (H/Hkv).
 * The sequence's K/V are gathered first, then the definition applies. */
int oracle_prefill_paged(const double *q, const double *k_pages, const double *v_pages,
                         const int64_t *page_table, const int64_t *seq_lens,
                         const int64_t *cu_q, double *o, double *lse, int64_t B, int64_t H,
                         int64_t Hkv, int64_t d, int64_t page_size, int causal, double scale) {
    if (page_size <= 0 || d <= 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0 || B < 0) return -1;
    const int64_t group = H / Hkv;
    const int64_t total_q = cu_q[B];
    int64_t off = 0;
    int rc = 0;
    for (int64_t b = 0; b < B && rc == 0; ++b) {
        const int64_t len = seq_lens[b];
        const int64_t nq = cu_q[b + 1] - cu_q[b];
        if (len < 0 || nq < 0 || nq > len) return -1;
        double *kc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * Hkv * d));
        double *vc = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * Hkv * d));
        if (!kc || !vc) {
            free(kc);
            free(vc);
            return -2;
        }
        oracle_gather_paged(k_pages, page_table + off, &len, kc, 1, Hkv, d, page_size);
        oracle_gather_paged(v_pages, page_table + off, &len, vc, 1, Hkv, d, page_size);
        int failed = 0;
#pragma omp parallel
        {
            double *srow = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
            if (!srow) {
#pragma omp atomic write
                failed = 1;
            } else {
#pragma omp for schedule(dynamic, 4)
                for (int64_t t = 0; t < nq * H; ++t) {
                    const int64_t i = t / H, h = t % H;
                    const int64_t g = h / group;
                    const int64_t row = cu_q[b] + i;
                    const int64_t nk = causal ? (len - nq + i + 1) : len;
                    double l;
                    attention_row(q + (row * H + h) * d, kc + g * d, Hkv * d, vc + g * d,
                                  Hkv * d, nk, d, d, scale, srow, o + (row * H + h) * d, &l);
                    lse[h * total_q + row] = l;
                }
                free(srow);
            }
        }
        if (failed) rc = -2;
        free(kc);
        free(vc);
        off += (len + page_size - 1) / page_size;
    }
    return rc;
}

/* Rotary position embedding, applied to q and k before the scores (the page
 * "“Flash”不是那个被时代淘汰的插件" (0539edu.com), section 2 -- the kernel
 * fuses RoPE -- and section 3 -- from a precomputed sin/cos lookup table).
 * Rotate-half pairing: for position p and i < d/2 the pair (x_i, x_{i+d/2})
 * is rotated by the angle whose cosine and sine are cos_t[p*(d/2) + i],
 * sin_t[p*(d/2) + i]:
 *     x'_i       = x_i cos - x_{i+d/2} sin
 *     x'_{i+d/2} = x_{i+d/2} cos + x_i sin
 * x is [rows, N, d] (row r, position n at x + (r*N + n)*d), rotated in place.
 * oracle_rope_exact computes in fp64.  oracle_rope_bf16 is the rotation as
 * the attention then consumes it: the rotated q and k are inputs of bf16
 * tensor-core products, so each rotated value is the fp64 rotation (of the
 * fp32 table entries) rounded once to the nearest bf16, ties to even.  It
 * depends on no order of fp32 operations: any implementation that rotates in
 * higher precision and rounds once gets these values, and one that rotates
 * in fp32 differs from them only where its fp32 rounding error crosses a bf16
 * rounding boundary (a rare one-ulp difference). */
void oracle_rope_exact(double *x, const float *cos_t, const float *sin_t, int64_t rows,
                       int64_t N, int64_t d) {
    const int64_t half = d / 2;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t n = 0; n < N; ++n) {
            double *v = x + (r * N + n) * d;
            for (int64_t i = 0; i < half; ++i) {
                const double c = cos_t[n * half + i], sn = sin_t[n * half + i];
                const double a = v[i], b = v[i + half];
                v[i] = a * c - b * sn;
                v[i + half] = b * c + a * sn;
            }
        }
}

/* Round a double to the nearest bf16 value (8 significant bits, the fp32
 * exponent range), ties to even, in one step (no intermediate fp32 value, so
 * no double rounding). */
static double rne_bf16(double x) {
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    int e;
    frexp(x, &e);                 /* |x| = m 2^e, 1/2 <= m < 1 */
    int qe = e - 8;               /* weight of the last of 8 significant bits */
    if (qe < -133) qe = -133;     /* bf16 subnormals: quantum 2^-133 */
    const double r = ldexp(nearbyint(ldexp(x, -qe)), qe); /* default mode: ties to even */
    if (fabs(r) >= 0x1p128) return x > 0 ? INFINITY : -INFINITY;
    return r;
}

void oracle_rope_bf16(double *x, const float *cos_t, const float *sin_t, int64_t rows,
                      int64_t N, int64_t d) {
    oracle_rope_exact(x, cos_t, sin_t, rows, N, d);
    const int64_t n = rows * N * d;
    for (int64_t i = 0; i < n; ++i) x[i] = rne_bf16(x[i]);
}

/* Gradients of the attention of one problem with respect to q, k and v,
 * given the output gradient do -- the backward pass the saved row statistics
 * serve (page "Flash Attention 是什么", section 核心工作机制, recomputation
 * paragraph: the max and sum kept from the forward pass let the backward pass
 * rebuild the scores instead of storing them).  The oracle recomputes
 * everything from q, k, v: for each (b, h) and row i,
 *   p_ij  = exp(s_ij - lse_i),  s_ij = scale q_i.k_j  (j admissible)
 *   dV_j += p_ij do_i
 *   dp_ij = do_i . v_j
 *   D_i   = sum_j p_ij dp_ij        (= do_i . o_i)
 *   ds_ij = p_ij (dp_ij - D_i)
 *   dQ_i  = scale sum_j ds_ij k_j
 *   dK_j += scale ds_ij q_i
 * q, do, dq are [B,H,N,d]; k, v, dk, dv are [B,Hkv,N,d] and query head h
 * uses K/V head h / (H / Hkv) (grouped-query attention; Hkv = H is plain
 * multi-head), so a K/V head's dK and dV are the sums of the contributions of
 * every query head of its group.  Rows are split over threads; each thread
 * accumulates dK, dV of its rows privately and the partial sums are added in
 * thread order (query heads in order), so the result does not depend on
 * scheduling for a fixed thread count. */
int oracle_attention_bwd(const double *q, const double *k, const double *v, const double *dout,
                         double *dq, double *dk, double *dv, int64_t B, int64_t H, int64_t Hkv,
                         int64_t N, int64_t d, int causal, double scale) {
    if (B < 0 || H < 0 || N < 0 || d <= 0 || Hkv <= 0 || H % Hkv != 0) return -1;
    const int64_t group = H / Hkv;
    for (int64_t x = 0; x < B * Hkv * N * d; ++x) dk[x] = dv[x] = 0.0;
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t bkv = (bh / H) * Hkv + (bh % H) / group;
        const double *qb = q + bh * N * d, *kb = k + bkv * N * d, *vb = v + bkv * N * d;
        const double *gb = dout + bh * N * d;
        double *dqb = dq + bh * N * d, *dkb = dk + bkv * N * d, *dvb = dv + bkv * N * d;
        int nthr = 1;
#ifdef _OPENMP
        nthr = omp_get_max_threads();
#endif
        double *acc = (double *)calloc((size_t)nthr * 2 * (size_t)(N * d), sizeof(double));
        if (!acc) return -2;
        int failed = 0;
#pragma omp parallel
        {
            int tid = 0;
#ifdef _OPENMP
            tid = omp_get_thread_num();
#endif
            double *tdk = acc + (size_t)tid * 2 * (size_t)(N * d), *tdv = tdk + N * d;
            double *srow = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
            double *prow = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
            if (!srow || !prow) {
#pragma omp atomic write
                failed = 1;
            } else {
#pragma omp for schedule(static)
                for (int64_t i = 0; i < N; ++i) {
                    const int64_t nk = causal ? i + 1 : N;
                    const double *qi = qb + i * d, *gi = gb + i * d;
                    double m = -INFINITY;
                    for (int64_t j = 0; j < nk; ++j) {
                        double dot = 0.0;
                        for (int64_t c = 0; c < d; ++c) dot += qi[c] * kb[j * d + c];
                        srow[j] = scale * dot;
                        if (srow[j] > m) m = srow[j];
                    }
                    double l = 0.0;
                    for (int64_t j = 0; j < nk; ++j) l += exp(srow[j] - m);
                    const double lse = m + log(l);
                    double Di = 0.0;
                    for (int64_t j = 0; j < nk; ++j) {
                        prow[j] = exp(srow[j] - lse);
                        double dp = 0.0;
                        for (int64_t c = 0; c < d; ++c) dp += gi[c] * vb[j * d + c];
                        srow[j] = dp; /* srow now holds dp_ij */
                        Di += prow[j] * dp;
                    }
                    double *dqi = dqb + i * d;
                    for (int64_t c = 0; c < d; ++c) dqi[c] = 0.0;
                    for (int64_t j = 0; j < nk; ++j) {
                        const double ds = prow[j] * (srow[j] - Di);
                        for (int64_t c = 0; c < d; ++c) {
                            dqi[c] += scale * ds * kb[j * d + c];
                            tdk[j * d + c] += scale * ds * qi[c];
                            tdv[j * d + c] += prow[j] * gi[c];
                        }
                    }
                }
            }
            free(srow);
            free(prow);
        }
        for (int t = 0; t < nthr; ++t) {
            const double *tdk = acc + (size_t)t * 2 * (size_t)(N * d), *tdv = tdk + N * d;
            for (int64_t x = 0; x < N * d; ++x) {
                dkb[x] += tdk[x];
                dvb[x] += tdv[x];
            }
        }
        free(acc);
        if (failed) return -2;
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
