/*
 * Exact attention oracle: plain, slow, fp64 CPU implementation of
 *
 *     O = softmax(Q K^T * scale + mask) V,   LSE_i = ln sum_{visible j} exp(scale * q_i . k_j)
 *
 * and of its backward pass (dQ, dK, dV for a given dO; oracle_attn_bwd at the end).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library.  It shares no code, header or constant with the CUDA
 * library and includes no CUDA header.
 *
 * What it follows:
 *  - "Chapter 3.1 - The Cost of Attention" (llmis.ru), section 2: Q, K, V of shape (n, d),
 *    output softmax(Q K^T / sqrt(d)) V.  The caller passes the scale (1/sqrt(d) in every
 *    workload) so scale = 0 and other finite values can be checked too.
 *  - Same page, section 5: the tiled method must give this exact result, so the oracle is the
 *    definition written out with no tiling, no blocking and no online softmax: for each query
 *    row it materialises the full row of scores over all Nk keys, masks it, takes the
 *    max-subtracted softmax and forms P V.
 *  - Masks: sliding window of w neighbouring tokens ("Quadratic Complexity Bottleneck",
 *    sparse attention and sliding window sections; "Attention Research", section 4), read as
 *    the causal left window of w keys including the diagonal; always-visible sink tokens
 *    ("Attention Research", section 4), read as key positions 0..n_sink-1, still causal.
 *  - Local + global (Longformer; "Chapter 3.1 - The Cost of Attention", section 3: a window of
 *    neighbours on either side plus a few global tokens that attend to, and are attended by,
 *    every token; "Quadratic Complexity Bottleneck", sliding window: W tokens to the left and
 *    right): not causal; key j is visible to position p iff |p - j| <= w, or j is a global
 *    token, or p is one.  The global tokens are positions 0..n_global-1 (n_global is passed in
 *    n_sink); a query row is global iff 0 <= p < n_global.
 *  - GQA ("Quadratic Complexity Bottleneck", grouped-query attention): query heads are
 *    partitioned into Hkv contiguous groups of G = Hq / Hkv; query head h reads kv head h / G.
 *  - Causal alignment when Nq != Nk (the pages are silent): bottom-right, query row i sits at
 *    key position p_i = i + Nk - Nq, so a one-token decode equals the last prefill row.
 *  - A row with no visible key gets O = 0 and LSE = -inf.
 *
 * Layouts (row-major, d innermost): Q, O [B][Hq][Nq][d]; K, V [B][Hkv][Nk][d]; LSE [B][Hq][Nq].
 * Parallelism: OpenMP over independent query rows; each row's arithmetic is sequential.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MASK_FULL 0
#define ORACLE_MASK_CAUSAL 1
#define ORACLE_MASK_SLIDING 2
#define ORACLE_MASK_LOCAL_GLOBAL 3

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Visibility of key j to the query at absolute key position p (see header comment). */
int oracle_visible(int64_t p, int64_t j, int mask_kind, int64_t window, int64_t n_sink) {
    if (mask_kind == ORACLE_MASK_FULL) return 1;
    if (mask_kind == ORACLE_MASK_LOCAL_GLOBAL) {
        if (j < n_sink) return 1;            /* global key */
        if (p >= 0 && p < n_sink) return 1;  /* global query */
        return j >= p - window && j <= p + window;
    }
    if (j > p) return 0; /* causal */
    if (mask_kind == ORACLE_MASK_CAUSAL) return 1;
    if (j > p - window) return 1; /* inside the window: p - w < j <= p */
    if (j < n_sink) return 1;     /* sink tokens */
    return 0;
}

static int check_args(int B, int Hq, int Hkv, int Nq, int Nk, int d, int mask_kind, int window,
                      int n_sink) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 0 || Nk < 0 || d < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    if (mask_kind < 0 || mask_kind > 3) return -1;
    if (mask_kind == ORACLE_MASK_SLIDING && window < 1) return -1;
    if (mask_kind == ORACLE_MASK_LOCAL_GLOBAL && window < 0) return -1;
    if (n_sink < 0) return -1;
    return 0;
}

/*
 * One query row: scores over every key, mask, softmax, P V.
 * s and vis are caller-provided scratch of Nk entries each.  kblocks, when not NULL, is the
 * row's entry of a block-sparse layout (one byte per block of block_k keys): a key is visible
 * only if its block is selected as well.
 */
static void attend_row(const double *q, const double *K, const double *V, int Nk, int d,
                       int64_t p, int mask_kind, int window, int n_sink, double scale,
                       const unsigned char *kblocks, int block_k,
                       double *s, unsigned char *vis, double *o, double *lse) {
    int64_t j;
    int t;
    int any = 0;
    double m = -INFINITY, l = 0.0;
    /* 1. the full row of scores s_j = scale * q . k_j */
    for (j = 0; j < Nk; ++j) {
        double acc = 0.0;
        for (t = 0; t < d; ++t) acc += q[t] * K[j * (int64_t)d + t];
        s[j] = scale * acc;
        vis[j] = (unsigned char)(oracle_visible(p, j, mask_kind, window, n_sink) &&
                                 (kblocks == NULL || kblocks[j / block_k] != 0));
        if (vis[j]) {
            if (!any || s[j] > m) m = s[j];
            any = 1;
        }
    }
    for (t = 0; t < d; ++t) o[t] = 0.0;
    if (!any) {
        *lse = -INFINITY;
        return;
    }
    /* 2. max-subtracted exponentials and their sum */
    for (j = 0; j < Nk; ++j) {
        s[j] = vis[j] ? exp(s[j] - m) : 0.0;
        l += s[j];
    }
    /* 3. O = P V with P = e / l */
    for (j = 0; j < Nk; ++j) {
        if (!vis[j]) continue;
        double pj = s[j] / l;
        for (t = 0; t < d; ++t) o[t] += pj * V[j * (int64_t)d + t];
    }
    *lse = m + log(l);
}

/* Full forward: every row of every (b, h). Returns 0, or -1 on invalid arguments. */
int oracle_attn(const double *q, const double *k, const double *v, double *o, double *lse, int B,
                int Hq, int Hkv, int Nq, int Nk, int d, int mask_kind, int window, int n_sink,
                double scale) {
    if (check_args(B, Hq, Hkv, Nq, Nk, d, mask_kind, window, n_sink)) return -1;
    const int G = Hq / Hkv;
    const int64_t rows = (int64_t)B * Hq * Nq;
    int failed = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        unsigned char *vis = (unsigned char *)malloc((size_t)(Nk > 0 ? Nk : 1));
        if (!s || !vis) {
#pragma omp atomic write
            failed = 1;
        } else {
            int64_t r;
#pragma omp for schedule(dynamic, 16)
            for (r = 0; r < rows; ++r) {
                int64_t i = r % Nq;
                int64_t bh = r / Nq;
                int64_t h = bh % Hq, b = bh / Hq;
                int64_t hk = h / G;
                const double *Kb = k + ((b * Hkv + hk) * (int64_t)Nk) * d;
                const double *Vb = v + ((b * Hkv + hk) * (int64_t)Nk) * d;
                double l_out;
                attend_row(q + r * d, Kb, Vb, Nk, d, i + (int64_t)Nk - Nq, mask_kind, window,
                           n_sink, scale, NULL, 1, s, vis, o + r * d, &l_out);
                if (lse) lse[r] = l_out;
            }
        }
        free(s);
        free(vis);
    }
    return failed ? -2 : 0;
}

/*
 * Selected rows only.  rows[] holds flat row indices r = (b * Hq + h) * Nq + i; the results go
 * to o_rows[n_rows][d] and lse_rows[n_rows].  Same arithmetic as oracle_attn, row by row.
 */
int oracle_attn_rows(const double *q, const double *k, const double *v, int B, int Hq, int Hkv,
                     int Nq, int Nk, int d, int mask_kind, int window, int n_sink, double scale,
                     const int64_t *rows, int64_t n_rows, double *o_rows, double *lse_rows) {
    if (check_args(B, Hq, Hkv, Nq, Nk, d, mask_kind, window, n_sink)) return -1;
    const int G = Hq / Hkv;
    const int64_t total = (int64_t)B * Hq * Nq;
    int64_t n;
    for (n = 0; n < n_rows; ++n)
        if (rows[n] < 0 || rows[n] >= total) return -1;
    int failed = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        unsigned char *vis = (unsigned char *)malloc((size_t)(Nk > 0 ? Nk : 1));
        if (!s || !vis) {
#pragma omp atomic write
            failed = 1;
        } else {
            int64_t t;
#pragma omp for schedule(dynamic, 1)
            for (t = 0; t < n_rows; ++t) {
                int64_t r = rows[t];
                int64_t i = r % Nq;
                int64_t bh = r / Nq;
                int64_t h = bh % Hq, b = bh / Hq;
                int64_t hk = h / G;
                const double *Kb = k + ((b * Hkv + hk) * (int64_t)Nk) * d;
                const double *Vb = v + ((b * Hkv + hk) * (int64_t)Nk) * d;
                attend_row(q + r * d, Kb, Vb, Nk, d, i + (int64_t)Nk - Nq, mask_kind, window,
                           n_sink, scale, NULL, 1, s, vis, o_rows + t * d, &lse_rows[t]);
            }
        }
        free(s);
        free(vis);
    }
    return failed ? -2 : 0;
}

/*
 * Block-sparse forward ("Quadratic Complexity Bottleneck", sparse attention patterns: the
 * sequence is cut into blocks and attention is computed within and between selected blocks).
 * The selection is fixed and given by the caller: block_mask[hm][i / block_q][j / block_k]
 * != 0 selects the block of query rows and keys that holds row i and key j, with
 * hm = h when mask_heads == Hq (one layout per query head) and hm = 0 when mask_heads == 1 (one
 * layout for every head); layout [mask_heads][ceil(Nq / block_q)][ceil(Nk / block_k)] bytes,
 * shared by the batch.  Blocks are cut on row indices i and key indices j.  A key is visible
 * iff its block is selected and the base mask (mask_kind, window, n_sink) admits it; the rest
 * is oracle_attn.  Returns 0, or -1 on invalid arguments.
 */
int oracle_attn_block_sparse(const double *q, const double *k, const double *v, double *o,
                             double *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             int mask_kind, int window, int n_sink, double scale,
                             const unsigned char *block_mask, int mask_heads, int block_q,
                             int block_k) {
    if (check_args(B, Hq, Hkv, Nq, Nk, d, mask_kind, window, n_sink)) return -1;
    if (block_q < 1 || block_k < 1 || (mask_heads != 1 && mask_heads != Hq)) return -1;
    if (block_mask == NULL && Nq > 0 && Nk > 0) return -1;
    const int G = Hq / Hkv;
    const int64_t nqb = ((int64_t)Nq + block_q - 1) / block_q;
    const int64_t nkb = ((int64_t)Nk + block_k - 1) / block_k;
    const int64_t rows = (int64_t)B * Hq * Nq;
    int failed = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        unsigned char *vis = (unsigned char *)malloc((size_t)(Nk > 0 ? Nk : 1));
        if (!s || !vis) {
#pragma omp atomic write
            failed = 1;
        } else {
            int64_t r;
#pragma omp for schedule(dynamic, 16)
            for (r = 0; r < rows; ++r) {
                int64_t i = r % Nq;
                int64_t bh = r / Nq;
                int64_t h = bh % Hq, b = bh / Hq;
                int64_t hk = h / G;
                int64_t hm = mask_heads == 1 ? 0 : h;
                const double *Kb = k + ((b * Hkv + hk) * (int64_t)Nk) * d;
                const double *Vb = v + ((b * Hkv + hk) * (int64_t)Nk) * d;
                const unsigned char *row_blocks = block_mask + (hm * nqb + i / block_q) * nkb;
                double l_out;
                attend_row(q + r * d, Kb, Vb, Nk, d, i + (int64_t)Nk - Nq, mask_kind, window,
                           n_sink, scale, row_blocks, block_k, s, vis, o + r * d, &l_out);
                if (lse) lse[r] = l_out;
            }
        }
        free(s);
        free(vis);
    }
    return failed ? -2 : 0;
}

/* Number of visible (query, key) pairs of one (b, h) slice: the pair count behind FLOP totals. */
int64_t oracle_visible_pairs(int Nq, int Nk, int mask_kind, int window, int n_sink) {
    int64_t i, j, c = 0;
    for (i = 0; i < Nq; ++i)
        for (j = 0; j < Nk; ++j)
            c += oracle_visible(i + (int64_t)Nk - Nq, j, mask_kind, window, n_sink);
    return c;
}

/*
 * Backward pass: gradients of a scalar loss L through O = softmax(Q K^T * scale + mask) V,
 * given dO = dL/dO.  Written from the chain rule of the definition above (the pages name the
 * backward pass and its recomputation of attention, "Quadratic Complexity Bottleneck",
 * FlashAttention section, and "Chapter 3.1 - The Cost of Attention", section 5, but print no
 * formula for it):
 *
 *     P_ij  = exp(scale * q_i . k_j - LSE_i) on visible pairs, 0 elsewhere
 *     dV_j  = sum_i P_ij dO_i
 *     dP_ij = dO_i . v_j
 *     D_i   = sum_j P_ij dP_ij
 *     dS_ij = P_ij (dP_ij - D_i)
 *     dQ_i  = scale * sum_j dS_ij k_j          dK_j = scale * sum_i dS_ij q_i
 *
 * With GQA the kv head's gradients sum over the G query heads that read it.  Rows with no
 * visible key contribute nothing.  Two plain passes, each parallel over independent rows:
 * pass 1 (query rows) forms the whole score row, LSE_i, D_i and dQ_i; pass 2 (key rows)
 * forms column j of P and dS for every query row of every head of the group and sums dK_j,
 * dV_j.  No tiling, no blocking.
 *
 * Layouts as the forward: Q, dO, dQ [B][Hq][Nq][d]; K, V, dK, dV [B][Hkv][Nk][d].
 */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                    double *dq, double *dk, double *dv, int B, int Hq, int Hkv, int Nq, int Nk,
                    int d, int mask_kind, int window, int n_sink, double scale) {
    if (check_args(B, Hq, Hkv, Nq, Nk, d, mask_kind, window, n_sink)) return -1;
    const int G = Hq / Hkv;
    const int64_t rows = (int64_t)B * Hq * Nq;
    const int64_t krows = (int64_t)B * Hkv * Nk;
    double *lse = (double *)malloc(sizeof(double) * (size_t)(rows > 0 ? rows : 1));
    double *Dv = (double *)malloc(sizeof(double) * (size_t)(rows > 0 ? rows : 1));
    int failed = (lse == NULL || Dv == NULL);
    if (!failed) {
        /* ---- pass 1: per query row, LSE_i, D_i and dQ_i ---- */
#pragma omp parallel
        {
            double *s = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
            double *dp = (double *)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
            unsigned char *vis = (unsigned char *)malloc((size_t)(Nk > 0 ? Nk : 1));
            if (!s || !dp || !vis) {
#pragma omp atomic write
                failed = 1;
            } else {
                int64_t r;
#pragma omp for schedule(dynamic, 16)
                for (r = 0; r < rows; ++r) {
                    const int64_t i = r % Nq, bh = r / Nq;
                    const int64_t h = bh % Hq, b = bh / Hq, hk = h / G;
                    const int64_t p = i + (int64_t)Nk - Nq;
                    const double *qi = q + r * d, *doi = dout + r * d;
                    const double *Kb = k + ((b * Hkv + hk) * (int64_t)Nk) * d;
                    const double *Vb = v + ((b * Hkv + hk) * (int64_t)Nk) * d;
                    double *dqi = dq + r * d;
                    int64_t j;
                    int t, any = 0;
                    double m = -INFINITY, l = 0.0, D = 0.0;
                    for (t = 0; t < d; ++t) dqi[t] = 0.0;
                    for (j = 0; j < Nk; ++j) {
                        double acc = 0.0;
                        for (t = 0; t < d; ++t) acc += qi[t] * Kb[j * (int64_t)d + t];
                        s[j] = scale * acc;
                        vis[j] = (unsigned char)oracle_visible(p, j, mask_kind, window, n_sink);
                        if (vis[j]) {
                            if (!any || s[j] > m) m = s[j];
                            any = 1;
                        }
                    }
                    if (!any) {
                        lse[r] = -INFINITY;
                        Dv[r] = 0.0;
                        continue;
                    }
                    for (j = 0; j < Nk; ++j) l += vis[j] ? exp(s[j] - m) : 0.0;
                    lse[r] = m + log(l);
                    /* P_ij, dP_ij and D_i */
                    for (j = 0; j < Nk; ++j) {
                        if (!vis[j]) continue;
                        double acc = 0.0;
                        for (t = 0; t < d; ++t) acc += doi[t] * Vb[j * (int64_t)d + t];
                        dp[j] = acc;
                        s[j] = exp(s[j] - lse[r]); /* s now holds P_ij */
                        D += s[j] * dp[j];
                    }
                    Dv[r] = D;
                    /* dQ_i = scale * sum_j P_ij (dP_ij - D_i) k_j */
                    for (j = 0; j < Nk; ++j) {
                        if (!vis[j]) continue;
                        const double ds = s[j] * (dp[j] - D);
                        for (t = 0; t < d; ++t) dqi[t] += scale * ds * Kb[j * (int64_t)d + t];
                    }
                }
            }
            free(s);
            free(dp);
            free(vis);
        }
    }
    if (!failed) {
        /* ---- pass 2: per key row, dK_j and dV_j over every query row of the group ---- */
        int64_t kr;
#pragma omp parallel for schedule(dynamic, 16)
        for (kr = 0; kr < krows; ++kr) {
            const int64_t j = kr % Nk, bk = kr / Nk;
            const int64_t hk = bk % Hkv, b = bk / Hkv;
            const double *kj = k + kr * d, *vj = v + kr * d;
            double *dkj = dk + kr * d, *dvj = dv + kr * d;
            int t, g;
            for (t = 0; t < d; ++t) dkj[t] = dvj[t] = 0.0;
            for (g = 0; g < G; ++g) {
                const int64_t h = hk * G + g;
                int64_t i;
                for (i = 0; i < Nq; ++i) {
                    const int64_t r = (b * Hq + h) * (int64_t)Nq + i;
                    if (!oracle_visible(i + (int64_t)Nk - Nq, j, mask_kind, window, n_sink))
                        continue;
                    const double *qi = q + r * d, *doi = dout + r * d;
                    double sc = 0.0, dpv = 0.0;
                    for (t = 0; t < d; ++t) {
                        sc += qi[t] * kj[t];
                        dpv += doi[t] * vj[t];
                    }
                    const double pij = exp(scale * sc - lse[r]);
                    const double ds = pij * (dpv - Dv[r]);
                    for (t = 0; t < d; ++t) {
                        dvj[t] += pij * doi[t];
                        dkj[t] += scale * ds * qi[t];
                    }
                }
            }
        }
    }
    free(lse);
    free(Dv);
    return failed ? -2 : 0;
}
