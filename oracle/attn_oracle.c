/*
 * attn_oracle.c -- fp64 CPU oracle for exact softmax attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file; only the test
 * suite, the package's smoke check and the CPU-baseline leg of the benchmark do.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * What it computes (the method's result has a plain definition, so the oracle is that definition written out):
 *
 *   FlashAttention review page, "Method" and claim C2 (exact attention): the tiled method returns exactly
 *   standard attention.  Standard attention (papermap explainer page, "standard attention" section) is
 *       S = scale * Q K^T,   masked entries set to -inf,
 *       P = softmax(S) row by row,
 *       O = P V.
 *   The small normalisation state written next to O (review page, "Method"; slide deck "Action grammar",
 *   normalization state) is read as the per-row natural-log logsumexp LSE_r = log sum_c exp(S_rc).
 *
 *   Backward (review page, claim C7 / E-recompute: gradients from recomputed tiles and the saved
 *   normalisation): the pages print no equations; the reading used is the calculus of the definition above
 *   for the loss L = sum(O * dO):
 *       D_r  = sum_j dO_rj O_rj
 *       dV   = P^T dO
 *       dP   = dO V^T
 *       dS   = P o (dP - D)
 *       dQ   = scale * dS K
 *       dK   = scale * dS^T Q
 *
 *   Masks (explainer page, block-sparse section: whole tiles can be masked): key c is allowed for query row r
 *   of sequence b iff all of
 *       causal      -> c <= r
 *       key_lens    -> c <  key_lens[b]
 *       block_mask  -> block_mask[(r / tile) * nT + (c / tile)] != 0,  nT = ceil(N / tile)
 *   A row with no allowed key has O = 0, LSE = -inf and zero gradients.
 *
 *   oracle_fwd_online follows the online-softmax recurrence of the explainer page ("online softmax" section:
 *   running max m and running sum l, earlier partial outputs rescaled when the max grows) and the loop of the
 *   slide deck's "Executable shape" slide (state per q block, K/V blocks streamed), in either loop order.
 *
 * Layout: every tensor is [B, H, N, d] (d innermost) in fp64; LSE is [B, H, N].
 * Parallelism: OpenMP over independent (b, h) heads or selected rows; no blocking or reordering of the
 * arithmetic beyond the definitions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, H, N, d;
    double scale;
    int causal;
    const int32_t *key_lens; /* [B] or NULL */
    const uint8_t *block_mask; /* [nT * nT] or NULL */
    int tile;                  /* block-mask tile size (128 in the product; any >= 1 here) */
} attn_problem;

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the OpenMP regions that follow (the host-baseline timing runs once on one core, once on all). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Is key c visible from query row r of sequence b? */
static int allowed(const attn_problem *p, int b, int r, int c) {
    if (p->causal && c > r) return 0;
    if (p->key_lens && c >= p->key_lens[b]) return 0;
    if (p->block_mask) {
        int nT = (p->N + p->tile - 1) / p->tile;
        if (!p->block_mask[(size_t)(r / p->tile) * nT + (c / p->tile)]) return 0;
    }
    return 1;
}

static double dot(const double *a, const double *b, int d) {
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += a[i] * b[i];
    return s;
}

/*
 * One query row, two-pass softmax: fills prob[0..N) (0 where masked), o_row[0..d), returns LSE.
 * scores is scratch of length N.
 */
static double row_forward(const attn_problem *p, const double *Q, const double *K, const double *V, int b,
                          int r, double *scores, double *prob, double *o_row) {
    const int N = p->N, d = p->d;
    double m = -INFINITY;
    for (int c = 0; c < N; ++c) {
        if (allowed(p, b, r, c)) {
            scores[c] = p->scale * dot(Q + (size_t)r * d, K + (size_t)c * d, d);
            if (scores[c] > m) m = scores[c];
        } else {
            scores[c] = -INFINITY;
        }
    }
    for (int j = 0; j < d; ++j) o_row[j] = 0.0;
    if (m == -INFINITY) { /* no visible key */
        for (int c = 0; c < N; ++c) prob[c] = 0.0;
        return -INFINITY;
    }
    double sum = 0.0;
    for (int c = 0; c < N; ++c) sum += (scores[c] == -INFINITY) ? 0.0 : exp(scores[c] - m);
    double lse = m + log(sum);
    for (int c = 0; c < N; ++c) {
        prob[c] = (scores[c] == -INFINITY) ? 0.0 : exp(scores[c] - lse);
        if (prob[c] != 0.0)
            for (int j = 0; j < d; ++j) o_row[j] += prob[c] * V[(size_t)c * d + j];
    }
    return lse;
}

static attn_problem make_problem(int B, int H, int N, int d, double scale, int causal, const int32_t *key_lens,
                                 const uint8_t *block_mask, int tile) {
    attn_problem p;
    p.B = B; p.H = H; p.N = N; p.d = d; p.scale = scale; p.causal = causal;
    p.key_lens = key_lens; p.block_mask = block_mask; p.tile = tile > 0 ? tile : 1;
    return p;
}

/* Full forward: O [B,H,N,d], LSE [B,H,N]. */
void oracle_fwd(const double *q, const double *k, const double *v, int B, int H, int N, int d, double scale,
                int causal, const int32_t *key_lens, const uint8_t *block_mask, int tile, double *o, double *lse) {
    attn_problem p = make_problem(B, H, N, d, scale, causal, key_lens, block_mask, tile);
    const size_t head = (size_t)N * d;
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)N);
        double *prob = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int bh = 0; bh < B * H; ++bh)
            for (int r = 0; r < N; ++r) {
                const size_t base = (size_t)bh * head;
                lse[(size_t)bh * N + r] = row_forward(&p, q + base, k + base, v + base, bh / H, r, scores, prob,
                                                      o + base + (size_t)r * d);
            }
        free(scores);
        free(prob);
    }
}

/* Forward for selected rows only: sel_bh[i] in [0, B*H), sel_r[i] in [0, N); o_sel [nsel, d], lse_sel [nsel]. */
void oracle_fwd_rows(const double *q, const double *k, const double *v, int B, int H, int N, int d, double scale,
                     int causal, const int32_t *key_lens, const uint8_t *block_mask, int tile, int nsel,
                     const int64_t *sel_bh, const int64_t *sel_r, double *o_sel, double *lse_sel) {
    attn_problem p = make_problem(B, H, N, d, scale, causal, key_lens, block_mask, tile);
    const size_t head = (size_t)N * d;
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)N);
        double *prob = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < nsel; ++i) {
            const size_t base = (size_t)sel_bh[i] * head;
            lse_sel[i] = row_forward(&p, q + base, k + base, v + base, (int)(sel_bh[i] / H), (int)sel_r[i], scores,
                                     prob, o_sel + (size_t)i * d);
        }
        free(scores);
        free(prob);
    }
}

/*
 * Online (tiled) forward, explainer page "online softmax": per query block a state (m, l, acc); K/V blocks
 * arrive one at a time; when a block raises the running max, the earlier acc and l are scaled by
 * exp(m_old - m_new).  kv_outer != 0 runs the slide deck's order (K/V blocks outer, Q blocks inner, state kept
 * per q block); kv_outer == 0 runs Q blocks outer.  Fully-masked score tiles are skipped.
 */
void oracle_fwd_online(const double *q, const double *k, const double *v, int B, int H, int N, int d, double scale,
                       int causal, const int32_t *key_lens, const uint8_t *block_mask, int tile, int tile_q,
                       int tile_k, int kv_outer, double *o, double *lse) {
    attn_problem p = make_problem(B, H, N, d, scale, causal, key_lens, block_mask, tile);
    const size_t head = (size_t)N * d;
    const int nq = (N + tile_q - 1) / tile_q, nk = (N + tile_k - 1) / tile_k;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H;
        const double *Q = q + (size_t)bh * head, *K = k + (size_t)bh * head, *V = v + (size_t)bh * head;
        double *m = (double *)malloc(sizeof(double) * (size_t)N);
        double *l = (double *)malloc(sizeof(double) * (size_t)N);
        double *acc = (double *)calloc(head, sizeof(double));
        double *s = (double *)malloc(sizeof(double) * (size_t)tile_k);
        for (int r = 0; r < N; ++r) { m[r] = -INFINITY; l[r] = 0.0; }
        const int outer = kv_outer ? nk : nq, inner = kv_outer ? nq : nk;
        for (int a = 0; a < outer; ++a)
            for (int bb = 0; bb < inner; ++bb) {
                const int iq = kv_outer ? bb : a, jk = kv_outer ? a : bb;
                const int r0 = iq * tile_q, r1 = (r0 + tile_q < N) ? r0 + tile_q : N;
                const int c0 = jk * tile_k, c1 = (c0 + tile_k < N) ? c0 + tile_k : N;
                for (int r = r0; r < r1; ++r) {
                    double tmax = -INFINITY;
                    for (int c = c0; c < c1; ++c) {
                        s[c - c0] = allowed(&p, b, r, c) ? p.scale * dot(Q + (size_t)r * d, K + (size_t)c * d, d)
                                                         : -INFINITY;
                        if (s[c - c0] > tmax) tmax = s[c - c0];
                    }
                    if (tmax == -INFINITY) continue; /* this score tile row is fully masked: skip it */
                    const double m_new = (tmax > m[r]) ? tmax : m[r];
                    const double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - m_new);
                    double *arow = acc + (size_t)r * d;
                    for (int j = 0; j < d; ++j) arow[j] *= alpha;
                    l[r] *= alpha;
                    for (int c = c0; c < c1; ++c) {
                        if (s[c - c0] == -INFINITY) continue;
                        const double e = exp(s[c - c0] - m_new);
                        l[r] += e;
                        for (int j = 0; j < d; ++j) arow[j] += e * V[(size_t)c * d + j];
                    }
                    m[r] = m_new;
                }
            }
        for (int r = 0; r < N; ++r) {
            double *orow = o + (size_t)bh * head + (size_t)r * d;
            if (l[r] == 0.0) {
                for (int j = 0; j < d; ++j) orow[j] = 0.0;
                lse[(size_t)bh * N + r] = -INFINITY;
            } else {
                for (int j = 0; j < d; ++j) orow[j] = acc[(size_t)r * d + j] / l[r];
                lse[(size_t)bh * N + r] = m[r] + log(l[r]);
            }
        }
        free(m); free(l); free(acc); free(s);
    }
}

/*
 * Full backward for the loss sum(O * dO).  Outputs dq, dk, dv [B,H,N,d]; o and lse (may be NULL) receive the
 * forward result used.
 */
void oracle_bwd(const double *q, const double *k, const double *v, const double *dout, int B, int H, int N, int d,
                double scale, int causal, const int32_t *key_lens, const uint8_t *block_mask, int tile, double *dq,
                double *dk, double *dv, double *o, double *lse) {
    attn_problem p = make_problem(B, H, N, d, scale, causal, key_lens, block_mask, tile);
    const size_t head = (size_t)N * d;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H;
        const size_t base = (size_t)bh * head;
        const double *Q = q + base, *K = k + base, *V = v + base, *dO = dout + base;
        double *dQ = dq + base, *dK = dk + base, *dV = dv + base;
        double *scores = (double *)malloc(sizeof(double) * (size_t)N);
        double *prob = (double *)malloc(sizeof(double) * (size_t)N);
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);
        memset(dK, 0, sizeof(double) * head);
        memset(dV, 0, sizeof(double) * head);
        for (int r = 0; r < N; ++r) {
            const double l = row_forward(&p, Q, K, V, b, r, scores, prob, orow);
            if (o) memcpy(o + base + (size_t)r * d, orow, sizeof(double) * (size_t)d);
            if (lse) lse[(size_t)bh * N + r] = l;
            const double *dOr = dO + (size_t)r * d;
            const double D = dot(dOr, orow, d); /* D_r = sum_j dO_rj O_rj */
            double *dQr = dQ + (size_t)r * d;
            for (int j = 0; j < d; ++j) dQr[j] = 0.0;
            for (int c = 0; c < N; ++c) {
                if (prob[c] == 0.0) continue;
                const double dP = dot(dOr, V + (size_t)c * d, d); /* dP_rc = dO_r . V_c */
                const double dS = prob[c] * (dP - D);              /* dS_rc = P_rc (dP_rc - D_r) */
                for (int j = 0; j < d; ++j) {
                    dQr[j] += scale * dS * K[(size_t)c * d + j];
                    dK[(size_t)c * d + j] += scale * dS * Q[(size_t)r * d + j];
                    dV[(size_t)c * d + j] += prob[c] * dOr[j];
                }
            }
        }
        free(scores); free(prob); free(orow);
    }
}

/* dQ for selected rows: only the row's own forward is needed. dq_sel [nsel, d]. */
void oracle_bwd_rows(const double *q, const double *k, const double *v, const double *dout, int B, int H, int N, int d,
                     double scale, int causal, const int32_t *key_lens, const uint8_t *block_mask, int tile, int nsel,
                     const int64_t *sel_bh, const int64_t *sel_r, double *dq_sel) {
    attn_problem p = make_problem(B, H, N, d, scale, causal, key_lens, block_mask, tile);
    const size_t head = (size_t)N * d;
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)N);
        double *prob = (double *)malloc(sizeof(double) * (size_t)N);
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < nsel; ++i) {
            const size_t base = (size_t)sel_bh[i] * head;
            const int r = (int)sel_r[i];
            const double *Q = q + base, *K = k + base, *V = v + base, *dOr = dout + base + (size_t)r * d;
            row_forward(&p, Q, K, V, (int)(sel_bh[i] / H), r, scores, prob, orow);
            const double D = dot(dOr, orow, d);
            double *out = dq_sel + (size_t)i * d;
            for (int j = 0; j < d; ++j) out[j] = 0.0;
            for (int c = 0; c < N; ++c) {
                if (prob[c] == 0.0) continue;
                const double dS = prob[c] * (dot(dOr, V + (size_t)c * d, d) - D);
                for (int j = 0; j < d; ++j) out[j] += scale * dS * K[(size_t)c * d + j];
            }
        }
        free(scores); free(prob); free(orow);
    }
}

/*
 * dK and dV for selected keys.  Column c of P needs LSE_r and D_r of every row r of the head, so the forward of
 * every row of each head that appears in sel_bh is computed first (once per distinct head).
 * dk_sel, dv_sel [nsel, d].
 */
void oracle_bwd_keys(const double *q, const double *k, const double *v, const double *dout, int B, int H, int N,
                     int d, double scale, int causal, const int32_t *key_lens, const uint8_t *block_mask, int tile,
                     int nsel, const int64_t *sel_bh, const int64_t *sel_c, double *dk_sel, double *dv_sel) {
    attn_problem p = make_problem(B, H, N, d, scale, causal, key_lens, block_mask, tile);
    const size_t head = (size_t)N * d;
    /* distinct heads, in order of first appearance */
    int64_t *heads = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nsel > 0 ? nsel : 1));
    int nh = 0;
    for (int i = 0; i < nsel; ++i) {
        int seen = 0;
        for (int t = 0; t < nh; ++t) seen |= (heads[t] == sel_bh[i]);
        if (!seen) heads[nh++] = sel_bh[i];
    }
    double *lse_h = (double *)malloc(sizeof(double) * (size_t)N);
    double *D_h = (double *)malloc(sizeof(double) * (size_t)N);
    for (int t = 0; t < nh; ++t) {
        const int64_t bh = heads[t];
        const int b = (int)(bh / H);
        const size_t base = (size_t)bh * head;
        const double *Q = q + base, *K = k + base, *V = v + base, *dO = dout + base;
#pragma omp parallel
        {
            double *scores = (double *)malloc(sizeof(double) * (size_t)N);
            double *prob = (double *)malloc(sizeof(double) * (size_t)N);
            double *orow = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
            for (int r = 0; r < N; ++r) {
                lse_h[r] = row_forward(&p, Q, K, V, b, r, scores, prob, orow);
                D_h[r] = dot(dO + (size_t)r * d, orow, d);
            }
            free(scores); free(prob); free(orow);
        }
#pragma omp parallel for schedule(dynamic, 1)
        for (int i = 0; i < nsel; ++i) {
            if (sel_bh[i] != bh) continue;
            const int c = (int)sel_c[i];
            double *dKc = dk_sel + (size_t)i * d, *dVc = dv_sel + (size_t)i * d;
            for (int j = 0; j < d; ++j) { dKc[j] = 0.0; dVc[j] = 0.0; }
            for (int r = 0; r < N; ++r) {
                if (lse_h[r] == -INFINITY || !allowed(&p, b, r, c)) continue;
                const double P = exp(scale * dot(Q + (size_t)r * d, K + (size_t)c * d, d) - lse_h[r]);
                const double dS = P * (dot(dO + (size_t)r * d, V + (size_t)c * d, d) - D_h[r]);
                for (int j = 0; j < d; ++j) {
                    dKc[j] += scale * dS * Q[(size_t)r * d + j];
                    dVc[j] += P * dO[(size_t)r * d + j];
                }
            }
        }
    }
    free(heads); free(lse_h); free(D_h);
}

/*
 * Block-mask index lists (explainer page, block-sparse section: kept tiles are the only ones loaded).
 * CSR over tile rows: row_ptr[nT + 1], col_idx[nnz], columns ascending within a row.
 * CSC over tile columns: col_ptr[nT + 1], row_idx[nnz], rows ascending within a column.
 * Returns nnz.
 */
int64_t oracle_blockmask_csr(const uint8_t *mask, int nT, int32_t *row_ptr, int32_t *col_idx) {
    int64_t nnz = 0;
    for (int i = 0; i < nT; ++i) {
        row_ptr[i] = (int32_t)nnz;
        for (int j = 0; j < nT; ++j)
            if (mask[(size_t)i * nT + j]) col_idx[nnz++] = j;
    }
    row_ptr[nT] = (int32_t)nnz;
    return nnz;
}

int64_t oracle_blockmask_csc(const uint8_t *mask, int nT, int32_t *col_ptr, int32_t *row_idx) {
    int64_t nnz = 0;
    for (int j = 0; j < nT; ++j) {
        col_ptr[j] = (int32_t)nnz;
        for (int i = 0; i < nT; ++i)
            if (mask[(size_t)i * nT + j]) row_idx[nnz++] = i;
    }
    col_ptr[nT] = (int32_t)nnz;
    return nnz;
}
