/*
 * Reference oracle for block-sparse attention with hybrid top-k + top-p block masks.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, fp64 CPU statement of what the
 * block-sparse attention path computes.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header, table or helper
 * with the CUDA path, and it never reads anything the CUDA path produced.
 *
 * Sources (page title, section):
 *   [SA2]  "SpargeAttention2とは？Top-k+Top-pハイブリッドマスキングでビデオ生成を16.2倍高速化",
 *          section "Top-kとTop-pの限界を解剖する" (top-k keeps the k largest probabilities; top-p
 *          takes blocks from the top until the cumulative probability passes p) and section
 *          "ハイブリッドマスキングと蒸留微調整" (the hybrid mask is the union of both sets).
 *   [SVG2] "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
 *          Semantic-Aware Permutation", section 1 (block representatives by mean pooling) and
 *          section 2.B (scores between representatives, sorted, cumulative top-p that reaches p).
 *   The block size, mean pooling, the 1/sqrt(d) score scale and the bf16 [B,H,N,d] layout are
 *   fixed by the problem statement this library implements; the pages leave them open.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - pooling is the mean over the valid tokens of a block (a tail block has fewer than bs);
 *   - block probabilities are softmax_j(Qp_i . Kp_j * scale) over all key blocks of the row;
 *   - ranking is by probability descending, ties broken by the lower block index;
 *   - top-p keeps the shortest ranked prefix whose cumulative probability is >= p
 *     ("reaches", [SVG2] 2.B); p <= 0 keeps nothing, p >= 1 keeps every block;
 *   - keys at or beyond N never enter attention; a query block with no kept key block
 *     produces zeros.
 *
 * Parity pins: every function here is pinned in tests/test_oracle_pins.py against closed forms,
 * brute force and independent library routines (numpy, scipy, torch), not against itself.
 *
 * Everything is fp64.  bf16 inputs arrive as their raw 16-bit patterns and are widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* exact widening of a bf16 bit pattern: it is the top half of an IEEE binary32 */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int or_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------------------------
 * Block representatives: xp[bh, i, c] = mean over tokens t of block i (t < N) of x[bh, t, c].
 * [SVG2] section 1 names mean pooling of contiguous token blocks as the representative.
 * x: [BH, N, d] bf16 bits.  xp: [BH, nb, d] fp64, nb = ceil(N / bs).
 * ------------------------------------------------------------------------------------------- */
void or_pool_blocks(const uint16_t *x, int64_t BH, int64_t N, int64_t d, int64_t bs, double *xp) {
    int64_t nb = (N + bs - 1) / bs;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t i = 0; i < nb; ++i) {
            int64_t t0 = i * bs;
            int64_t t1 = t0 + bs < N ? t0 + bs : N;
            double n = (double)(t1 - t0);
            for (int64_t c = 0; c < d; ++c) {
                double s = 0.0;
                for (int64_t t = t0; t < t1; ++t) s += bf16_to_double(x[(bh * N + t) * d + c]);
                xp[(bh * nb + i) * d + c] = s / n;
            }
        }
    }
}

/* ---------------------------------------------------------------------------------------------
 * Block scores and their row softmax ([SVG2] 2.B: scores between representatives stand in
 * for the full attention map; the problem statement fixes softmax(Qp Kp^T * scale)).
 * qp: [BH, nbq, d], kp: [BH, nbk, d] fp64.  prob: [BH, nbq, nbk] fp64.
 * ------------------------------------------------------------------------------------------- */
void or_block_probs(const double *qp, const double *kp, int64_t BH, int64_t nbq, int64_t nbk,
                    int64_t d, double scale, double *prob) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t i = 0; i < nbq; ++i) {
            const double *q = qp + (bh * nbq + i) * d;
            double *row = prob + (bh * nbq + i) * nbk;
            double mx = -INFINITY;
            for (int64_t j = 0; j < nbk; ++j) {
                const double *k = kp + (bh * nbk + j) * d;
                double s = 0.0;
                for (int64_t c = 0; c < d; ++c) s += q[c] * k[c];
                row[j] = s * scale;
                if (row[j] > mx) mx = row[j];
            }
            double z = 0.0;
            for (int64_t j = 0; j < nbk; ++j) {
                row[j] = exp(row[j] - mx);
                z += row[j];
            }
            for (int64_t j = 0; j < nbk; ++j) row[j] /= z;
        }
    }
}

/* The block scores themselves, L[i, j] = Qp_i . Kp_j * scale (the logits of the softmax above).
 * [SVG2] 2.B calls them the estimated attention scores; the near-threshold rule of the parity
 * tests is stated on them. */
void or_block_logits(const double *qp, const double *kp, int64_t BH, int64_t nbq, int64_t nbk,
                     int64_t d, double scale, double *logit) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t i = 0; i < nbq; ++i) {
            const double *q = qp + (bh * nbq + i) * d;
            double *row = logit + (bh * nbq + i) * nbk;
            for (int64_t j = 0; j < nbk; ++j) {
                const double *k = kp + (bh * nbk + j) * d;
                double s = 0.0;
                for (int64_t c = 0; c < d; ++c) s += q[c] * k[c];
                row[j] = s * scale;
            }
        }
    }
}

/* softmax of given logits, row by row (used to feed hand-made rows into the selection) */
void or_softmax_rows(const double *logits, int64_t rows, int64_t n, double *prob) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *x = logits + r * n;
        double *y = prob + r * n;
        double mx = -INFINITY;
        for (int64_t j = 0; j < n; ++j) if (x[j] > mx) mx = x[j];
        double z = 0.0;
        for (int64_t j = 0; j < n; ++j) { y[j] = exp(x[j] - mx); z += y[j]; }
        for (int64_t j = 0; j < n; ++j) y[j] /= z;
    }
}

/* ---------------------------------------------------------------------------------------------
 * Hybrid selection, one row at a time ([SA2] "Top-kとTop-pの限界を解剖する" and
 * "ハイブリッドマスキングと蒸留微調整"; [SVG2] 2.B for the sort-then-accumulate top-p).
 *
 *   order  : block ids sorted by probability descending, lower id first on equal probability
 *   S_k    : the first min(k, nb) blocks of the order
 *   S_p    : the first m blocks, m the least count with sum of their probabilities >= p
 *            (p <= 0: m = 0; p >= 1: m = nb)
 *   keep   : S_k union S_p
 *
 * Outputs per row: mask[nb] (0/1), cnt (|keep|), and diagnostics used by the parity rule:
 *   tau_k  : probability of the last block of S_k (NaN if S_k is empty)
 *   tau_p  : probability of the last block of S_p (NaN if S_p is empty)
 *   m_p    : |S_p|
 *   cum_lo : sum of the first m-1 ranked probabilities (the mass just before the cut)
 *   cum_hi : sum of the first m ranked probabilities (the mass at the cut)
 *   rank   : rank[j] = position of block j in the order
 * ------------------------------------------------------------------------------------------- */
typedef struct {
    double p;
    int32_t j;
} ranked_t;

static int ranked_cmp(const void *a, const void *b) {
    const ranked_t *x = (const ranked_t *)a, *y = (const ranked_t *)b;
    if (x->p > y->p) return -1;
    if (x->p < y->p) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

void or_select_rows(const double *prob, int64_t rows, int64_t nb, int64_t topk, double topp,
                    uint8_t *mask, int32_t *cnt, double *tau_k, double *tau_p, int32_t *m_p,
                    double *cum_lo, double *cum_hi, int32_t *rank) {
#pragma omp parallel
    {
        ranked_t *ord = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(nb > 0 ? nb : 1));
        uint8_t *in_k = (uint8_t *)malloc((size_t)(nb > 0 ? nb : 1));
        uint8_t *in_p = (uint8_t *)malloc((size_t)(nb > 0 ? nb : 1));
#pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            const double *P = prob + r * nb;
            for (int64_t j = 0; j < nb; ++j) { ord[j].p = P[j]; ord[j].j = (int32_t)j; }
            qsort(ord, (size_t)nb, sizeof(ranked_t), ranked_cmp);
            if (rank) for (int64_t q = 0; q < nb; ++q) rank[r * nb + ord[q].j] = (int32_t)q;

            /* top-k: the k largest probabilities */
            int64_t kk = topk < nb ? topk : nb;
            if (kk < 0) kk = 0;
            memset(in_k, 0, (size_t)nb);
            for (int64_t q = 0; q < kk; ++q) in_k[ord[q].j] = 1;

            /* top-p: shortest ranked prefix whose cumulative probability reaches p */
            int64_t m;
            double lo = 0.0, hi = 0.0;
            if (topp <= 0.0) {
                m = 0;
            } else if (topp >= 1.0) {
                m = nb;
                for (int64_t q = 0; q < nb; ++q) { lo = hi; hi += ord[q].p; }
            } else {
                double cum = 0.0;
                m = nb;
                for (int64_t q = 0; q < nb; ++q) {
                    lo = cum;
                    cum += ord[q].p;
                    hi = cum;
                    if (cum >= topp) { m = q + 1; break; }
                }
            }
            memset(in_p, 0, (size_t)nb);
            for (int64_t q = 0; q < m; ++q) in_p[ord[q].j] = 1;

            /* hybrid: union of the two sets */
            int32_t c = 0;
            for (int64_t j = 0; j < nb; ++j) {
                uint8_t keep = (uint8_t)(in_k[j] | in_p[j]);
                mask[r * nb + j] = keep;
                c += keep;
            }
            cnt[r] = c;
            if (tau_k) tau_k[r] = kk > 0 ? ord[kk - 1].p : NAN;
            if (tau_p) tau_p[r] = m > 0 ? ord[m - 1].p : NAN;
            if (m_p) m_p[r] = (int32_t)m;
            if (cum_lo) cum_lo[r] = lo;
            if (cum_hi) cum_hi[r] = hi;
        }
        free(ord);
        free(in_k);
        free(in_p);
    }
}

/* ---------------------------------------------------------------------------------------------
 * Masked attention: for every query token t of query block i (t < N),
 *   O[t] = sum_{s in kept blocks of i, s < N} softmax_s(scale * Q[t].K[s]) V[s]
 * with the softmax normalised over the kept keys only; two passes (max, then sum) in fp64.
 * A query block with no kept key block yields O = 0.
 *
 * q, k, v: [BH, N, d] bf16 bits.  mask: [BH, nbq, nbk] 0/1 with nbq = nbk = ceil(N / bs).
 * The query blocks to evaluate are listed in (sel_bh[s], sel_i[s]) for s < nsel; their rows are
 * written to out[s, r, :] for r < bs (rows at or beyond N are left at 0).  out: [nsel, bs, d].
 * ------------------------------------------------------------------------------------------- */
void or_masked_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t N,
                         int64_t d, int64_t bs, const uint8_t *mask, double scale,
                         const int64_t *sel_bh, const int64_t *sel_i, int64_t nsel, double *out) {
    int64_t nb = (N + bs - 1) / bs;
#pragma omp parallel
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)N);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for collapse(2) schedule(dynamic, 1)
        for (int64_t s = 0; s < nsel; ++s) {
            for (int64_t r = 0; r < bs; ++r) {
                int64_t bh = sel_bh[s], i = sel_i[s];
                int64_t t = i * bs + r;
                double *o = out + (s * bs + r) * d;
                for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
                if (t >= N) continue;
                const uint8_t *mrow = mask + (bh * nb + i) * nb;
                for (int64_t c = 0; c < d; ++c) qr[c] = bf16_to_double(q[(bh * N + t) * d + c]);
                /* pass 1: logits of the kept keys and their maximum */
                double mx = -INFINITY;
                int any = 0;
                for (int64_t j = 0; j < nb; ++j) {
                    if (!mrow[j]) continue;
                    int64_t s1 = (j + 1) * bs < N ? (j + 1) * bs : N;
                    for (int64_t sk = j * bs; sk < s1; ++sk) {
                        const uint16_t *kr = k + (bh * N + sk) * d;
                        double x = 0.0;
                        for (int64_t c = 0; c < d; ++c) x += qr[c] * bf16_to_double(kr[c]);
                        x *= scale;
                        w[sk] = x;
                        if (x > mx) mx = x;
                        any = 1;
                    }
                }
                if (!any) continue;
                /* pass 2: normaliser and weighted sum of values */
                double z = 0.0;
                for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
                for (int64_t j = 0; j < nb; ++j) {
                    if (!mrow[j]) continue;
                    int64_t s1 = (j + 1) * bs < N ? (j + 1) * bs : N;
                    for (int64_t sk = j * bs; sk < s1; ++sk) {
                        double e = exp(w[sk] - mx);
                        z += e;
                        const uint16_t *vr = v + (bh * N + sk) * d;
                        for (int64_t c = 0; c < d; ++c) acc[c] += e * bf16_to_double(vr[c]);
                    }
                }
                for (int64_t c = 0; c < d; ++c) o[c] = acc[c] / z;
            }
        }
        free(w);
        free(qr);
        free(acc);
    }
}

/* ---------------------------------------------------------------------------------------------
 * Dense attention, the 0 %-sparsity control: O[t] = sum_{s<N} softmax_s(scale Q[t].K[s]) V[s].
 * Written without blocks so that it is an independent statement of the same softmax.
 * Rows to evaluate: (sel_bh[s], sel_t[s]); out: [nsel, d].
 * ------------------------------------------------------------------------------------------- */
void or_dense_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t N,
                        int64_t d, double scale, const int64_t *sel_bh, const int64_t *sel_t,
                        int64_t nsel, double *out) {
#pragma omp parallel
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)N);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 8)
        for (int64_t s = 0; s < nsel; ++s) {
            int64_t bh = sel_bh[s], t = sel_t[s];
            double *o = out + s * d;
            for (int64_t c = 0; c < d; ++c) qr[c] = bf16_to_double(q[(bh * N + t) * d + c]);
            double mx = -INFINITY;
            for (int64_t sk = 0; sk < N; ++sk) {
                const uint16_t *kr = k + (bh * N + sk) * d;
                double x = 0.0;
                for (int64_t c = 0; c < d; ++c) x += qr[c] * bf16_to_double(kr[c]);
                w[sk] = x * scale;
                if (w[sk] > mx) mx = w[sk];
            }
            double z = 0.0;
            for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t sk = 0; sk < N; ++sk) {
                double e = exp(w[sk] - mx);
                z += e;
                const uint16_t *vr = v + (bh * N + sk) * d;
                for (int64_t c = 0; c < d; ++c) o[c] += e * bf16_to_double(vr[c]);
            }
            for (int64_t c = 0; c < d; ++c) o[c] /= z;
        }
        free(w);
        free(qr);
    }
}

/* ---------------------------------------------------------------------------------------------
 * Static block patterns.  Sparse-vDiT page ("Sparse-vDiT：動画拡散トランスフォーマの高速化を可能に
 * するスパースアテンションの解放"), section 3: attention maps of video DiT heads repeat as diagonal,
 * multi-diagonal and vertical-stripe patterns, fixed per layer and head, and some heads can be
 * skipped.  Read at block granularity, per head h with pat[h] = {flags, w, p, s}, key block j
 * is kept for query block i when any enabled part holds:
 *   flags & 1: |i - j| <= w                                  (diagonal band)
 *   flags & 2: |(i - j) - m p| <= w for some integer m, p > 0 (diagonals every p blocks)
 *   flags & 4: j < s                                         (vertical stripe of the first s)
 * flags == 0 keeps nothing (a skipped head).  mask: [H, nb, nb].
 * ------------------------------------------------------------------------------------------- */
void or_static_mask(const int32_t *pat, int64_t H, int64_t nb, uint8_t *mask) {
    for (int64_t h = 0; h < H; ++h) {
        const int64_t flags = pat[4 * h], w = pat[4 * h + 1], p = pat[4 * h + 2], s = pat[4 * h + 3];
        for (int64_t i = 0; i < nb; ++i) {
            for (int64_t j = 0; j < nb; ++j) {
                const int64_t diff = i - j;
                int keep = 0;
                if ((flags & 1) && llabs(diff) <= w) keep = 1;
                if ((flags & 2) && p > 0) {
                    /* every integer m whose diagonal m p can reach within w of diff */
                    for (int64_t m = -(nb / p) - 1; m <= nb / p + 1 && !keep; ++m)
                        if (llabs(diff - m * p) <= w) keep = 1;
                }
                if ((flags & 4) && j < s) keep = 1;
                mask[(h * nb + i) * nb + j] = (uint8_t)keep;
            }
        }
    }
}

/* ---------------------------------------------------------------------------------------------
 * SQuad attention.  SQuad page ("SQuad: Sub-Quadratic Attention Distillation for Efficient
 * Video Generation"), method section 1, the SQuad attention operator: full attention is split
 * into a local pass, softmax attention among the tokens of each fixed window of w tokens, and a
 * global pass, softmax attention among the tokens at the same relative position in every window,
 * whose values are the local pass's outputs.  With n = W w tokens, token t = a w + r (window a,
 * position r):
 *   Y[a w + r] = sum_{r'} softmax_{r'}(scale q[a w + r] . k[a w + r']) v[a w + r']
 *   O[a w + r] = sum_{a'} softmax_{a'}(scale q[a w + r] . k[a' w + r]) Y[a' w + r]
 * q, k, v: [BH, n, d] bf16 bits; out: [BH, n, d].  n must be a multiple of w.
 * ------------------------------------------------------------------------------------------- */
static void softmax_mix(const double *qr, const uint16_t *k, const double *vd, const uint16_t *vb,
                        const int64_t *rows, int64_t m, int64_t d, double scale, double *w,
                        double *o) {
    /* o = sum over the m rows listed of softmax(scale qr . k[row]) * value[row]; the values are
       vd (double) when given, else vb (bf16 bits) */
    double mx = -INFINITY;
    for (int64_t x = 0; x < m; ++x) {
        const uint16_t *kr = k + rows[x] * d;
        double s = 0.0;
        for (int64_t c = 0; c < d; ++c) s += qr[c] * bf16_to_double(kr[c]);
        w[x] = s * scale;
        if (w[x] > mx) mx = w[x];
    }
    double z = 0.0;
    for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
    for (int64_t x = 0; x < m; ++x) {
        const double e = exp(w[x] - mx);
        z += e;
        for (int64_t c = 0; c < d; ++c)
            o[c] += e * (vd ? vd[rows[x] * d + c] : bf16_to_double(vb[rows[x] * d + c]));
    }
    for (int64_t c = 0; c < d; ++c) o[c] /= z;
}

void or_squad_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t BH,
                        int64_t n, int64_t d, int64_t win, double scale, double *out) {
    const int64_t W = n / win;
    double *y = (double *)malloc(sizeof(double) * (size_t)(n * d));
    double *qr = (double *)malloc(sizeof(double) * (size_t)d);
    double *wt = (double *)malloc(sizeof(double) * (size_t)(win > W ? win : W));
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(win > W ? win : W));
    for (int64_t bh = 0; bh < BH; ++bh) {
        const uint16_t *qb = q + bh * n * d, *kb = k + bh * n * d, *vb = v + bh * n * d;
        /* local pass: the tokens of window a */
        for (int64_t t = 0; t < n; ++t) {
            const int64_t a = t / win;
            for (int64_t x = 0; x < win; ++x) rows[x] = a * win + x;
            for (int64_t c = 0; c < d; ++c) qr[c] = bf16_to_double(qb[t * d + c]);
            softmax_mix(qr, kb, NULL, vb, rows, win, d, scale, wt, y + t * d);
        }
        /* global pass: the tokens at position r of every window, values from the local pass */
        for (int64_t t = 0; t < n; ++t) {
            const int64_t r = t % win;
            for (int64_t x = 0; x < W; ++x) rows[x] = x * win + r;
            for (int64_t c = 0; c < d; ++c) qr[c] = bf16_to_double(qb[t * d + c]);
            softmax_mix(qr, kb, y, NULL, rows, W, d, scale, wt, out + (bh * n + t) * d);
        }
    }
    free(y);
    free(qr);
    free(wt);
    free(rows);
}

/* ---------------------------------------------------------------------------------------------
 * Sparse VideoGen2 semantic-aware permutation with centroid top-p.  SVG2 page ("Sparse
 * VideoGen2: Accelerate Video Generation with Sparse Attention via Semantic-Aware Permutation"),
 * method A (Q and K clustered separately by k-means into Cq and Ck groups, tokens reordered so
 * that a cluster is contiguous; the permutations leave the result equal to attention in token
 * order), B (scores between cluster centroids, clusters taken in order of the estimated score
 * until the cumulative score reaches p) and C (k-means warm-started from cached centroids).
 * ------------------------------------------------------------------------------------------- */

/* k-means (Lloyd): `iters` rounds of assigning every row of x [n, d] to its nearest centroid
 * (squared Euclidean distance, the lower index on a tie) and moving every centroid to the mean of
 * its rows (a centroid without rows stays where it is), then a final assignment.  cent [C, d]
 * holds the starting centroids on entry and the final ones on return; assign [n]. */
void or_kmeans(const double *x, int64_t n, int64_t d, int64_t C, int64_t iters, double *cent,
               int32_t *assign) {
    double *sum = (double *)malloc(sizeof(double) * (size_t)(C * d));
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)C);
    for (int64_t it = 0; it <= iters; ++it) {
        for (int64_t t = 0; t < n; ++t) {
            double best = INFINITY;
            int64_t arg = 0;
            for (int64_t c = 0; c < C; ++c) {
                double dist = 0.0;
                for (int64_t e = 0; e < d; ++e) {
                    const double diff = x[t * d + e] - cent[c * d + e];
                    dist += diff * diff;
                }
                if (dist < best) {
                    best = dist;
                    arg = c;
                }
            }
            assign[t] = (int32_t)arg;
        }
        if (it == iters) break;
        for (int64_t i = 0; i < C * d; ++i) sum[i] = 0.0;
        for (int64_t c = 0; c < C; ++c) cnt[c] = 0;
        for (int64_t t = 0; t < n; ++t) {
            const int64_t c = assign[t];
            cnt[c] += 1;
            for (int64_t e = 0; e < d; ++e) sum[c * d + e] += x[t * d + e];
        }
        for (int64_t c = 0; c < C; ++c)
            if (cnt[c] > 0)
                for (int64_t e = 0; e < d; ++e) cent[c * d + e] = sum[c * d + e] / (double)cnt[c];
    }
    free(sum);
    free(cnt);
}

/* Centroid top-p: for query cluster a, key cluster j is estimated to receive
 *   w[a, j] = size_k[j] exp(scale cq[a] . ck[j]) / sum_j' size_k[j'] exp(scale cq[a] . ck[j'])
 * of the attention (every key of a cluster represented by its centroid).  Key clusters are
 * taken in order of w descending (the lower id first on a tie) until the cumulative w reaches p
 * (p <= 0 takes none, p >= 1 takes every cluster with keys).  sel [Cq, Ck] 0/1. */
void or_centroid_topp(const double *cq, const double *ck, const int64_t *size_k, int64_t Cq,
                      int64_t Ck, int64_t d, double scale, double p, uint8_t *sel) {
    ranked_t *ord = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)Ck);
    double *logit = (double *)malloc(sizeof(double) * (size_t)Ck);
    for (int64_t a = 0; a < Cq; ++a) {
        double mx = -INFINITY;
        for (int64_t j = 0; j < Ck; ++j) {
            double s = 0.0;
            for (int64_t e = 0; e < d; ++e) s += cq[a * d + e] * ck[j * d + e];
            logit[j] = s * scale;
            if (size_k[j] > 0 && logit[j] > mx) mx = logit[j];
        }
        double z = 0.0;
        for (int64_t j = 0; j < Ck; ++j) {
            ord[j].p = size_k[j] > 0 ? (double)size_k[j] * exp(logit[j] - mx) : 0.0;
            ord[j].j = (int32_t)j;
            z += ord[j].p;
        }
        for (int64_t j = 0; j < Ck; ++j) ord[j].p /= z;
        qsort(ord, (size_t)Ck, sizeof(ranked_t), ranked_cmp);
        uint8_t *row = sel + a * Ck;
        for (int64_t j = 0; j < Ck; ++j) row[j] = 0;
        if (p <= 0.0) continue;
        double cum = 0.0;
        for (int64_t q = 0; q < Ck; ++q) {
            if (ord[q].p <= 0.0) break;  /* clusters without keys are never taken */
            row[ord[q].j] = 1;
            cum += ord[q].p;
            if (p < 1.0 && cum >= p) break;
        }
    }
    free(ord);
    free(logit);
}

/* Attention of every query token over the keys of the clusters its cluster selected:
 *   O[t] = sum_{s : sel[aq[t], ak[s]]} softmax_s(scale q[t] . k[s]) v[s]
 * (zero when the selection is empty).  q, k, v: [n, d] bf16 bits of one head; out [n, d]. */
void or_cluster_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t n,
                          int64_t d, const int32_t *aq, const int32_t *ak, const uint8_t *sel,
                          int64_t Ck, double scale, double *out) {
    double *w = (double *)malloc(sizeof(double) * (size_t)n);
    for (int64_t t = 0; t < n; ++t) {
        const uint8_t *row = sel + (int64_t)aq[t] * Ck;
        double mx = -INFINITY;
        for (int64_t s = 0; s < n; ++s) {
            if (!row[ak[s]]) continue;
            double x = 0.0;
            for (int64_t c = 0; c < d; ++c) x += bf16_to_double(q[t * d + c]) * bf16_to_double(k[s * d + c]);
            w[s] = x * scale;
            if (w[s] > mx) mx = w[s];
        }
        double z = 0.0;
        double *o = out + t * d;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        for (int64_t s = 0; s < n; ++s) {
            if (!row[ak[s]]) continue;
            const double e = exp(w[s] - mx);
            z += e;
            for (int64_t c = 0; c < d; ++c) o[c] += e * bf16_to_double(v[s * d + c]);
        }
        if (z > 0.0)
            for (int64_t c = 0; c < d; ++c) o[c] /= z;
    }
    free(w);
}
