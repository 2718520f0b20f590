/*
 * HiLS attention forward -- CPU oracle (test infrastructure only).
 *
 * This file is the plain, slow, fp64 statement of what the HiLS forward pass
 * computes.  It is the checker for the CUDA library and is used only by the
 * tests, by the smoke check and by the CPU-baseline leg of the benchmark.  It
 * shares no code, header or constant with the CUDA path; the product never
 * links or calls it.
 *
 * Sources (web pages on "Hierarchical Sparse Attention Done Right: Toward
 * Infinite Context Modeling", HiLS):
 *   [MC]  axforge.ai model card "HiLS-Attention", section "What HiLS-Attention
 *         is": chunk-mass surrogate from compressed chunk (landmark) keys,
 *         attention factorised into an inter-chunk and an intra-chunk softmax,
 *         top-k chunk selection; the naive alternative selects by exact chunk
 *         mass from a full QK product.
 *   [AW]  aiweekly.co "HiLS Attention Extrapolates 64x at 90% Retrieval
 *         Accuracy", paragraph on the mechanism: each query attends to each
 *         retrieved chunk independently and the per-chunk outputs are fused by
 *         the chunk retrieval scores.
 *   [KR]  molayo1419.me "HiLS Attention: ..." (Korean), section "Core idea:
 *         landmark tokens and hierarchical factorization": step 1 inter-chunk
 *         attention over the landmark keys gives a distribution over chunks;
 *         step 2 standard attention inside the selected chunks.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - completed chunks of query t are c < floor(t/C); the query's own chunk
 *     floor(t/C) is always attended, causally (keys j <= t), and its fusion
 *     logit is the log-sum-exp of its own causal scores (its exact log mass);
 *     it does not use a top-k slot;
 *   - landmark logits use the token softmax scale;
 *   - selection key is (score descending, chunk index ascending); the decision
 *     is taken on the score rounded to fp32, the precision the GPU kernels
 *     decide in; all other arithmetic is fp64;
 *   - fusion weights are a softmax over {selected landmark logits} plus the
 *     own-chunk logit (the global inter-chunk denominator cancels);
 *   - rows with fewer than k completed chunks select all of them.
 *
 * Parity status of each entry point is stated in the test suite header
 * (tests/test_oracle_pins.py); every function here is pinned by at least one
 * closed form or brute-force case there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Element load: inputs are stored either as fp32 or as bf16 bit patterns.
 * A bf16 value is the upper 16 bits of an fp32 value, so the widening is
 * exact. */
static double ld(const void *base, int64_t i, int bf16) {
  if (bf16) {
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)base)[i];
}

typedef struct {
  int B, Hq, Hkv, L, d, C, topk;
  double scale;
  int bf16;                /* element format of q, k, v, lmk */
  const void *k, *v, *lmk; /* [B,Hkv,L,d], [B,Hkv,L,d], [B,Hkv,floor(L/C),d] */
} problem;

/* dot(q_t, row r of a [.., d] array), fp64, sequential over the d axis */
static double dot(const double *qt, const void *a, int64_t row, int d, int bf16) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) s += qt[i] * ld(a, row * (int64_t)d + i, bf16);
  return s;
}

/* Intra-chunk attention [KR step 2]: keys j in [j0, j1) of head (b, hkv).
 * Returns lse_c = log sum_j exp(x_j) with x_j = scale * <q_t, k_j>, and
 * writes o_c = sum_j softmax(x)_j v_j into o (length d). */
static double chunk_attend(const problem *P, const double *qt, int b, int hkv,
                           int j0, int j1, double *o, double *xbuf) {
  const int64_t head_row = ((int64_t)b * P->Hkv + hkv) * P->L;
  double m = -INFINITY;
  for (int j = j0; j < j1; ++j) {
    xbuf[j - j0] = P->scale * dot(qt, P->k, head_row + j, P->d, P->bf16);
    if (xbuf[j - j0] > m) m = xbuf[j - j0];
  }
  double l = 0.0;
  for (int j = j0; j < j1; ++j) l += exp(xbuf[j - j0] - m);
  const double lse = m + log(l);
  for (int i = 0; i < P->d; ++i) o[i] = 0.0;
  for (int j = j0; j < j1; ++j) {
    const double p = exp(xbuf[j - j0] - lse);
    for (int i = 0; i < P->d; ++i)
      o[i] += p * ld(P->v, (head_row + j) * (int64_t)P->d + i, P->bf16);
  }
  return lse;
}

typedef struct {
  double s;  /* score (fp64) */
  float s32; /* score rounded to fp32: the precision the selection is decided in */
  int c;     /* chunk index */
} cand;

/* Selection order [MC "selects top-k chunks"]: higher score first; on equal
 * (fp32) scores the lower chunk index first. */
static int by_score_desc(const void *pa, const void *pb) {
  const cand *a = (const cand *)pa, *b = (const cand *)pb;
  if (a->s32 > b->s32) return -1;
  if (a->s32 < b->s32) return 1;
  return (a->c > b->c) - (a->c < b->c);
}
static int by_chunk_asc(const void *pa, const void *pb) {
  const cand *a = (const cand *)pa, *b = (const cand *)pb;
  return (a->c > b->c) - (a->c < b->c);
}

enum { MODE_LANDMARK = 0, MODE_GIVEN = 1, MODE_EXACT_MASS = 2 };

/* One query row (b, hq, t) with query vector qt (already widened to fp64).
 *  mode MODE_LANDMARK : score completed chunks by their landmark keys [KR step 1]
 *  mode MODE_GIVEN    : use the selection sel_in / logits w_in (padding -1)
 *  mode MODE_EXACT_MASS: score completed chunks by their exact log mass
 *                        lse_c(t) -- the naive selector of [MC]
 * Outputs (any may be NULL): sel[k] (ascending chunk ids, -1 pad), w[k]
 * (selected logits, -inf pad), *lse_lmk (log-sum-exp over all completed
 * landmark logits; -inf if none), out[d], *lse, wfin[k+1] (fusion weights of
 * the selected chunks in sel order, own chunk last). */
static void ref_row(const problem *P, const double *qt, int b, int hq, int t, int mode,
                    const int32_t *sel_in, const double *w_in, int32_t *sel, double *w,
                    double *lse_lmk, double *out, double *lse, double *wfin) {
  const int C = P->C, d = P->d, k = P->topk;
  const int hkv = hq / (P->Hq / P->Hkv);
  const int own = t / C;
  const int n_c = own; /* completed chunks: c < floor(t/C) */
  double *xbuf = (double *)malloc(sizeof(double) * (size_t)C);
  double *oc = (double *)malloc(sizeof(double) * (size_t)d);
  cand *cs = (cand *)malloc(sizeof(cand) * (size_t)(n_c > 0 ? n_c : 1));
  int nsel = 0;

  if (mode == MODE_GIVEN) {
    for (int i = 0; i < k; ++i)
      if (sel_in[i] >= 0) {
        cs[nsel].c = sel_in[i];
        cs[nsel].s = w_in[i];
        cs[nsel].s32 = (float)w_in[i];
        ++nsel;
      }
    qsort(cs, (size_t)nsel, sizeof(cand), by_chunk_asc);
    if (lse_lmk) *lse_lmk = NAN; /* not defined without the landmark scores */
  } else {
    const int64_t lmk_head = ((int64_t)b * P->Hkv + hkv) * (P->L / C);
    for (int c = 0; c < n_c; ++c) {
      double s;
      if (mode == MODE_LANDMARK)
        s = P->scale * dot(qt, P->lmk, lmk_head + c, d, P->bf16);
      else
        s = chunk_attend(P, qt, b, hkv, c * C, c * C + C, oc, xbuf);
      cs[c].s = s;
      cs[c].s32 = (float)s;
      cs[c].c = c;
    }
    if (lse_lmk) { /* inter-chunk softmax normaliser [MC], [KR step 1] */
      double m = -INFINITY, l = 0.0;
      for (int c = 0; c < n_c; ++c) if (cs[c].s > m) m = cs[c].s;
      if (n_c > 0) {
        for (int c = 0; c < n_c; ++c) l += exp(cs[c].s - m);
        *lse_lmk = m + log(l);
      } else {
        *lse_lmk = -INFINITY;
      }
    }
    qsort(cs, (size_t)n_c, sizeof(cand), by_score_desc);
    nsel = n_c < k ? n_c : k;
    qsort(cs, (size_t)nsel, sizeof(cand), by_chunk_asc);
  }

  if (sel)
    for (int i = 0; i < k; ++i) sel[i] = i < nsel ? cs[i].c : -1;
  if (w)
    for (int i = 0; i < k; ++i) w[i] = i < nsel ? cs[i].s : -INFINITY;

  /* Own chunk: causal keys [own*C, t], logit = its exact log mass. */
  double *acc = (double *)calloc((size_t)(nsel + 1) * (size_t)d, sizeof(double));
  double *g = (double *)malloc(sizeof(double) * (size_t)(nsel + 1));
  for (int i = 0; i < nsel; ++i) {
    const int c = cs[i].c;
    (void)chunk_attend(P, qt, b, hkv, c * C, c * C + C, acc + (size_t)i * d, xbuf);
    g[i] = cs[i].s;
  }
  g[nsel] = chunk_attend(P, qt, b, hkv, own * C, t + 1, acc + (size_t)nsel * d, xbuf);

  /* Fusion [AW]: softmax over the logits of the attended chunks. */
  double m = -INFINITY;
  for (int i = 0; i <= nsel; ++i) if (g[i] > m) m = g[i];
  double l = 0.0;
  for (int i = 0; i <= nsel; ++i) l += exp(g[i] - m);
  const double lse_row = m + log(l);
  if (lse) *lse = lse_row;
  if (out) {
    for (int e = 0; e < d; ++e) out[e] = 0.0;
    for (int i = 0; i <= nsel; ++i) {
      const double wi = exp(g[i] - lse_row);
      for (int e = 0; e < d; ++e) out[e] += wi * acc[(size_t)i * d + e];
    }
  }
  if (wfin) {
    for (int i = 0; i < k; ++i) wfin[i] = i < nsel ? exp(g[i] - lse_row) : 0.0;
    wfin[k] = exp(g[nsel] - lse_row);
  }
  free(g);
  free(acc);
  free(cs);
  free(oc);
  free(xbuf);
}

/* Widen the query vector for row (b, hq, t); q_is_decode selects the
 * [B,Hq,d] decode layout (one query per head, position t = L-1). */
static void load_q(const problem *P, const void *q, int q_is_decode, int b, int hq, int t,
                   double *qt) {
  const int64_t row = q_is_decode ? ((int64_t)b * P->Hq + hq)
                                  : (((int64_t)b * P->Hq + hq) * P->L + t);
  for (int i = 0; i < P->d; ++i) qt[i] = ld(q, row * (int64_t)P->d + i, P->bf16);
}

/* Decode a flat row index.  Prefill (q_decode = 0): rows are
 * (b*Hq + hq)*L + t and q is [B,Hq,L,d].  Decode (q_decode = 1): rows are
 * heads b*Hq + hq, q is [B,Hq,d], and the query sits at position t = L-1 of a
 * cache of length L that already holds the new token. */
static int row_of(const problem *P, int q_decode, int64_t flat, int *b, int *hq, int *t) {
  if (q_decode) {
    if (flat < 0 || flat >= (int64_t)P->B * P->Hq) return 0;
    *hq = (int)(flat % P->Hq);
    *b = (int)(flat / P->Hq);
    *t = P->L - 1;
  } else {
    if (flat < 0 || flat >= (int64_t)P->B * P->Hq * P->L) return 0;
    *t = (int)(flat % P->L);
    *hq = (int)((flat / P->L) % P->Hq);
    *b = (int)(flat / ((int64_t)P->L * P->Hq));
  }
  return 1;
}

/*
 * Rows of the forward pass (see row_of for the row numbering).  Every output
 * pointer may be NULL; per-row outputs are packed in the order of rows[].
 * Returns 0, or -1 on an invalid argument.
 */
int hils_oracle_rows(int B, int Hq, int Hkv, int L, int d, int C, int topk, double scale,
                     int bf16, int q_decode, const void *q, const void *k, const void *v,
                     const void *lmk, int64_t nrows, const int64_t *rows, int mode,
                     const int32_t *sel_in, const double *w_in, int32_t *sel_out, double *w_out,
                     double *lse_lmk_out, double *out, double *lse_out, double *wfin_out,
                     int nthreads) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || L < 1 || d < 1 || C < 1 || topk < 1)
    return -1;
  if (mode == MODE_GIVEN && (!sel_in || !w_in)) return -1;
  problem P = {B, Hq, Hkv, L, d, C, topk, scale, bf16, k, v, lmk};
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int b, hq, t;
    if (!row_of(&P, q_decode, rows[r], &b, &hq, &t)) { bad = 1; continue; }
    double *qt = (double *)malloc(sizeof(double) * (size_t)d);
    load_q(&P, q, q_decode, b, hq, t, qt);
    ref_row(&P, qt, b, hq, t, mode, sel_in ? sel_in + r * topk : NULL,
            w_in ? w_in + r * topk : NULL, sel_out ? sel_out + r * topk : NULL,
            w_out ? w_out + r * topk : NULL, lse_lmk_out ? lse_lmk_out + r : NULL,
            out ? out + r * d : NULL, lse_out ? lse_out + r : NULL,
            wfin_out ? wfin_out + r * (topk + 1) : NULL);
    free(qt);
  }
  return bad ? -1 : 0;
}

/*
 * Chunk union [KR, "hardware-efficient kernel": the union of the chunks
 * selected by M adjacent queries is loaded once].  For the group of query rows
 * [g*M, min((g+1)*M, L)) of head (b, hq): the sorted set of all selected
 * chunk ids of those rows together with each row's own chunk.  sel is
 * [nrows_total, topk] for all B*Hq*L rows.  Writes the set to u (capacity
 * cap) and returns its size, or -1 if it does not fit.
 */
int64_t hils_oracle_union(int L, int C, int topk, int M, int64_t head, int64_t g,
                          const int32_t *sel, int32_t *u, int64_t cap) {
  const int nchunks = (L + C - 1) / C;
  unsigned char *mark = (unsigned char *)calloc((size_t)nchunks, 1);
  for (int64_t t = g * M; t < (g + 1) * M && t < L; ++t) {
    const int32_t *row = sel + (head * L + t) * (int64_t)topk;
    for (int i = 0; i < topk; ++i)
      if (row[i] >= 0 && row[i] < nchunks) mark[row[i]] = 1;
    mark[t / C] = 1;
  }
  int64_t n = 0;
  for (int c = 0; c < nchunks; ++c)
    if (mark[c]) {
      if (n < cap) u[n] = c;
      ++n;
    }
  free(mark);
  return n <= cap ? n : -1;
}

/*
 * Landmark logits of every completed chunk of each row [KR step 1]:
 * s[r][c] = scale * <q_t, lmk_c> for c < floor(t/C); entries c >= floor(t/C)
 * are set to -inf.  s is [nrows, ncols]; ncols must be >= floor(L/C).
 * Row numbering as in hils_oracle_rows.  The tests use these logits to
 * enumerate the selections admissible at a near-tie.
 */
int hils_oracle_scores(int B, int Hq, int Hkv, int L, int d, int C, double scale, int bf16,
                       int q_decode, const void *q, const void *lmk, int64_t nrows,
                       const int64_t *rows, double *s, int ncols, int nthreads) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || L < 1 || d < 1 || C < 1 || ncols < L / C)
    return -1;
  problem P = {B, Hq, Hkv, L, d, C, 1, scale, bf16, NULL, NULL, lmk};
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int b, hq, t;
    if (!row_of(&P, q_decode, rows[r], &b, &hq, &t)) { bad = 1; continue; }
    const int hkv = hq / (Hq / Hkv);
    double *qt = (double *)malloc(sizeof(double) * (size_t)d);
    load_q(&P, q, q_decode, b, hq, t, qt);
    const int64_t lmk_head = ((int64_t)b * Hkv + hkv) * (L / C);
    for (int c = 0; c < ncols; ++c)
      s[r * ncols + c] = c < t / C ? scale * dot(qt, lmk, lmk_head + c, d, bf16) : -INFINITY;
    free(qt);
  }
  return bad ? -1 : 0;
}
