/*
 * pba_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what the pair-biased attention path
 * computes.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg load this file (through oracle/__init__.py); the CUDA library never
 * links, includes or calls it, and it shares no code, header or constant with
 * the library.  Every loop here follows the plain definition; there is no
 * blocking, fusion or reordering beyond what the definition states.
 *
 * Sources (the pages give names and complexities; the formula itself is the
 * plain reading of the cited titles):
 *   - "Fold-CP: A Context Parallelism Framework for Biomolecular Modeling",
 *     Table 1 (rows "Attn Pair Bias (Ring)" and "Triangle Attention": serial
 *     time B*H*N^2*D and B*H*N^3*D) and Figure 2 (a) and (c): attention whose
 *     logits carry an additive pair bias, computed per block of keys and
 *     combined by a tiled-softmax merge; triangle attention as the same
 *     operation along one axis of the pair tensor, with a cross-axis
 *     transpose of the triangular bias for the ending node.
 *   - "Design-CP: Context Parallelism for Design of Protein Nanoparticles",
 *     the "Builds on" list: "Online normalizer calculation for softmax" and
 *     "Self-attention Does Not Need O(n2) Memory" (a softmax over keys
 *     computed block by block keeps, per query row, a running maximum m, a
 *     running sum l of exp(s - m) and an output normalised by l).
 *
 * Definition used throughout (natural logarithms, fp64):
 *   s_j   = tau * sum_d q_d k_jd + b_j        for keys j in V (valid keys)
 *   V     = { j : key mask_j != 0 and b_j != -inf }
 *   m     = max_{j in V} s_j
 *   l     = sum_{j in V} exp(s_j - m)
 *   O     = sum_{j in V} exp(s_j - m) v_j / l
 *   lse   = m + ln l
 * An empty V gives m = -inf, l = 0, O = 0, lse = -inf.
 *
 * Parity is pinned by the CPU tests in tests/test_oracle_pins.py (library
 * attention in fp64, brute force, closed forms, invariants, a hand-derived
 * worked example and planted-mistake checks).
 *
 * A planted mistake for those checks can be compiled in with
 * -DORACLE_MUTANT=<n>; the default build (no macro) has none.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* ------------------------------------------------------------------ */
/* Simple row-parallel driver: rows [0, nrows) are split into nthreads  */
/* contiguous ranges, one pthread each.                                 */
/* ------------------------------------------------------------------ */
typedef void (*row_fn)(const void *ctx, int64_t row, double *scratch);

typedef struct {
  row_fn fn;
  const void *ctx;
  int64_t begin, end;
  int64_t scratch_len;
} row_job;

static void *run_rows(void *arg) {
  row_job *job = (row_job *)arg;
  double *scratch = (double *)malloc(sizeof(double) * (size_t)(job->scratch_len > 0 ? job->scratch_len : 1));
  if (!scratch) return NULL;
  for (int64_t r = job->begin; r < job->end; ++r) job->fn(job->ctx, r, scratch);
  free(scratch);
  return NULL;
}

static int default_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

static void parallel_rows(row_fn fn, const void *ctx, int64_t nrows, int64_t scratch_len, int nthreads) {
  int nt = default_threads(nthreads);
  if (nt > nrows) nt = (int)(nrows > 0 ? nrows : 1);
  row_job *jobs = (row_job *)calloc((size_t)nt, sizeof(row_job));
  pthread_t *tids = (pthread_t *)calloc((size_t)nt, sizeof(pthread_t));
  for (int t = 0; t < nt; ++t) {
    jobs[t].fn = fn;
    jobs[t].ctx = ctx;
    jobs[t].begin = nrows * t / nt;
    jobs[t].end = nrows * (t + 1) / nt;
    jobs[t].scratch_len = scratch_len;
  }
  for (int t = 1; t < nt; ++t) pthread_create(&tids[t], NULL, run_rows, &jobs[t]);
  run_rows(&jobs[0]);
  for (int t = 1; t < nt; ++t) pthread_join(tids[t], NULL);
  free(jobs);
  free(tids);
}

int oracle_threads_used(int nthreads) { return default_threads(nthreads); }

/* ------------------------------------------------------------------ */
/* One query row against keys [k0, k1): the definition above.          */
/*   q      : [D]            query row                                 */
/*   k, v   : [Nk][D]        keys and values (row j at k + j*D)        */
/*   brow   : [Nk]           this query's bias row                     */
/*   mask   : [Nk] or NULL   key mask, nonzero = key takes part        */
/*   s      : scratch of length Nk                                     */
/* Writes o[D], *m, *l.                                                */
/* ------------------------------------------------------------------ */
static void attend_row(int64_t D, double tau, const double *q, const double *k, const double *v,
                       const double *brow, const uint8_t *mask, int64_t k0, int64_t k1, double *s,
                       double *o, double *m_out, double *l_out) {
  double m = -INFINITY;
  for (int64_t j = k0; j < k1; ++j) {
#if ORACLE_MUTANT == 8 /* planted: key mask ignored */
    int valid = brow[j] != -INFINITY;
#else
    int valid = (mask == NULL || mask[j] != 0) && brow[j] != -INFINITY;
#endif
    if (!valid) {
      s[j] = -INFINITY;
      continue;
    }
    double dot = 0.0;
    for (int64_t d = 0; d < D; ++d) dot += q[d] * k[j * D + d];
#if ORACLE_MUTANT == 1 /* planted: bias dropped */
    s[j] = tau * dot;
#elif ORACLE_MUTANT == 2 /* planted: scale applied to the bias too */
    s[j] = tau * (dot + brow[j]);
#elif ORACLE_MUTANT == 3 /* planted: wrong sign on the bias */
    s[j] = tau * dot - brow[j];
#else
    s[j] = tau * dot + brow[j];
#endif
    if (s[j] > m) m = s[j];
  }
  for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
  if (m == -INFINITY) { /* no valid key */
    *m_out = -INFINITY;
    *l_out = 0.0;
    return;
  }
  double l = 0.0;
  for (int64_t j = k0; j < k1; ++j) {
    if (s[j] == -INFINITY) continue;
    double p = exp(s[j] - m);
    l += p;
    for (int64_t d = 0; d < D; ++d) o[d] += p * v[j * D + d];
  }
#if ORACLE_MUTANT == 4 /* planted: output not normalised */
  (void)0;
#else
  for (int64_t d = 0; d < D; ++d) o[d] /= l;
#endif
  *m_out = m;
  *l_out = l;
}

/* ------------------------------------------------------------------ */
/* Pair-biased attention, contiguous fp64 tensors:                     */
/*   q [B][H][Nq][D], k,v [B][H][Nk][D], bias [B][H][Nq][Nk],          */
/*   key_mask [B][Nk] or NULL.                                         */
/* Keys [k0, k1) take part (k0 = 0, k1 = Nk for the full pass; one     */
/* key block for a ring-step partial).                                  */
/* Outputs (any may be NULL): o [B][H][Nq][D] (normalised by l),       */
/* m, l, lse [B][H][Nq].                                               */
/* ------------------------------------------------------------------ */
typedef struct {
  int64_t B, H, Nq, Nk, D, k0, k1;
  double tau;
  const double *q, *k, *v, *bias;
  const uint8_t *mask;
  double *o, *m, *l, *lse;
} pba_ctx;

static void pba_row(const void *vctx, int64_t row, double *scratch) {
  const pba_ctx *c = (const pba_ctx *)vctx;
  int64_t i = row % c->Nq;
  int64_t bh = row / c->Nq;
  int64_t b = bh / c->H;
  double *s = scratch;
  double *o = scratch + c->Nk;
  double m, l;
  attend_row(c->D, c->tau, c->q + row * c->D, c->k + bh * c->Nk * c->D, c->v + bh * c->Nk * c->D,
             c->bias + (bh * c->Nq + i) * c->Nk, c->mask ? c->mask + b * c->Nk : NULL, c->k0, c->k1, s, o,
             &m, &l);
  if (c->o) memcpy(c->o + row * c->D, o, sizeof(double) * (size_t)c->D);
  if (c->m) c->m[row] = m;
  if (c->l) c->l[row] = l;
#if ORACLE_MUTANT == 7 /* planted: log-sum-exp without the maximum */
  if (c->lse) c->lse[row] = (l > 0.0) ? log(l) : -INFINITY;
#else
  if (c->lse) c->lse[row] = (l > 0.0) ? m + log(l) : -INFINITY;
#endif
}

int oracle_pba_range(int64_t B, int64_t H, int64_t Nq, int64_t Nk, int64_t D, double tau, const double *q,
                     const double *k, const double *v, const double *bias, const uint8_t *key_mask, int64_t k0,
                     int64_t k1, double *o, double *m, double *l, double *lse, int nthreads) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || D < 1 || k0 < 0 || k1 < k0 || k1 > Nk) return 1;
  pba_ctx c = {B, H, Nq, Nk, D, k0, k1, tau, q, k, v, bias, key_mask, o, m, l, lse};
  parallel_rows(pba_row, &c, B * H * Nq, Nk + D, nthreads);
  return 0;
}

/* Full pass over all keys: O and the log-sum-exp. */
int oracle_pba(int64_t B, int64_t H, int64_t Nq, int64_t Nk, int64_t D, double tau, const double *q,
               const double *k, const double *v, const double *bias, const uint8_t *key_mask, double *o,
               double *lse, int nthreads) {
  return oracle_pba_range(B, H, Nq, Nk, D, tau, q, k, v, bias, key_mask, 0, Nk, o, NULL, NULL, lse, nthreads);
}

/* One ring step: the partial (O_p normalised, m_p, l_p) over keys
 * [k0, k0 + L).  Figure 2(c) of the Fold-CP page: each step attends the
 * local queries to the key/value/bias block it holds. */
int oracle_pba_partial(int64_t B, int64_t H, int64_t Nq, int64_t Nk, int64_t D, double tau, const double *q,
                       const double *k, const double *v, const double *bias, const uint8_t *key_mask, int64_t k0,
                       int64_t L, double *o_p, double *m_p, double *l_p, int nthreads) {
  return oracle_pba_range(B, H, Nq, Nk, D, tau, q, k, v, bias, key_mask, k0, k0 + L, o_p, m_p, l_p, NULL,
                          nthreads);
}

/* ------------------------------------------------------------------ */
/* Tiled-softmax merge (Fold-CP, Figure 2 (a) and (c)): partials       */
/* (O_p, m_p, l_p), p = 0..P-1, each over a disjoint key block, give   */
/*   M = max_p m_p over blocks with l_p > 0                            */
/*   w_p = l_p exp(m_p - M),  L = sum_p w_p                            */
/*   O = sum_p w_p O_p / L,   lse = M + ln L                           */
/* o_parts [P][rows][D], m_parts/l_parts [P][rows]; out [rows][D],     */
/* lse [rows] (nullable).                                              */
/* ------------------------------------------------------------------ */
int oracle_merge(int64_t P, int64_t rows, int64_t D, const double *o_parts, const double *m_parts,
                 const double *l_parts, double *out, double *lse) {
  if (P < 1 || rows < 0 || D < 1) return 1;
  for (int64_t r = 0; r < rows; ++r) {
    double M = -INFINITY;
    for (int64_t p = 0; p < P; ++p) {
      double lp = l_parts[p * rows + r], mp = m_parts[p * rows + r];
      if (lp > 0.0 && mp > M) M = mp;
    }
    for (int64_t d = 0; d < D; ++d) out[r * D + d] = 0.0;
    if (M == -INFINITY) {
      if (lse) lse[r] = -INFINITY;
      continue;
    }
    double L = 0.0;
    for (int64_t p = 0; p < P; ++p) {
      double lp = l_parts[p * rows + r];
      if (!(lp > 0.0)) continue;
#if ORACLE_MUTANT == 5 /* planted: merge weight ignores the block sum */
      double w = exp(m_parts[p * rows + r] - M);
#else
      double w = lp * exp(m_parts[p * rows + r] - M);
#endif
      L += w;
      for (int64_t d = 0; d < D; ++d) out[r * D + d] += w * o_parts[(p * rows + r) * D + d];
    }
    for (int64_t d = 0; d < D; ++d) out[r * D + d] /= L;
    if (lse) lse[r] = M + log(L);
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* Triangle attention (Fold-CP Table 1 "Triangle Attention"; Figure    */
/* 2(a)).  Pair tensor projections q,k,v,g are [N][N][H][D] (pair      */
/* (i,j)), the triangular bias is [H][N][N], pair_mask [N][N].         */
/*                                                                      */
/* Starting node, for each row i:                                      */
/*   o[i][j] = sum_k softmax_k( tau q[i][j].k[i][k] + b[h][j][k] )     */
/*             v[i][k],  keys k with pair_mask[i][k] != 0              */
/* Ending node, for each column j:                                     */
/*   o[i][j] = sum_k softmax_k( tau q[i][j].k[k][j] + b[h][k][i] )     */
/*             v[k][j],  keys k with pair_mask[k][j] != 0              */
/* then out = o * sigmoid(g) when g is given.                          */
/*                                                                      */
/* The caller passes LINES: for the starting node line l is row i_l    */
/* (x_lines[l][j][h][d] = x[i_l][j][h][d], mask_lines[l][k] =          */
/* pair_mask[i_l][k]); for the ending node line l is column j_l         */
/* (x_lines[l][i][h][d] = x[i][j_l][h][d], mask_lines[l][k] =          */
/* pair_mask[k][j_l]).  The two orientations index the bias by their   */
/* own explicit formulas above; neither is derived from the other.     */
/* out_lines and lse_lines ([nl][N][H][D], [nl][N][H]) use the same    */
/* line layout.                                                        */
/* ------------------------------------------------------------------ */
typedef struct {
  int64_t N, H, D, nl;
  int ending;
  double tau;
  const double *q, *k, *v, *g, *bias;
  const uint8_t *mask;
  double *out, *lse;
} tri_ctx;

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static void tri_row(const void *vctx, int64_t row, double *scratch) {
  const tri_ctx *c = (const tri_ctx *)vctx;
  const int64_t N = c->N, H = c->H, D = c->D;
  /* row enumerates (line, query position a, head h) */
  int64_t h = row % H;
  int64_t a = (row / H) % N;
  int64_t line = row / (H * N);
  const int64_t lstride = N * H * D; /* one line of q/k/v/g */
  double *s = scratch;
  double *o = scratch + N;
  double *brow = scratch + N + D;
  /* gather the bias row this query uses */
  for (int64_t kk = 0; kk < N; ++kk) {
#if ORACLE_MUTANT == 6 /* planted: ending node reads the bias untransposed */
    brow[kk] = c->bias[(h * N + a) * N + kk];
#else
    if (!c->ending)
      brow[kk] = c->bias[(h * N + a) * N + kk]; /* b[h][j=a][k]  */
    else
      brow[kk] = c->bias[(h * N + kk) * N + a]; /* b[h][k][i=a]  */
#endif
  }
  /* keys of this line, head h: key kk at (line, kk, h) */
  const double *qrow = c->q + line * lstride + (a * H + h) * D;
  /* keys/values for head h are strided by H*D inside the line */
  double m = -INFINITY, l = 0.0;
  for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
  for (int64_t kk = 0; kk < N; ++kk) {
    int valid = (c->mask == NULL || c->mask[line * N + kk] != 0) && brow[kk] != -INFINITY;
    if (!valid) {
      s[kk] = -INFINITY;
      continue;
    }
    const double *krow = c->k + line * lstride + (kk * H + h) * D;
    double dot = 0.0;
    for (int64_t d = 0; d < D; ++d) dot += qrow[d] * krow[d];
    s[kk] = c->tau * dot + brow[kk];
    if (s[kk] > m) m = s[kk];
  }
  if (m != -INFINITY) {
    for (int64_t kk = 0; kk < N; ++kk) {
      if (s[kk] == -INFINITY) continue;
      double p = exp(s[kk] - m);
      l += p;
      const double *vrow = c->v + line * lstride + (kk * H + h) * D;
      for (int64_t d = 0; d < D; ++d) o[d] += p * vrow[d];
    }
    for (int64_t d = 0; d < D; ++d) o[d] /= l;
  }
  double *orow = c->out + line * lstride + (a * H + h) * D;
  for (int64_t d = 0; d < D; ++d) {
#if ORACLE_MUTANT == 9 /* planted: gate applied without the sigmoid */
    double gate = c->g ? c->g[line * lstride + (a * H + h) * D + d] : 1.0;
#else
    double gate = c->g ? sigmoid(c->g[line * lstride + (a * H + h) * D + d]) : 1.0;
#endif
    orow[d] = o[d] * gate;
  }
  if (c->lse) c->lse[(line * N + a) * H + h] = (l > 0.0) ? m + log(l) : -INFINITY;
}

int oracle_tri_attn_lines(int64_t N, int64_t H, int64_t D, int ending, double tau, int64_t nl, const double *q_lines,
                          const double *k_lines, const double *v_lines, const double *g_lines, const double *bias,
                          const uint8_t *mask_lines, double *out_lines, double *lse_lines, int nthreads) {
  if (N < 0 || H < 1 || D < 1 || nl < 0) return 1;
  tri_ctx c = {N, H, D, nl, ending ? 1 : 0, tau, q_lines, k_lines, v_lines, g_lines, bias, mask_lines, out_lines,
               lse_lines};
  parallel_rows(tri_row, &c, nl * N * H, 2 * N + D, nthreads);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Triangle projections (Fold-CP, Figure 2(a): the pair tensor z gives  */
/* the queries, keys, values, gate and the per-head bias of triangle     */
/* attention).  For every pair row r = (i, j) of z [N*N][c]:            */
/*   out[r][f] = sum_c z[r][c] * w[c][f]     f < F (w [c][F])           */
/*   bias[h][r] = sum_c z[r][c] * wb[c][h]   h < H (wb [c][H])           */
/* i.e. q|k|v|g are the column blocks of out, and the bias is laid out   */
/* [H][N][N].  Plain fp64 dot products, one pair row per call.           */
/* ------------------------------------------------------------------ */
typedef struct {
  int64_t c, F, H;
  const double *z, *w, *wb;
  double *out, *bias;
  int64_t rows;
} proj_ctx;

static void proj_row(const void *vctx, int64_t r, double *scratch) {
  (void)scratch;
  const proj_ctx *x = (const proj_ctx *)vctx;
  const double *zr = x->z + r * x->c;
  for (int64_t f = 0; f < x->F; ++f) {
    double acc = 0.0;
    for (int64_t cc = 0; cc < x->c; ++cc)
#if ORACLE_MUTANT == 10 /* planted: weight read transposed */
      acc += zr[cc] * x->w[(f % x->c) * x->F + (cc % x->F)];
#else
      acc += zr[cc] * x->w[cc * x->F + f];
#endif
    x->out[r * x->F + f] = acc;
  }
  for (int64_t h = 0; h < x->H; ++h) {
    double acc = 0.0;
    for (int64_t cc = 0; cc < x->c; ++cc)
#if ORACLE_MUTANT == 11 /* planted: bias taken from the first weight columns */
      acc += zr[cc] * x->w[cc * x->F + h];
#else
      acc += zr[cc] * x->wb[cc * x->H + h];
#endif
    x->bias[h * x->rows + r] = acc;
  }
}

int oracle_tri_proj(int64_t rows, int64_t c, int64_t F, int64_t H, const double *z, const double *w,
                    const double *wb, double *out, double *bias, int nthreads) {
  if (rows < 0 || c < 1 || F < 0 || H < 0) return 1;
  proj_ctx x = {c, F, H, z, w, wb, out, bias, rows};
  parallel_rows(proj_row, &x, rows, 1, nthreads);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Pair weighted averaging (Fold-CP, Table 1 row "Pair Weighted Avg.": */
/* serial time B*H*S*N^2*D, distributed as a "2D ring + tiled softmax", */
/* and Figure 2, which groups it with the ring attention: a softmax    */
/* whose per-block partials are merged).  The pages give no formula; the reading used here is a   */
/* softmax over the pair-bias logits alone, shared by the S sequences:  */
/*   w[h][i][j] = exp(b[h][i][j] - m) / l  over valid keys j            */
/*     (m = max, l = sum of exp(b - m) over valid j of row (h, i))      */
/*   o[s][i][h][:] = sum_j w[h][i][j] v[s][j][h][:]                      */
/*   out = o * sigmoid(g) when a gate is given; lse[h][i] = m + ln l.   */
/* v, g, out [S][N][H][D]; bias [H][N][N]; key mask [N] or NULL.        */
/* ------------------------------------------------------------------ */
typedef struct {
  int64_t S, N, H, D;
  const double *v, *bias, *g;
  const uint8_t *mask;
  double *out, *lse;
} pwa_ctx;

static void pwa_row(const void *vctx, int64_t row, double *w) {
  const pwa_ctx *x = (const pwa_ctx *)vctx;
  const int64_t h = row / x->N, i = row % x->N, N = x->N, H = x->H, D = x->D;
  const double *brow = x->bias + (h * N + i) * N;
  double m = -INFINITY, l = 0.0;
  for (int64_t j = 0; j < N; ++j) {
    int valid = (x->mask == NULL || x->mask[j] != 0) && brow[j] != -INFINITY;
#if ORACLE_MUTANT == 12 /* planted: key mask ignored */
    valid = brow[j] != -INFINITY;
#endif
    w[j] = valid ? brow[j] : -INFINITY;
    if (w[j] > m) m = w[j];
  }
  if (m != -INFINITY)
    for (int64_t j = 0; j < N; ++j) {
      w[j] = (w[j] == -INFINITY) ? 0.0 : exp(w[j] - m);
      l += w[j];
    }
  for (int64_t s = 0; s < x->S; ++s) {
    for (int64_t d = 0; d < D; ++d) {
      double acc = 0.0;
      if (l > 0.0)
        for (int64_t j = 0; j < N; ++j)
#if ORACLE_MUTANT == 13 /* planted: values of sequence 0 for every sequence */
          acc += w[j] * x->v[((0 * N + j) * H + h) * D + d];
#else
          acc += w[j] * x->v[((s * N + j) * H + h) * D + d];
#endif
      const double o = (l > 0.0) ? acc / l : 0.0;
      const int64_t at = ((s * N + i) * H + h) * D + d;
      x->out[at] = x->g ? o * sigmoid(x->g[at]) : o;
    }
  }
  if (x->lse) x->lse[h * N + i] = (l > 0.0) ? m + log(l) : -INFINITY;
}

int oracle_pwa(int64_t S, int64_t N, int64_t H, int64_t D, const double *v, const double *bias, const double *g,
               const uint8_t *mask, double *out, double *lse, int nthreads) {
  if (S < 0 || N < 0 || H < 1 || D < 1) return 1;
  pwa_ctx x = {S, N, H, D, v, bias, g, mask, out, lse};
  parallel_rows(pwa_row, &x, H * N, N, nthreads);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Backward of pair-biased attention (training is distributed too:     */
/* Fold-CP, Figure 3 right, training scaling).  For one (b, h), with    */
/* s_ij = tau q_i.k_j + b_ij over valid keys and P_ij = exp(s_ij - lse_i)*/
/* (0 for invalid keys), given dO = dL/dO:                              */
/*   O_i      = sum_j P_ij v_j                                          */
/*   Delta_i  = sum_d dO_id O_id                                        */
/*   dP_ij    = dO_i . v_j                                              */
/*   dS_ij    = P_ij (dP_ij - Delta_i)        = dL/ds_ij = dL/db_ij     */
/*   dq_i     = tau sum_j dS_ij k_j,  dk_j = tau sum_i dS_ij q_i        */
/*   dv_j     = sum_i P_ij dO_i                                         */
/* Contiguous fp64: q, dO [B][H][Nq][D]; k, v [B][H][Nk][D]; bias and    */
/* dbias [B][H][Nq][Nk]; key_mask [B][Nk] or NULL.  One (b, h) per call  */
/* of the row function; dbias of invalid keys is 0.                     */
/* ------------------------------------------------------------------ */
typedef struct {
  int64_t B, H, Nq, Nk, D;
  double tau;
  const double *q, *k, *v, *bias, *dout;
  const uint8_t *mask;
  double *dq, *dk, *dv, *dbias;
} bwd_ctx;

static void bwd_bh(const void *vctx, int64_t bh, double *scratch) {
  const bwd_ctx *c = (const bwd_ctx *)vctx;
  const int64_t Nq = c->Nq, Nk = c->Nk, D = c->D, b = bh / c->H;
  const double *q = c->q + bh * Nq * D, *k = c->k + bh * Nk * D, *v = c->v + bh * Nk * D;
  const double *bias = c->bias + bh * Nq * Nk, *dout = c->dout + bh * Nq * D;
  const uint8_t *mask = c->mask ? c->mask + b * Nk : NULL;
  double *dq = c->dq + bh * Nq * D, *dk = c->dk + bh * Nk * D, *dv = c->dv + bh * Nk * D;
  double *dbias = c->dbias + bh * Nq * Nk;
  double *p = scratch, *o = scratch + Nk;
  for (int64_t x = 0; x < Nk * D; ++x) dk[x] = dv[x] = 0.0;
  for (int64_t i = 0; i < Nq; ++i) {
    double m = -INFINITY;
    for (int64_t j = 0; j < Nk; ++j) {
      const int valid = (mask == NULL || mask[j] != 0) && bias[i * Nk + j] != -INFINITY;
      double s = -INFINITY;
      if (valid) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += q[i * D + d] * k[j * D + d];
        s = c->tau * dot + bias[i * Nk + j];
      }
      p[j] = s;
      if (s > m) m = s;
    }
    double l = 0.0;
    for (int64_t j = 0; j < Nk; ++j) {
      p[j] = (p[j] == -INFINITY) ? 0.0 : exp(p[j] - m);
      l += p[j];
    }
    for (int64_t j = 0; j < Nk; ++j) p[j] = (l > 0.0) ? p[j] / l : 0.0;
    for (int64_t d = 0; d < D; ++d) {
      o[d] = 0.0;
      for (int64_t j = 0; j < Nk; ++j) o[d] += p[j] * v[j * D + d];
    }
    double delta = 0.0;
    for (int64_t d = 0; d < D; ++d) delta += dout[i * D + d] * o[d];
    for (int64_t d = 0; d < D; ++d) dq[i * D + d] = 0.0;
    for (int64_t j = 0; j < Nk; ++j) {
      double dp = 0.0;
      for (int64_t d = 0; d < D; ++d) dp += dout[i * D + d] * v[j * D + d];
#if ORACLE_MUTANT == 14 /* planted: the row term Delta dropped */
      const double ds = p[j] * dp;
#else
      const double ds = p[j] * (dp - delta);
#endif
      dbias[i * Nk + j] = ds;
      for (int64_t d = 0; d < D; ++d) {
        dq[i * D + d] += c->tau * ds * k[j * D + d];
#if ORACLE_MUTANT == 15 /* planted: dk without the scale */
        dk[j * D + d] += ds * q[i * D + d];
#else
        dk[j * D + d] += c->tau * ds * q[i * D + d];
#endif
        dv[j * D + d] += p[j] * dout[i * D + d];
      }
    }
  }
}

int oracle_pba_backward(int64_t B, int64_t H, int64_t Nq, int64_t Nk, int64_t D, double tau, const double *q,
                        const double *k, const double *v, const double *bias, const uint8_t *key_mask,
                        const double *dout, double *dq, double *dk, double *dv, double *dbias, int nthreads) {
  if (B < 1 || H < 1 || Nq < 0 || Nk < 0 || D < 1) return 1;
  bwd_ctx c = {B, H, Nq, Nk, D, tau, q, k, v, bias, dout, key_mask, dq, dk, dv, dbias};
  parallel_rows(bwd_bh, &c, B * H, Nk + D, nthreads);
  return 0;
}
