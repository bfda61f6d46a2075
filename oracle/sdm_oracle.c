/*
 * sdm_oracle.c -- CPU oracle of the Sparse Delta Memory (SDM) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg load this library.  It shares no
 * code, header, table or helper with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it computes (source: the SDM technical summaries of arXiv 2607.07386 on
 * gist.science, Spanish "Resumen Tecnico: Memoria Delta Dispersa (SDM)" and
 * French "Resume Technique : Memoire Delta Creuse (SDM)", section
 * "Mecanismo Central" / "Mecanisme Central", items 1-4), for every (b,h) head
 * and every step t, in the pages' order:
 *
 *  item 1  a slot table M in R^{N x d_v}, N = n^2 (float32 state);
 *  item 2  k'_t and q'_t are cut into two contiguous halves; each half is
 *          scored against its sub-key codebook (C1 for the first half, C2 for
 *          the second); each half keeps its top-k; the k x k "outer sum"
 *          candidates give slot i = i1*n + i2 with score s1[i1] + s2[i2]; the
 *          top-W candidates of k' are the write slots, the top-R of q' the read
 *          slots (topk(s1 (+) s2) = topk(topk(s1) (+) topk(s2)));
 *  item 3  for each write slot: forget gate  M~[i] = alpha_t * M[i],
 *          delta update M[i] = M~[i] + beta_t * w_i * (v_t - M~[i]);
 *          every other slot is left unchanged;
 *  item 4  the output is the weighted sum of the R read slots.
 *
 * Readings where the pages are silent, each stated here:
 *  - half scores are dot products taken in float64 from the exact input
 *    values, then rounded to float32 ("fp32 scores");
 *  - ordering is (score descending, index ascending): the lower index wins a
 *    tie, for the half top-k (codebook row index) and for slots (slot index);
 *  - candidate score = float32 sum of the two float32 half scores;
 *  - the per-slot weight k_t^(i) of item 3 is w = softmax over the W selected
 *    write scores; the read weights are u = softmax over the R selected read
 *    scores; softmax in float64 with the maximum subtracted, no temperature;
 *  - the update is evaluated as (1 - c) * M~ + c * v_t with c = beta_t * w_i,
 *    which is item 3's expression regrouped; float64, rounded to float32;
 *  - alpha_t, beta_t are per (b,h,t) scalars;
 *  - the read of step t happens after the write of step t;
 *  - o_t = sum_r u_r * M_t[r] in float64 in selection-rank order, rounded to
 *    float32.
 *
 * Near-tie flags (for the parity tests): bit 0 / bit 3 when the float64 gap
 * between the W-th and (W+1)-th (R-th and (R+1)-th) candidate is below 1e-5
 * relative; bits 1,2 / 4,5 when the same holds at the k-th/(k+1)-th entry of
 * half 1, half 2 of the key (query).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int B, H, T, d_qk, d_v, n_sub, k, W, R;
  int rule; /* write rule: 0 = gated delta (item 3), 1 = selective decay (Raven) */
} odims_t;

typedef struct {
  float s;   /* float32 score */
  int id;    /* codebook row */
} half_t;

typedef struct {
  float s;        /* float32 candidate score */
  int64_t slot;   /* i1 * n + i2 */
  double s64;     /* float64 candidate score, for near-tie flags only */
} cand_t;

static int cmp_half(const void* pa, const void* pb) {
  const half_t* a = (const half_t*)pa;
  const half_t* b = (const half_t*)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->id < b->id) ? -1 : (a->id > b->id);
}

static int cmp_cand(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->slot < b->slot) ? -1 : (a->slot > b->slot);
}

static int near_tie(double a, double b) {
  double m = fabs(a) > fabs(b) ? fabs(a) : fabs(b);
  return fabs(a - b) < 1e-5 * m;
}

typedef struct {
  double* s64_1;
  double* s64_2;
  half_t* h1;
  half_t* h2;
  cand_t* cand;
} scratch_t;

static int scratch_init(scratch_t* w, const odims_t* d) {
  int n = d->n_sub, k = d->k;
  w->s64_1 = (double*)malloc(sizeof(double) * (size_t)n);
  w->s64_2 = (double*)malloc(sizeof(double) * (size_t)n);
  w->h1 = (half_t*)malloc(sizeof(half_t) * (size_t)n);
  w->h2 = (half_t*)malloc(sizeof(half_t) * (size_t)n);
  w->cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)k * (size_t)k);
  return (w->s64_1 && w->s64_2 && w->h1 && w->h2 && w->cand) ? 0 : -1;
}

static void scratch_free(scratch_t* w) {
  free(w->s64_1); free(w->s64_2); free(w->h1); free(w->h2); free(w->cand);
}

/*
 * Product-key selection of one projected vector x (k'_t or q'_t), item 2.
 * C1, C2: this head's codebooks, [n][d_h] row-major.  Writes the n_sel
 * selected slots in rank order, their softmax weights (float64) and float32
 * scores; returns the near-tie flag bits (boundary bit = flag_shift,
 * half-1 bit = flag_shift+1, half-2 bit = flag_shift+2).
 */
static int select_side(const float* x, const float* C1, const float* C2, const odims_t* d,
                       int n_sel, scratch_t* w, int64_t* slot_out, double* wt_out,
                       float* score_out, int flag_shift) {
  const int n = d->n_sub, dh = d->d_qk / 2, k = d->k;
  int flags = 0;
  /* half scores: first half of x against C1, second half against C2 */
  for (int j = 0; j < n; ++j) {
    double a = 0.0, b = 0.0;
    for (int c = 0; c < dh; ++c) {
      a += (double)x[c] * (double)C1[(size_t)j * dh + c];
      b += (double)x[dh + c] * (double)C2[(size_t)j * dh + c];
    }
    w->s64_1[j] = a;
    w->s64_2[j] = b;
    w->h1[j].s = (float)a; w->h1[j].id = j;
    w->h2[j].s = (float)b; w->h2[j].id = j;
  }
  /* top-k of each half: full sort, keep the first k */
  qsort(w->h1, (size_t)n, sizeof(half_t), cmp_half);
  qsort(w->h2, (size_t)n, sizeof(half_t), cmp_half);
  if (k < n) {
    if (near_tie(w->s64_1[w->h1[k - 1].id], w->s64_1[w->h1[k].id])) flags |= 2 << flag_shift;
    if (near_tie(w->s64_2[w->h2[k - 1].id], w->s64_2[w->h2[k].id])) flags |= 4 << flag_shift;
  }
  /* k x k outer-sum candidates */
  int nc = 0;
  for (int a = 0; a < k; ++a) {
    for (int b = 0; b < k; ++b) {
      cand_t* c = &w->cand[nc++];
      float s = w->h1[a].s + w->h2[b].s;          /* float32 sum */
      c->s = s;
      c->slot = (int64_t)w->h1[a].id * n + w->h2[b].id;
      c->s64 = w->s64_1[w->h1[a].id] + w->s64_2[w->h2[b].id];
    }
  }
  /* top-n_sel of the candidates: full sort, keep the first n_sel */
  qsort(w->cand, (size_t)nc, sizeof(cand_t), cmp_cand);
  if (n_sel < nc && near_tie(w->cand[n_sel - 1].s64, w->cand[n_sel].s64)) flags |= 1 << flag_shift;
  /* weights: softmax over the selected float32 scores, in float64 */
  double m = (double)w->cand[0].s;
  for (int j = 1; j < n_sel; ++j)
    if ((double)w->cand[j].s > m) m = (double)w->cand[j].s;
  double z = 0.0;
  for (int j = 0; j < n_sel; ++j) z += exp((double)w->cand[j].s - m);
  for (int j = 0; j < n_sel; ++j) {
    slot_out[j] = w->cand[j].slot;
    wt_out[j] = exp((double)w->cand[j].s - m) / z;
    if (score_out) score_out[j] = w->cand[j].s;
  }
  return flags;
}

/* one head: steps [t0, t1).  All pointers are this head's blocks. */
typedef struct {
  const float *q, *k, *v, *alpha, *beta, *C1, *C2;
  float *M, *o;
  int64_t *idx_w, *idx_r;
  double *w_w, *w_r;
  uint8_t* flags;
} head_io_t;

/*
 * The selective-decay write of the Raven page ("Raven - Modelado de Secuencias
 * de Alta Recuperacion con Enrutamiento de Memoria Dispersa", section 2.2),
 * on the slots the product keys selected: the router weights are the sigmoid
 * of the W selected float32 scores normalised to sum 1 (reading: the page
 * normalises the kept sigmoid scores; dividing by their sum is the plainest
 * form), and each selected row decays toward v_t by exp(a_t r_i):
 *     M[i] = exp(a_t r_i) M[i] + (1 - exp(a_t r_i)) v_t;
 * unselected rows stay frozen.  Float64, rounded to float32.  ww receives r.
 */
static void decay_write(float* M, const int64_t* ws, const float* sw, double* ww, int W, int dv,
                        double at, const float* vt) {
  double z = 0.0;
  for (int j = 0; j < W; ++j) {
    ww[j] = 1.0 / (1.0 + exp(-(double)sw[j]));
    z += ww[j];
  }
  for (int j = 0; j < W; ++j) ww[j] /= z;
  for (int j = 0; j < W; ++j) {
    float* row = M + (size_t)ws[j] * dv;
    const double dcy = exp(at * ww[j]);
    for (int col = 0; col < dv; ++col)
      row[col] = (float)(dcy * (double)row[col] + (1.0 - dcy) * (double)vt[col]);
  }
}

static int forward_head(const head_io_t* io, const odims_t* d, int t0, int t1) {
  scratch_t w;
  if (scratch_init(&w, d) != 0) { scratch_free(&w); return -1; }
  const int dv = d->d_v, dq = d->d_qk;
  int64_t* ws = (int64_t*)malloc(sizeof(int64_t) * (size_t)(d->W + d->R));
  double* ww = (double*)malloc(sizeof(double) * (size_t)(d->W + d->R));
  double* acc = (double*)malloc(sizeof(double) * (size_t)dv);
  float* sw = (float*)malloc(sizeof(float) * (size_t)d->W);
  if (!ws || !ww || !acc || !sw) {
    free(ws); free(ww); free(acc); free(sw); scratch_free(&w); return -1;
  }
  int64_t* rs = ws + d->W;
  double* rw = ww + d->W;
  for (int t = t0; t < t1; ++t) {
    /* write selection from k'_t, read selection from q'_t (item 2) */
    int fl = select_side(io->k + (size_t)t * dq, io->C1, io->C2, d, d->W, &w, ws, ww, sw, 0);
    fl |= select_side(io->q + (size_t)t * dq, io->C1, io->C2, d, d->R, &w, rs, rw, NULL, 3);
    const double a = (double)io->alpha[t], be = io->beta ? (double)io->beta[t] : 0.0;
    const float* vt = io->v + (size_t)t * dv;
    if (d->rule == 1) decay_write(io->M, ws, sw, ww, d->W, dv, a, vt);
    /* gated delta write on the W selected slots (item 3) */
    for (int j = 0; d->rule == 0 && j < d->W; ++j) {
      float* row = io->M + (size_t)ws[j] * dv;
      const double c = be * ww[j];
      for (int col = 0; col < dv; ++col) {
        const double mt = a * (double)row[col];                 /* forget gate */
        row[col] = (float)((1.0 - c) * mt + c * (double)vt[col]);  /* delta update */
      }
    }
    /* sparse read after the write (item 4) */
    for (int col = 0; col < dv; ++col) acc[col] = 0.0;
    for (int j = 0; j < d->R; ++j) {
      const float* row = io->M + (size_t)rs[j] * dv;
      for (int col = 0; col < dv; ++col) acc[col] += rw[j] * (double)row[col];
    }
    if (io->o)
      for (int col = 0; col < dv; ++col) io->o[(size_t)t * dv + col] = (float)acc[col];
    if (io->idx_w) memcpy(io->idx_w + (size_t)t * d->W, ws, sizeof(int64_t) * (size_t)d->W);
    if (io->w_w) memcpy(io->w_w + (size_t)t * d->W, ww, sizeof(double) * (size_t)d->W);
    if (io->idx_r) memcpy(io->idx_r + (size_t)t * d->R, rs, sizeof(int64_t) * (size_t)d->R);
    if (io->w_r) memcpy(io->w_r + (size_t)t * d->R, rw, sizeof(double) * (size_t)d->R);
    if (io->flags) io->flags[t] = (uint8_t)fl;
  }
  free(ws); free(ww); free(acc); free(sw);
  scratch_free(&w);
  return 0;
}

static int dims_ok(const odims_t* d) {
  if (d->B < 1 || d->H < 1 || d->T < 0 || d->d_qk < 2 || (d->d_qk & 1) || d->d_v < 1) return 0;
  if (d->n_sub < 1 || d->k < 1 || d->k > d->n_sub) return 0;
  if (d->W < 1 || d->R < 1) return 0;
  if ((int64_t)d->W > (int64_t)d->k * d->k || (int64_t)d->R > (int64_t)d->k * d->k) return 0;
  return 1;
}

/* ---------------- threaded driver over heads ---------------- */
typedef struct {
  const float *q, *k, *v, *alpha, *beta, *C1, *C2;
  float *M, *o;
  int64_t *idx_w, *idx_r;
  double *w_w, *w_r;
  uint8_t* flags;
  odims_t d;
  int t0, t1;
  const int32_t* heads;
  int n_heads;
  int next;
  int err;
  pthread_mutex_t mu;
} job_t;

static void* worker(void* arg) {
  job_t* J = (job_t*)arg;
  const odims_t* d = &J->d;
  const int N = d->n_sub * d->n_sub, dh = d->d_qk / 2;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int i = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (i >= J->n_heads) break;
    const int bh = J->heads ? J->heads[i] : i;
    const int h = bh % d->H;
    const size_t tq = (size_t)bh * d->T;
    head_io_t io;
    io.q = J->q + tq * d->d_qk;
    io.k = J->k + tq * d->d_qk;
    io.v = J->v + tq * d->d_v;
    io.alpha = J->alpha + tq;
    io.beta = J->beta ? J->beta + tq : NULL;
    io.C1 = J->C1 + (size_t)h * d->n_sub * dh;
    io.C2 = J->C2 + (size_t)h * d->n_sub * dh;
    io.M = J->M + (size_t)bh * N * d->d_v;
    io.o = J->o ? J->o + tq * d->d_v : NULL;
    io.idx_w = J->idx_w ? J->idx_w + tq * d->W : NULL;
    io.w_w = J->w_w ? J->w_w + tq * d->W : NULL;
    io.idx_r = J->idx_r ? J->idx_r + tq * d->R : NULL;
    io.w_r = J->w_r ? J->w_r + tq * d->R : NULL;
    io.flags = J->flags ? J->flags + tq : NULL;
    if (forward_head(&io, d, J->t0, J->t1) != 0) {
      pthread_mutex_lock(&J->mu);
      J->err = 1;
      pthread_mutex_unlock(&J->mu);
    }
  }
  return NULL;
}

/*
 * Full forward pass over the heads listed in `heads` (flat b*H + h; NULL means
 * all B*H heads), steps [t_begin, t_end).  Layouts (row-major, float32):
 *   q, k [B][H][T][d_qk];  v [B][H][T][d_v];  alpha, beta [B][H][T];
 *   C1, C2 [H][n][d_qk/2];  M [B][H][N][d_v] (read as M_{t_begin}, left as
 *   M_{t_end});  o [B][H][T][d_v] (may be NULL).
 * Optional outputs (NULL to skip): idx_w [B][H][T][W] int64, w_w float64,
 *   idx_r / w_r likewise with R, flags [B][H][T].
 * dims = {B, H, T, d_qk, d_v, n_sub, k, W, R}.  Returns 0, or -1 on bad
 * dimensions / allocation failure.
 */
int sdm_oracle_forward(const float* q, const float* k, const float* v, const float* alpha,
                       const float* beta, const float* C1, const float* C2, float* M, float* o,
                       const int* dims, int t_begin, int t_end, int64_t* idx_w, double* w_w,
                       int64_t* idx_r, double* w_r, uint8_t* flags, const int32_t* heads,
                       int n_heads, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.d.B = dims[0]; J.d.H = dims[1]; J.d.T = dims[2]; J.d.d_qk = dims[3]; J.d.d_v = dims[4];
  J.d.n_sub = dims[5]; J.d.k = dims[6]; J.d.W = dims[7]; J.d.R = dims[8];
  if (!dims_ok(&J.d) || t_begin < 0 || t_end > J.d.T || t_begin > t_end) return -1;
  J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.C1 = C1; J.C2 = C2;
  J.M = M; J.o = o; J.idx_w = idx_w; J.w_w = w_w; J.idx_r = idx_r; J.w_r = w_r;
  J.flags = flags;
  J.t0 = t_begin; J.t1 = t_end;
  J.heads = heads;
  J.n_heads = heads ? n_heads : J.d.B * J.d.H;
  pthread_mutex_init(&J.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > J.n_heads) nthreads = J.n_heads > 0 ? J.n_heads : 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -1;
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, worker, &J) == 0) ++started;
  if (started == 0) worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J.mu);
  return J.err ? -1 : 0;
}

/*
 * Selection of one projected vector x (length d_qk) against one head's
 * codebooks C1, C2 ([n][d_qk/2]), keeping n_sel slots (item 2).  Writes
 * slots (rank order), float64 softmax weights and float32 scores; *flag gets
 * the near-tie bits (boundary = bit 0, half 1 = bit 1, half 2 = bit 2).
 */
int sdm_oracle_select(const float* x, const float* C1, const float* C2, const int* dims,
                      int n_sel, int64_t* slots, double* weights, float* scores, int* flag) {
  odims_t d;
  d.B = 1; d.H = 1; d.T = 1; d.d_qk = dims[3]; d.d_v = 1; d.n_sub = dims[5]; d.k = dims[6];
  d.W = n_sel; d.R = n_sel; d.rule = 0;
  if (!dims_ok(&d)) return -1;
  scratch_t w;
  if (scratch_init(&w, &d) != 0) { scratch_free(&w); return -1; }
  int f = select_side(x, C1, C2, &d, n_sel, &w, slots, weights, scores, 0);
  if (flag) *flag = f;
  scratch_free(&w);
  return 0;
}

/*
 * The forward pass with the Raven page's selective-decay write in place of the
 * gated delta write (see decay_write): same selection, read, layouts and
 * optional outputs as sdm_oracle_forward, with a [B][H][T] (a_t <= 0, the
 * decay rate) in place of alpha and no beta.  w_w receives the normalised
 * router weights r.
 */
int sdm_oracle_forward_decay(const float* q, const float* k, const float* v, const float* a,
                             const float* C1, const float* C2, float* M, float* o,
                             const int* dims, int t_begin, int t_end, int64_t* idx_w, double* w_w,
                             int64_t* idx_r, double* w_r, uint8_t* flags, const int32_t* heads,
                             int n_heads, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.d.B = dims[0]; J.d.H = dims[1]; J.d.T = dims[2]; J.d.d_qk = dims[3]; J.d.d_v = dims[4];
  J.d.n_sub = dims[5]; J.d.k = dims[6]; J.d.W = dims[7]; J.d.R = dims[8];
  J.d.rule = 1;
  if (!dims_ok(&J.d) || t_begin < 0 || t_end > J.d.T || t_begin > t_end) return -1;
  J.q = q; J.k = k; J.v = v; J.alpha = a; J.beta = NULL; J.C1 = C1; J.C2 = C2;
  J.M = M; J.o = o; J.idx_w = idx_w; J.w_w = w_w; J.idx_r = idx_r; J.w_r = w_r;
  J.flags = flags;
  J.t0 = t_begin; J.t1 = t_end;
  J.heads = heads;
  J.n_heads = heads ? n_heads : J.d.B * J.d.H;
  pthread_mutex_init(&J.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > J.n_heads) nthreads = J.n_heads > 0 ? J.n_heads : 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -1;
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, worker, &J) == 0) ++started;
  if (started == 0) worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J.mu);
  return J.err ? -1 : 0;
}
