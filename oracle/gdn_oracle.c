/*
 * gdn_oracle.c -- CPU oracle of the dense Gated DeltaNet (GDN) recurrence, the
 * baseline the SDM pages compare against.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite and the benchmark's CPU
 * baseline leg load this library.  It shares no code, header, table or helper
 * with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes.  The SDM summaries (gist.science 2607.07386, "Mecanismo
 * Central" item 3) apply "the Gated DeltaNet update rule" to each selected
 * slot; GDN itself applies it to a dense state.  The delta-mem page
 * (gist.science 2605.12357, section 2.A, OSAM update rule) writes the dense
 * delta rule as S_t = lambda_t S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T.
 * Reading, stated here: the GDN baseline is that rule with the SDM pages' gate
 * order -- the forget gate first, then the delta correction on the gated
 * state, exactly as item 3 writes it per slot:
 *     S~ = alpha_t S_{t-1};   S_t = S~ + beta_t (v_t - S~ k_t) k_t^T,
 * with S in R^{d_v x d_k} per (b,h) head, and the read after the write, as
 * for SDM: o_t = S_t q_t.  (Expanded, S_t = alpha_t S_{t-1} (I - beta_t k_t
 * k_t^T) + beta_t v_t k_t^T.)  Evaluated row by row in float64 with the
 * state kept in float64 through the whole sequence; o and the final S are
 * rounded to float32.  alpha_t, beta_t are per (b,h,t) scalars.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  const float *q, *k, *v, *alpha, *beta;
  float *S, *o;
  int B, H, T, dk, dv;
  int t0, t1;
  int next, err;
  pthread_mutex_t mu;
} gdn_job_t;

/* one head over steps [t0, t1): S (float32 in/out) is carried in float64 */
static int gdn_head(const gdn_job_t* J, int bh) {
  const int dk = J->dk, dv = J->dv;
  const size_t tq = (size_t)bh * J->T;
  double* S = (double*)malloc(sizeof(double) * (size_t)dv * dk);
  if (!S) return -1;
  float* Sf = J->S + (size_t)bh * dv * dk;
  for (size_t i = 0; i < (size_t)dv * dk; ++i) S[i] = (double)Sf[i];
  for (int t = J->t0; t < J->t1; ++t) {
    const float* kt = J->k + (tq + t) * dk;
    const float* qt = J->q + (tq + t) * dk;
    const float* vt = J->v + (tq + t) * dv;
    const double a = (double)J->alpha[tq + t], b = (double)J->beta[tq + t];
    for (int i = 0; i < dv; ++i) {
      double* s = S + (size_t)i * dk;
      /* forget gate, then the prediction of the gated row */
      double pred = 0.0;
      for (int j = 0; j < dk; ++j) {
        s[j] = a * s[j];
        pred += s[j] * (double)kt[j];
      }
      /* delta correction along k_t */
      const double e = b * ((double)vt[i] - pred);
      for (int j = 0; j < dk; ++j) s[j] += e * (double)kt[j];
      /* read after the write */
      double o = 0.0;
      for (int j = 0; j < dk; ++j) o += s[j] * (double)qt[j];
      if (J->o) J->o[(tq + t) * dv + i] = (float)o;
    }
  }
  for (size_t i = 0; i < (size_t)dv * dk; ++i) Sf[i] = (float)S[i];
  free(S);
  return 0;
}

static void* gdn_worker(void* arg) {
  gdn_job_t* J = (gdn_job_t*)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    const int bh = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (bh >= J->B * J->H) break;
    if (gdn_head(J, bh) != 0) {
      pthread_mutex_lock(&J->mu);
      J->err = 1;
      pthread_mutex_unlock(&J->mu);
    }
  }
  return NULL;
}

/*
 * Dense GDN forward over steps [t_begin, t_end).  Layouts (row-major, float32):
 *   q, k [B][H][T][d_k];  v [B][H][T][d_v];  alpha, beta [B][H][T];
 *   S [B][H][d_v][d_k] (read as S_{t_begin}, left as S_{t_end});
 *   o [B][H][T][d_v] (may be NULL).
 * dims = {B, H, T, d_k, d_v}.  Returns 0, or -1 on bad dimensions / memory.
 */
int gdn_oracle_forward(const float* q, const float* k, const float* v, const float* alpha,
                       const float* beta, float* S, float* o, const int* dims, int t_begin,
                       int t_end, int nthreads) {
  gdn_job_t J;
  memset(&J, 0, sizeof(J));
  J.B = dims[0]; J.H = dims[1]; J.T = dims[2]; J.dk = dims[3]; J.dv = dims[4];
  if (J.B < 1 || J.H < 1 || J.T < 0 || J.dk < 1 || J.dv < 1) return -1;
  if (t_begin < 0 || t_end > J.T || t_begin > t_end) return -1;
  J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.S = S; J.o = o;
  J.t0 = t_begin; J.t1 = t_end;
  pthread_mutex_init(&J.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > J.B * J.H) nthreads = J.B * J.H;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -1;
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, gdn_worker, &J) == 0) ++started;
  if (started == 0) gdn_worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J.mu);
  return J.err ? -1 : 0;
}
