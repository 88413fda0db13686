/*
 * kda_ref.c -- float64 CPU oracle for the Kimi Delta Attention (KDA) operator.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness oracle that the
 * GPU path is checked against.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the library's product path never
 * does.  It shares no code, header or constant table with the CUDA sources.
 *
 * What it computes (plain definition, one token at a time, in float64):
 *
 *   Kimi Linear summary (greeksharifa.github.io), "3 Kimi Delta Attention":
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t ; the memory is decayed first, then delta-corrected.
 *   Kimi K3 architecture summary (molayo1419.me), lower-bounded gate:
 *     g_t = g_min * Sigmoid(e^{A_h} z_t), g_min = -5, alpha_t = exp(g_t).
 *   Kimi Linear summary, "4 The Kimi Linear Model Architecture":
 *     queries and keys are normalised to unit length.
 *
 * Readings where the pages are silent (stated once, used everywhere):
 *   - no 1/sqrt(d) query scale (the recurrence shows none);
 *   - L2 normalisation x / sqrt(sum x^2 + 1e-6), done here for q and k;
 *   - e^{A_h} is one scalar per head, sigma is the logistic function, no bias;
 *   - o_t reads the state after token t's update.
 *
 * The product (I - b k k^T) S' is evaluated as S' - b k (k^T S') (associativity
 * only), which keeps the oracle O(dk*dv) per token.
 *
 * Layouts (row-major, token-major, matching the C ABI of the operator):
 *   q, k, z : [T, H, dk]   v, o : [T, H, dv]   beta : [T, H]   A : [H]
 *   g       : [T, H, dk]   (log-decay input of the g-entry)
 *   S0, S_final : [N, H, dk, dv]  state S[key][value]
 *   S_trace : [T, H, dk, dv] (optional) state after every token
 *   cu_seqlens : [N+1] int64, cu[0] = 0, non-decreasing, cu[N] = T.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KDA_REF_GMIN (-5.0)
#define KDA_REF_NORM_EPS (1e-6)

/* Lower-bounded channel-wise gate, one value:
 * g = g_min * sigmoid(e^{A} z) = g_min / (1 + exp(-e^{A} z)). */
static double gate_value(double z, double A) {
  return KDA_REF_GMIN / (1.0 + exp(-exp(A) * z));
}

void kda_ref_gate(const double* z, const double* A, int64_t T, int64_t H,
                  int64_t dk, double* g) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t h = 0; h < H; ++h)
      for (int64_t j = 0; j < dk; ++j) {
        int64_t idx = (t * H + h) * dk + j;
        g[idx] = gate_value(z[idx], A[h]);
      }
}

/* Unit-length normalisation x / sqrt(|x|^2 + eps). */
static void l2_normalise(const double* x, int64_t n, double* out) {
  double ss = 0.0;
  for (int64_t j = 0; j < n; ++j) ss += x[j] * x[j];
  double inv = 1.0 / sqrt(ss + KDA_REF_NORM_EPS);
  for (int64_t j = 0; j < n; ++j) out[j] = x[j] * inv;
}

typedef struct {
  const double *q, *k, *v, *z, *A, *g, *beta, *S0;
  const int64_t* cu;
  int64_t N, T, H, dk, dv;
  double *o, *S_final, *S_trace;
  int64_t next; /* shared work counter over (sequence, head) pairs */
} kda_ref_job;

/* One (sequence n, head h) recurrence. */
static void run_pair(const kda_ref_job* J, int64_t n, int64_t h, double* S,
                     double* scratch) {
  const int64_t dk = J->dk, dv = J->dv, H = J->H;
  double* khat = scratch;
  double* qhat = khat + dk;
  double* alpha = qhat + dk;
  double* p = alpha + dk; /* k^T S' , length dv */

  const int64_t sidx = (n * H + h) * dk * dv;
  if (J->S0)
    memcpy(S, J->S0 + sidx, sizeof(double) * dk * dv);
  else
    memset(S, 0, sizeof(double) * dk * dv);

  for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
    const int64_t xk = (t * H + h) * dk, xv = (t * H + h) * dv;
    l2_normalise(J->k + xk, dk, khat);
    l2_normalise(J->q + xk, dk, qhat);
    for (int64_t i = 0; i < dk; ++i) {
      double gi = J->g ? J->g[xk + i] : gate_value(J->z[xk + i], J->A[h]);
      alpha[i] = exp(gi);
    }
    const double b = J->beta[t * H + h];
    const double* vt = J->v + xv;

    /* decay first: S' = Diag(alpha) S */
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= alpha[i];

    /* delta correction: S = (I - b k k^T) S' + b k v^T
     *                     = S' - b k (k^T S') + b k v^T                     */
    for (int64_t j = 0; j < dv; ++j) p[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j) p[j] += khat[i] * S[i * dv + j];
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j)
        S[i * dv + j] += -b * khat[i] * p[j] + b * khat[i] * vt[j];

    /* output from the updated state: o_t = S_t^T q_t */
    double* ot = J->o + xv;
    for (int64_t j = 0; j < dv; ++j) ot[j] = 0.0;
    for (int64_t i = 0; i < dk; ++i)
      for (int64_t j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qhat[i];

    if (J->S_trace)
      memcpy(J->S_trace + (t * H + h) * dk * dv, S, sizeof(double) * dk * dv);
  }
  if (J->S_final) memcpy(J->S_final + sidx, S, sizeof(double) * dk * dv);
}

static void* worker(void* arg) {
  kda_ref_job* J = (kda_ref_job*)arg;
  double* S = (double*)malloc(sizeof(double) * J->dk * J->dv);
  double* scratch = (double*)malloc(sizeof(double) * (3 * J->dk + J->dv));
  const int64_t pairs = J->N * J->H;
  for (;;) {
    int64_t w = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
    if (w >= pairs) break;
    run_pair(J, w / J->H, w % J->H, S, scratch);
  }
  free(S);
  free(scratch);
  return NULL;
}

static int run(kda_ref_job* J, int threads) {
  if (J->N < 0 || J->T < 0 || J->H <= 0 || J->dk <= 0 || J->dv <= 0) return -1;
  if (!J->q || !J->k || !J->v || !J->beta || !J->o) return -1;
  if (!J->g && (!J->z || !J->A)) return -1;
  if (J->cu[0] != 0 || J->cu[J->N] != J->T) return -1;
  for (int64_t n = 0; n < J->N; ++n)
    if (J->cu[n + 1] < J->cu[n]) return -1;
  J->next = 0;
  if (threads < 1) threads = 1;
  if (threads == 1) {
    worker(J);
    return 0;
  }
  pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * threads);
  int started = 0;
  for (int i = 0; i < threads; ++i)
    if (pthread_create(&tid[i], NULL, worker, J) == 0) ++started;
  if (started == 0) worker(J);
  for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
  free(tid);
  return 0;
}

/* Forward over packed sequences with the gate computed from (z, A). */
int kda_ref_forward(const double* q, const double* k, const double* v,
                    const double* z, const double* A, const double* beta,
                    const double* S0, const int64_t* cu_seqlens, int64_t N,
                    int64_t T, int64_t H, int64_t dk, int64_t dv, double* o,
                    double* S_final, double* S_trace, int threads) {
  kda_ref_job J = {q, k, v, z, A, NULL, beta, S0, cu_seqlens, N, T, H, dk, dv,
                   o, S_final, S_trace, 0};
  return run(&J, threads);
}

/* Same recurrence, but the log-decay g [T,H,dk] is given directly. */
int kda_ref_forward_g(const double* q, const double* k, const double* v,
                      const double* g, const double* beta, const double* S0,
                      const int64_t* cu_seqlens, int64_t N, int64_t T,
                      int64_t H, int64_t dk, int64_t dv, double* o,
                      double* S_final, double* S_trace, int threads) {
  kda_ref_job J = {q, k, v, NULL, NULL, g, beta, S0, cu_seqlens, N, T, H, dk, dv,
                   o, S_final, S_trace, 0};
  return run(&J, threads);
}
