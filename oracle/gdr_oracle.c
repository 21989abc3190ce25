/*
 * oracle/gdr_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * The plain, slow, fp64 CPU definition of the gated delta rule, token by token.
 * Only tests/, the package's smoke check and bench.py's CPU-baseline leg may
 * load this file's library.  It shares no code, header or constant with the
 * CUDA path.
 *
 * What it computes (per sequence n and head h, tokens t in sequence order):
 *
 *   S~_t = D_t S_{t-1}                       D_t = diag(alpha_t) or alpha_t I or I
 *   r_t  = S~_t^T k_t                        the memory's current read of k_t
 *   u_t  = beta_t (v_t - r_t)                the delta-rule residual
 *   S_t  = S~_t + k_t u_t^T                  = (I - beta_t k_t k_t^T) D_t S_{t-1}
 *                                                + beta_t k_t v_t^T
 *   o_t  = S_t^T q_t                         read after the write of token t
 *
 * Sources:
 *  - "DeltaTTT: Layerwise Optimization for Nonlinear Recurrent Memory",
 *    §2 Background: with a linear memory and one-token updates, serial gradient
 *    descent gives DeltaNet's delta-rule update; §4.1: a gradient step on a
 *    linear-regression objective in the memory matrix is a delta-rule update.
 *    The gradient of 1/2 ||S^T k - v||^2 in S is k (S^T k - v)^T, so one step
 *    with learning rate beta is S - beta k (S^T k - v)^T, i.e. the two lines
 *    r_t / u_t / S_t above.
 *  - "Delta-Rule Linear Attention" topic page, FG^2-GDN card, and the
 *    Gated DeltaNet-2 abstract on the comparative-study page (2607.07953):
 *    GDN's decay is one scalar per head and token; KDA refines it into a
 *    channel-wise decay (one factor per key channel, i.e. a diagonal D_t).
 *  - The state is dk x dv; decay is applied to the state before the erase
 *    (reading: the product (I - b k k^T) diag(a) S is the only order of the
 *    two factors that type-checks for a dk x dv state with dk != dv once the
 *    printed row-vector form is transposed; for scalar decay the order does
 *    not matter).
 *
 * Variant "fixed base" (flag fixed_base = 1): the state-dependent erase term is
 * dropped, S_t = D_t S_{t-1} + beta_t k_t v_t^T.  With alpha = 1 and S_0 = 0 this
 * is additive causal linear attention (DeltaTTT page, §2 Background: evaluating
 * the gradient at the shared initial memory gives additive linear attention).
 *
 * Parity status: pinned by identities, special cases, brute force and an
 * independent chunkwise solve in tests/test_oracle.py; the pages print no
 * worked numeric example of the recurrence.
 *
 * Layouts (all row-major, fp64):
 *   q, k        [ntok][H][dk]        ntok = total tokens (B*T, or packed total)
 *   v, out      [ntok][H][dv]
 *   beta        [ntok][H]
 *   log_alpha   gate 0: unused (may be NULL); gate 1: [ntok][H];
 *               gate 2: [ntok][H][dk]
 *   s0, sT      [nseq][H][dk][dv]   s0 may be NULL (zero state), sT may be NULL
 *   cu          [nseq+1] int64 token offsets, cu[0] = 0, non-decreasing
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
  const double *q, *k, *v, *beta, *log_alpha, *s0;
  double *out, *sT;
  const int64_t *cu;
  int nseq, H, dk, dv, gate, fixed_base;
  /* work distribution: a shared counter over (n, h) pairs */
  pthread_mutex_t lock;
  int next;
} job_t;

static void one_chain(const job_t *J, int n, int h, double *S, double *r,
                      double *a) {
  const int H = J->H, dk = J->dk, dv = J->dv;
  if (J->s0)
    memcpy(S, J->s0 + ((size_t)n * H + h) * dk * dv, sizeof(double) * dk * dv);
  else
    memset(S, 0, sizeof(double) * dk * dv);

  for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
    const double *kt = J->k + ((size_t)t * H + h) * dk;
    const double *qt = J->q + ((size_t)t * H + h) * dk;
    const double *vt = J->v + ((size_t)t * H + h) * dv;
    const double bt = J->beta[(size_t)t * H + h];

    /* decay: a[c] = alpha_t for channel c */
    for (int c = 0; c < dk; ++c) {
      if (J->gate == 0)
        a[c] = 1.0;
      else if (J->gate == 1)
        a[c] = exp(J->log_alpha[(size_t)t * H + h]);
      else
        a[c] = exp(J->log_alpha[((size_t)t * H + h) * dk + c]);
    }
    for (int c = 0; c < dk; ++c)
      for (int j = 0; j < dv; ++j) S[c * dv + j] *= a[c];

    /* read r = S~^T k, residual u = beta (v - r) (or beta v, fixed base) */
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int c = 0; c < dk; ++c) acc += S[c * dv + j] * kt[c];
      r[j] = J->fixed_base ? bt * vt[j] : bt * (vt[j] - acc);
    }
    /* write S += k u^T */
    for (int c = 0; c < dk; ++c)
      for (int j = 0; j < dv; ++j) S[c * dv + j] += kt[c] * r[j];

    /* output o = S^T q */
    double *ot = J->out + ((size_t)t * H + h) * dv;
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int c = 0; c < dk; ++c) acc += S[c * dv + j] * qt[c];
      ot[j] = acc;
    }
  }
  if (J->sT)
    memcpy(J->sT + ((size_t)n * H + h) * dk * dv, S, sizeof(double) * dk * dv);
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  double *S = (double *)malloc(sizeof(double) * J->dk * J->dv);
  double *r = (double *)malloc(sizeof(double) * J->dv);
  double *a = (double *)malloc(sizeof(double) * J->dk);
  for (;;) {
    pthread_mutex_lock(&J->lock);
    int idx = J->next++;
    pthread_mutex_unlock(&J->lock);
    if (idx >= J->nseq * J->H) break;
    one_chain(J, idx / J->H, idx % J->H, S, r, a);
  }
  free(S);
  free(r);
  free(a);
  return NULL;
}

/* Returns the number of threads used, or a negative value on bad arguments. */
int oracle_gdr_fwd(const double *q, const double *k, const double *v,
                   const double *log_alpha, const double *beta,
                   const double *s0, double *out, double *sT,
                   const int64_t *cu, int nseq, int H, int dk, int dv,
                   int gate, int fixed_base, int nthreads) {
  if (!q || !k || !v || !beta || !out || !cu) return -1;
  if (nseq < 0 || H <= 0 || dk <= 0 || dv <= 0) return -2;
  if (gate < 0 || gate > 2 || (gate != 0 && !log_alpha)) return -3;
  for (int n = 0; n < nseq; ++n)
    if (cu[n + 1] < cu[n]) return -4;
  if (cu[0] != 0) return -4;

  job_t J;
  J.q = q; J.k = k; J.v = v; J.beta = beta; J.log_alpha = log_alpha;
  J.s0 = s0; J.out = out; J.sT = sT; J.cu = cu;
  J.nseq = nseq; J.H = H; J.dk = dk; J.dv = dv; J.gate = gate;
  J.fixed_base = fixed_base;
  J.next = 0;
  pthread_mutex_init(&J.lock, NULL);

  int nt = nthreads;
  if (nt <= 0) nt = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nt < 1) nt = 1;
  if (nt > nseq * H) nt = nseq * H > 0 ? nseq * H : 1;

  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nt);
  for (int i = 1; i < nt; ++i) pthread_create(&th[i], NULL, worker, &J);
  worker(&J);
  for (int i = 1; i < nt; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J.lock);
  return nt;
}
