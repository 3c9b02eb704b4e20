/*
 * pdn_oracle.c -- fp64 CPU oracle for the gated delta-rule forward recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, token-by-token
 * definition that the CUDA library is checked against. Only tests/,
 * __graft_entry__.smoke() and bench.py's CPU-baseline leg may load it. It
 * shares no code, header, table or helper with the CUDA library; the two only
 * consume the same seeded inputs.
 *
 * Sources (web explainer pages; "ja"/"de"/"fr" name the page language):
 *   [PDN]  "Preconditioned DeltaNet: Curvature-aware Sequence Modeling for
 *          Linear Recurrences" (gist.science/{ja,de,fr}/paper/2604.21100)
 *   [GDN2] "Gated DeltaNet-2" (gist.science/ja/paper/2605.22791)
 *   [FG2]  "FG2-GDN: Enhancing Long-Context Gated Delta Networks with Doubly
 *          Fine-Grained Control" (gist.science/ja/paper/2604.19021)
 *
 * State convention: S is d_v x d_k (row j = value channel, column i = key
 * channel) and the read-out is o_t = S_t q_t. The pages on GDN-2 and FG2 print
 * the transposed (d_k x d_v) state; their formulas are transposed here.
 *
 * Every variant is written as one generic token step
 *     S <- S Diag(alpha_t)                       (decay, applied first)
 *     S <- S + (u_t - S r_t) w_t^T               (delta step: read key r,
 *                                                 write key w, target u)
 *     o_t = q_scale * S q_t
 * with (r, w, u) per variant:
 *   DN/GDN/KDA      r = k,          w = beta k,          u = v
 *   PDN/PGDN/PKDA   r = k,          w = beta (B_t . k),  u = v
 *   FG2-GDN         r = sqrt(b).k,  w = sqrt(b).k,       u = sqrt(b).v
 *   GDN-2           r = e . k,      w = k,               u = g . v
 *   PLA             r = 0,          w = beta k,          u = v,  query B_t . q
 *   FG2-GDN+        r = sqrt(bk).k, w = sqrt(bk).k,      u = sqrt(bv).v
 * (". " is the elementwise product.)
 *
 * Parity status of each function is stated in its comment.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { OR_DN = 0, OR_GDN = 1, OR_KDA = 2, OR_PDN = 3, OR_PGDN = 4, OR_PKDA = 5,
       OR_FG2 = 6, OR_GDN2 = 7, OR_PLA = 8, OR_FG2P = 9 };
enum { OR_DECAY_NONE = 0, OR_DECAY_SCALAR = 1, OR_DECAY_CHANNEL = 2 };

/* ------------------------------------------------------------------------ */
/* Diagonal preconditioner coefficients B_t for one (batch, head) sequence.
 *
 * [PDN] ja §2.2 "diagonal preconditioner implementation", de §2
 * "Praktische Umsetzung", fr §2.B-C:
 *   A_t = A_{t-1} + k_t . k_t             (diagonal of the key Gram matrix,
 *                                          accumulated with no decay)
 *   P_t = Diag(A_t)^{-1}                   (raw form, replaced by B_t)
 *   stabilised: log space, centred, squashed by r/(1+|r|), then an inverse
 *   exponential that keeps B_t inside [1/x, x].
 * Readings where the pages are silent:
 *   - centring mu_t = mean over the d_k channels of log(A_{t,i} + eps);
 *   - eps is added inside the log (A_0 = 0 would give log 0);
 *   - "inverse exponential" read as B = x^(-s), decreasing in A like A^{-1};
 *   - A_t includes the current token.
 * Pinned by: x = 1 gives B = 1; equal channels give B = 1; d_k = 2 gives
 * B_0 B_1 = 1; B inside [1/x, x]; B decreasing in A (tests/test_oracle_pins.py).
 * Parity against the original paper's exact constants: unpinned (mu, eps and
 * the base are not printed on the pages). */
static void precond_step(int dk, const double *kt, double *A, double x,
                         double eps, double *Bt) {
  double mu = 0.0;
  for (int i = 0; i < dk; ++i) {
    A[i] += kt[i] * kt[i];
    Bt[i] = log(A[i] + eps); /* temporarily holds log(A + eps) */
    mu += Bt[i];
  }
  mu /= (double)dk;
  const double lnx = log(x);
  for (int i = 0; i < dk; ++i) {
    const double r = Bt[i] - mu;
    const double s = r / (1.0 + fabs(r));
    Bt[i] = exp(-s * lnx);
  }
}

int oracle_precond(int T, int dk, const double *k, const double *A0, double x,
                   double eps, double *Bcoef, double *AT) {
  if (T < 0 || dk <= 0 || !k || !Bcoef) return 1;
  double *A = (double *)calloc((size_t)dk, sizeof(double));
  if (!A) return 2;
  if (A0) memcpy(A, A0, sizeof(double) * (size_t)dk);
  for (int t = 0; t < T; ++t)
    precond_step(dk, k + (size_t)t * dk, A, x, eps, Bcoef + (size_t)t * dk);
  if (AT) memcpy(AT, A, sizeof(double) * (size_t)dk);
  free(A);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* One generic token step on a d_v x d_k state (row-major, S[j*dk + i]).
 * alpha: per key channel decay multipliers (NULL = no decay).
 * Pinned by: beta = 0 closed form (decay only); S_t r_t = u_t whenever
 * w.r = 1; brute-force product expansion for T <= 3; the recursive
 * least-squares identity with a dense preconditioned write key. */
static void token_step(int dk, int dv, double *S, const double *alpha,
                       const double *r, const double *w, const double *u,
                       const double *q, double q_scale, double *o) {
  for (int j = 0; j < dv; ++j) {
    double *Sj = S + (size_t)j * dk;
    if (alpha)
      for (int i = 0; i < dk; ++i) Sj[i] *= alpha[i];
    double y = 0.0;
    for (int i = 0; i < dk; ++i) y += Sj[i] * r[i];
    const double delta = u[j] - y;
    for (int i = 0; i < dk; ++i) Sj[i] += delta * w[i];
    if (o) {
      double z = 0.0;
      for (int i = 0; i < dk; ++i) z += Sj[i] * q[i];
      o[j] = q_scale * z;
    }
  }
}

/* ------------------------------------------------------------------------ */
typedef struct {
  int variant, decay, B, T, H, dk, dv;
  const double *q, *k, *v, *log_alpha, *beta, *erase, *write_gate, *S0, *A0;
  double q_scale, x, eps;
  double *o, *ST, *AT;
  /* generic mode */
  const double *r, *w, *u;
  int generic;
  int next_unit; /* shared work counter, protected by mu */
  pthread_mutex_t mu;
  int error;
} job_t;

static int uses_precond(int variant) {
  return variant == OR_PDN || variant == OR_PGDN || variant == OR_PKDA || variant == OR_PLA;
}

/* Forms r, w, u for one token (variant table in the file header).
 * [GDN2] ja §1 "Gated Delta Rule-2": erase gate on the key side
 *   (e_t = b_t . k_t), write gate on the value side (z_t = w_t . v_t).
 * [FG2] ja §2.1: per-channel beta vector applied as sqrt(beta) to both
 *   k and v (requires d_k = d_v).
 * [PDN] ja §2.2 "read key / write key": read key k_t, write key B_t . k_t
 *   (apply-to-key), scaled by the gain beta_t as in DeltaNet.
 * [PDN] ja §2.1 and fr §2.A: preconditioned linear attention (PLA) applies
 *   the preconditioner to the query instead (apply-to-query); linear
 *   attention writes without erasing, so its read key is 0 and its write is
 *   the gain times k_t (reading: the gain beta_t of the family's gain axis,
 *   1 for plain linear attention); the query transform is applied in
 *   run_unit.
 * [FG2] ja §2.2: FG2-GDN+ gives the key (erase strength) and the value (write
 *   strength) gain vectors of their own, beta^k in R^{d_k} and beta^v in
 *   R^{d_v}. The page prints no formula; the reading taken keeps FG2-GDN's
 *   symmetric square roots: sqrt(beta^k) on the key, sqrt(beta^v) on the
 *   value, so beta^k = beta^v is FG2-GDN (parity against the paper
 *   unpinned). beta^v arrives in the write-gate slot. */
static void form_vectors(const job_t *J, size_t tok, size_t tokh, const double *Bt,
                         double *r, double *w, double *u) {
  const int dk = J->dk, dv = J->dv;
  const double *kt = J->k + tok * dk;
  const double *vt = J->v + tok * dv;
  switch (J->variant) {
  case OR_DN: case OR_GDN: case OR_KDA: {
    const double b = J->beta[tokh];
    for (int i = 0; i < dk; ++i) { r[i] = kt[i]; w[i] = b * kt[i]; }
    for (int j = 0; j < dv; ++j) u[j] = vt[j];
  } break;
  case OR_PDN: case OR_PGDN: case OR_PKDA: {
    const double b = J->beta[tokh];
    for (int i = 0; i < dk; ++i) { r[i] = kt[i]; w[i] = b * Bt[i] * kt[i]; }
    for (int j = 0; j < dv; ++j) u[j] = vt[j];
  } break;
  case OR_FG2: {
    const double *bt = J->beta + tok * dk;
    for (int i = 0; i < dk; ++i) {
      const double sb = sqrt(bt[i]);
      r[i] = sb * kt[i];
      w[i] = sb * kt[i];
    }
    for (int j = 0; j < dv; ++j) u[j] = sqrt(bt[j]) * vt[j];
  } break;
  case OR_GDN2: {
    const double *et = J->erase + tok * dk;
    const double *gt = J->write_gate + tok * dv;
    for (int i = 0; i < dk; ++i) { r[i] = et[i] * kt[i]; w[i] = kt[i]; }
    for (int j = 0; j < dv; ++j) u[j] = gt[j] * vt[j];
  } break;
  case OR_PLA: {
    const double b = J->beta[tokh];
    for (int i = 0; i < dk; ++i) { r[i] = 0.0; w[i] = b * kt[i]; }
    for (int j = 0; j < dv; ++j) u[j] = vt[j];
  } break;
  case OR_FG2P: {
    const double *bk = J->beta + tok * dk;
    const double *bv = J->write_gate + tok * dv;
    for (int i = 0; i < dk; ++i) {
      const double sb = sqrt(bk[i]);
      r[i] = sb * kt[i];
      w[i] = sb * kt[i];
    }
    for (int j = 0; j < dv; ++j) u[j] = sqrt(bv[j]) * vt[j];
  } break;
  }
}

static int run_unit(job_t *J, int unit) {
  const int b = unit / J->H, h = unit % J->H;
  const int dk = J->dk, dv = J->dv, T = J->T, H = J->H;
  double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
  double *A = (double *)calloc((size_t)dk, sizeof(double));
  double *Bt = (double *)malloc(sizeof(double) * (size_t)dk);
  double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
  double *r = (double *)malloc(sizeof(double) * (size_t)dk);
  double *w = (double *)malloc(sizeof(double) * (size_t)dk);
  double *u = (double *)malloc(sizeof(double) * (size_t)dv);
  double *qq = (double *)malloc(sizeof(double) * (size_t)dk);
  if (!S || !A || !Bt || !alpha || !r || !w || !u || !qq) {
    free(S); free(A); free(Bt); free(alpha); free(r); free(w); free(u); free(qq);
    return 2;
  }
  const size_t sidx = ((size_t)b * H + h) * (size_t)dk * dv;
  if (J->S0) memcpy(S, J->S0 + sidx, sizeof(double) * (size_t)dk * dv);
  else memset(S, 0, sizeof(double) * (size_t)dk * dv);
  if (J->A0) memcpy(A, J->A0 + ((size_t)b * H + h) * dk, sizeof(double) * (size_t)dk);

  for (int t = 0; t < T; ++t) {
    const size_t tokh = ((size_t)b * T + t) * H + h; /* [B,T,H] index */
    const double *al = NULL;
    const int decay = J->generic ? (J->log_alpha ? OR_DECAY_CHANNEL : OR_DECAY_NONE)
                                 : J->decay;
    if (decay == OR_DECAY_SCALAR) {
      const double a = exp(J->log_alpha[tokh]);
      for (int i = 0; i < dk; ++i) alpha[i] = a;
      al = alpha;
    } else if (decay == OR_DECAY_CHANNEL) {
      const double *la = J->log_alpha + tokh * dk;
      for (int i = 0; i < dk; ++i) alpha[i] = exp(la[i]);
      al = alpha;
    }
    const double *rr, *ww, *uu, *qt = J->q + tokh * dk;
    if (J->generic) {
      rr = J->r + tokh * dk;
      ww = J->w + tokh * dk;
      uu = J->u + tokh * dv;
    } else {
      if (uses_precond(J->variant))
        precond_step(dk, J->k + tokh * dk, A, J->x, J->eps, Bt);
      form_vectors(J, tokh, tokh, Bt, r, w, u);
      rr = r; ww = w; uu = u;
      if (J->variant == OR_PLA) { /* apply-to-query: read out S_t (B_t . q_t) */
        for (int i = 0; i < dk; ++i) qq[i] = Bt[i] * qt[i];
        qt = qq;
      }
    }
    token_step(dk, dv, S, al, rr, ww, uu, qt, J->q_scale, J->o ? J->o + tokh * dv : NULL);
  }
  if (J->ST) memcpy(J->ST + sidx, S, sizeof(double) * (size_t)dk * dv);
  if (J->AT) memcpy(J->AT + ((size_t)b * H + h) * dk, A, sizeof(double) * (size_t)dk);
  free(S); free(A); free(Bt); free(alpha); free(r); free(w); free(u); free(qq);
  return 0;
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    const int unit = J->next_unit++;
    pthread_mutex_unlock(&J->mu);
    if (unit >= J->B * J->H) break;
    const int rc = run_unit(J, unit);
    if (rc) {
      pthread_mutex_lock(&J->mu);
      J->error = rc;
      pthread_mutex_unlock(&J->mu);
    }
  }
  return NULL;
}

static int run_job(job_t *J, int nthreads) {
  if (nthreads <= 0) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    nthreads = n > 0 ? (int)n : 1;
  }
  const int units = J->B * J->H;
  if (nthreads > units) nthreads = units;
  if (nthreads < 1) nthreads = 1;
  J->next_unit = 0;
  J->error = 0;
  pthread_mutex_init(&J->mu, NULL);
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return 2;
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, worker, J) == 0) ++started;
  if (started == 0) worker(J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J->mu);
  return J->error;
}

/* Variant forward: o [B,T,H,dv], ST [B,H,dv,dk], AT [B,H,dk] (any may be NULL).
 * Inputs use the [B,T,H,d] layout; log_alpha is [B,T,H] (scalar decay) or
 * [B,T,H,dk] (channel decay); beta is [B,T,H] or [B,T,H,dk] (FG2, FG2+);
 * erase [B,T,H,dk] for GDN-2, write_gate [B,T,H,dv] for GDN-2 (write gate)
 * and FG2+ (value-side gain beta^v).
 * Returns 0 on success, 1 on bad arguments, 2 on allocation failure. */
int oracle_forward(int variant, int decay, int B, int T, int H, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *log_alpha, const double *beta,
                   const double *erase, const double *write_gate,
                   const double *S0, const double *A0, double q_scale, double x,
                   double eps, double *o, double *ST, double *AT, int nthreads) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return 1;
  if (variant < OR_DN || variant > OR_FG2P) return 1;
  if (decay < OR_DECAY_NONE || decay > OR_DECAY_CHANNEL) return 1;
  if (!q || !k || !v) return 1;
  if (decay != OR_DECAY_NONE && !log_alpha) return 1;
  if (variant == OR_GDN2) {
    if (!erase || !write_gate) return 1;
  } else if (!beta) {
    return 1;
  }
  if (variant == OR_FG2P && !write_gate) return 1;
  if (variant == OR_FG2 && dk != dv) return 1;
  job_t J;
  memset(&J, 0, sizeof(J));
  J.variant = variant; J.decay = decay;
  J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
  J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta;
  J.erase = erase; J.write_gate = write_gate; J.S0 = S0; J.A0 = A0;
  J.q_scale = q_scale; J.x = x; J.eps = eps;
  J.o = o; J.ST = ST; J.AT = AT;
  J.generic = 0;
  return run_job(&J, nthreads);
}

/* Generic form: caller supplies the read key r [B,T,H,dk], write key
 * w [B,T,H,dk], target u [B,T,H,dv] and an optional channel log-decay
 * [B,T,H,dk] directly. Used by the pins that need an arbitrary (e.g. dense,
 * non-diagonal) write key, such as the least-squares equivalence
 * ([PDN] ja §2.1, Theorem 3.1). */
int oracle_generic(int B, int T, int H, int dk, int dv, const double *q,
                   const double *r, const double *w, const double *u,
                   const double *log_alpha, const double *S0, double q_scale,
                   double *o, double *ST, int nthreads) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return 1;
  if (!q || !r || !w || !u) return 1;
  job_t J;
  memset(&J, 0, sizeof(J));
  J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
  J.q = q; J.k = r; J.v = u; J.r = r; J.w = w; J.u = u;
  J.log_alpha = log_alpha; J.S0 = S0; J.q_scale = q_scale;
  J.o = o; J.ST = ST;
  J.generic = 1;
  return run_job(&J, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Backward of the token loop (gradients of a scalar loss L given dL/do_t and
 * dL/dS_T), fp64. "Gated DeltaNet-2", ja §3, single out the gate-aware
 * backward: the erase and write gates enter the gradient through the read
 * and write keys and the target. Written as the reverse-time adjoint of
 *   P = S_{t-1} D_t,  delta = u - P r,  S_t = P + delta w^T,  o_t = c S_t q'
 * (q' = q, or B_t . q for PLA):
 *   dS_t += c do_t q'^T;  dq' = c S_t^T do_t;  ddelta = dS_t w;
 *   dw = dS_t^T delta;  dr = -P^T ddelta;  du = ddelta;
 *   dP = dS_t - ddelta r^T;  dalpha_i = sum_j S_{t-1}[j,i] dP[j,i];
 *   dS_{t-1} = dP D_t,
 * then each variant's map from (k, v, beta, gates, B_t) to (r, w, u, q') and,
 * for the preconditioned variants, B_t's dependence on the accumulator
 * A_t = A_{t-1} + k_t . k_t (through log, centring, squash and x^{-s}).
 * Pinned by central finite differences of oracle_forward on every input
 * (tests/test_oracle_pins.py). Outputs may be NULL when not wanted. */
static void precond_coef_grad(int dk, const double *A, double x, double eps,
                              const double *dB, double *dA) {
  /* B_i = x^{-s_i}, s = c/(1+|c|), c_i = L_i - mean(L), L_i = log(A_i + eps) */
  double mu = 0.0;
  for (int i = 0; i < dk; ++i) mu += log(A[i] + eps);
  mu /= (double)dk;
  const double lnx = log(x);
  double mean_dc = 0.0;
  for (int i = 0; i < dk; ++i) {
    const double c = log(A[i] + eps) - mu;
    const double s = c / (1.0 + fabs(c));
    const double B = exp(-s * lnx);
    const double ds = dB[i] * (-lnx) * B;
    const double den = 1.0 + fabs(c);
    dA[i] = ds / (den * den); /* dc, temporarily */
    mean_dc += dA[i];
  }
  mean_dc /= (double)dk;
  for (int i = 0; i < dk; ++i) dA[i] = (dA[i] - mean_dc) / (A[i] + eps);
}

typedef struct {
  job_t *J;
  const double *dO, *dST;
  double *dq, *dk, *dv, *dla, *dbeta, *derase, *dwrite, *dS0, *dA0;
} bjob_t;

static int run_unit_bwd(bjob_t *BJ, int unit) {
  job_t *J = BJ->J;
  const int b = unit / J->H, h = unit % J->H;
  const int dk = J->dk, dv = J->dv, T = J->T, H = J->H;
  const size_t SS = (size_t)dk * dv;
  const int pre = uses_precond(J->variant);
  double *S = (double *)malloc(sizeof(double) * SS * (size_t)(T + 1)); /* S_0 .. S_T */
  double *Ahist = (double *)malloc(sizeof(double) * (size_t)dk * (size_t)(T + 1));
  double *Bc = (double *)malloc(sizeof(double) * (size_t)dk * (size_t)(T > 0 ? T : 1));
  double *dS = (double *)malloc(sizeof(double) * SS);
  double *dP = (double *)malloc(sizeof(double) * SS);
  double *dAcc = (double *)calloc((size_t)dk, sizeof(double)); /* sum_{s>=t} dA_s */
  double *dAt = (double *)malloc(sizeof(double) * (size_t)dk);
  double *dBt = (double *)malloc(sizeof(double) * (size_t)dk);
  double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
  double *r = (double *)malloc(sizeof(double) * (size_t)dk);
  double *w = (double *)malloc(sizeof(double) * (size_t)dk);
  double *u = (double *)malloc(sizeof(double) * (size_t)dv);
  double *qq = (double *)malloc(sizeof(double) * (size_t)dk);
  double *delta = (double *)malloc(sizeof(double) * (size_t)dv);
  double *dd = (double *)malloc(sizeof(double) * (size_t)dv);
  double *dqq = (double *)malloc(sizeof(double) * (size_t)dk);
  double *dr = (double *)malloc(sizeof(double) * (size_t)dk);
  double *dw = (double *)malloc(sizeof(double) * (size_t)dk);
  if (!S || !Ahist || !Bc || !dS || !dP || !dAcc || !dAt || !dBt || !alpha || !r || !w || !u ||
      !qq || !delta || !dd || !dqq || !dr || !dw) {
    free(S); free(Ahist); free(Bc); free(dS); free(dP); free(dAcc); free(dAt); free(dBt);
    free(alpha); free(r); free(w); free(u); free(qq); free(delta); free(dd); free(dqq);
    free(dr); free(dw);
    return 2;
  }
  const size_t sidx = ((size_t)b * H + h) * SS;
  if (J->S0) memcpy(S, J->S0 + sidx, sizeof(double) * SS);
  else memset(S, 0, sizeof(double) * SS);
  if (J->A0) memcpy(Ahist, J->A0 + ((size_t)b * H + h) * dk, sizeof(double) * (size_t)dk);
  else memset(Ahist, 0, sizeof(double) * (size_t)dk);

  /* alpha of token t (per key channel) */
#define ALPHA_OF(t_)                                                         \
  do {                                                                       \
    const size_t th_ = ((size_t)b * T + (t_)) * H + h;                       \
    for (int i = 0; i < dk; ++i)                                             \
      alpha[i] = J->decay == OR_DECAY_SCALAR ? exp(J->log_alpha[th_])        \
                 : J->decay == OR_DECAY_CHANNEL ? exp(J->log_alpha[th_ * dk + i]) \
                                                : 1.0;                       \
  } while (0)

  /* forward, keeping every state, accumulator and coefficient */
  for (int t = 0; t < T; ++t) {
    const size_t tokh = ((size_t)b * T + t) * H + h;
    double *A = Ahist + (size_t)(t + 1) * dk;
    memcpy(A, Ahist + (size_t)t * dk, sizeof(double) * (size_t)dk);
    if (pre) precond_step(dk, J->k + tokh * dk, A, J->x, J->eps, Bc + (size_t)t * dk);
    form_vectors(J, tokh, tokh, Bc + (size_t)t * dk, r, w, u);
    ALPHA_OF(t);
    memcpy(S + (size_t)(t + 1) * SS, S + (size_t)t * SS, sizeof(double) * SS);
    token_step(dk, dv, S + (size_t)(t + 1) * SS, alpha, r, w, u, J->q + tokh * dk, 1.0, NULL);
  }

  /* reverse sweep */
  if (BJ->dST) memcpy(dS, BJ->dST + sidx, sizeof(double) * SS);
  else memset(dS, 0, sizeof(double) * SS);
  const double c = J->q_scale;
  for (int t = T - 1; t >= 0; --t) {
    const size_t tokh = ((size_t)b * T + t) * H + h;
    const double *St = S + (size_t)(t + 1) * SS, *Sp = S + (size_t)t * SS;
    const double *Bt = Bc + (size_t)t * dk;
    form_vectors(J, tokh, tokh, Bt, r, w, u);
    ALPHA_OF(t);
    const double *qt = J->q + tokh * dk;
    for (int i = 0; i < dk; ++i) qq[i] = J->variant == OR_PLA ? Bt[i] * qt[i] : qt[i];
    const double *dot = BJ->dO ? BJ->dO + tokh * dv : NULL;
    /* output */
    for (int i = 0; i < dk; ++i) dqq[i] = 0.0;
    if (dot)
      for (int j = 0; j < dv; ++j)
        for (int i = 0; i < dk; ++i) {
          dS[(size_t)j * dk + i] += c * dot[j] * qq[i];
          dqq[i] += c * St[(size_t)j * dk + i] * dot[j];
        }
    /* delta = u - P r, P = S_{t-1} D */
    for (int j = 0; j < dv; ++j) {
      double y = 0.0;
      for (int i = 0; i < dk; ++i) y += Sp[(size_t)j * dk + i] * alpha[i] * r[i];
      delta[j] = u[j] - y;
      double s = 0.0;
      for (int i = 0; i < dk; ++i) s += dS[(size_t)j * dk + i] * w[i];
      dd[j] = s;
    }
    for (int i = 0; i < dk; ++i) {
      double sw = 0.0, sr = 0.0, sa = 0.0;
      for (int j = 0; j < dv; ++j) {
        const double P = Sp[(size_t)j * dk + i] * alpha[i];
        const double g = dS[(size_t)j * dk + i] - dd[j] * r[i];
        dP[(size_t)j * dk + i] = g;
        sw += dS[(size_t)j * dk + i] * delta[j];
        sr += P * dd[j];
        sa += Sp[(size_t)j * dk + i] * g;
      }
      dw[i] = sw;
      dr[i] = -sr;
      /* dL/dalpha_i = sa; dlog_alpha = alpha * sa */
      if (BJ->dla) {
        if (J->decay == OR_DECAY_CHANNEL) BJ->dla[tokh * dk + i] = alpha[i] * sa;
        else if (J->decay == OR_DECAY_SCALAR) {
          if (i == 0) BJ->dla[tokh] = 0.0;
          BJ->dla[tokh] += alpha[i] * sa;
        }
      }
    }
    for (int j = 0; j < dv; ++j)
      for (int i = 0; i < dk; ++i) dS[(size_t)j * dk + i] = dP[(size_t)j * dk + i] * alpha[i];

    /* variant maps: (r, w, u, q') -> inputs */
    const double *kt = J->k + tokh * dk, *vt = J->v + tokh * dv;
    double *gq = BJ->dq ? BJ->dq + tokh * dk : NULL;
    double *gk = BJ->dk ? BJ->dk + tokh * dk : NULL;
    double *gv = BJ->dv ? BJ->dv + tokh * dv : NULL;
    for (int i = 0; i < dk; ++i) dBt[i] = 0.0;
    switch (J->variant) {
    case OR_DN: case OR_GDN: case OR_KDA: {
      const double be = J->beta[tokh];
      double db = 0.0;
      for (int i = 0; i < dk; ++i) {
        if (gk) gk[i] = dr[i] + be * dw[i];
        db += kt[i] * dw[i];
      }
      if (BJ->dbeta) BJ->dbeta[tokh] = db;
      if (gv) for (int j = 0; j < dv; ++j) gv[j] = dd[j];
      if (gq) for (int i = 0; i < dk; ++i) gq[i] = dqq[i];
    } break;
    case OR_PDN: case OR_PGDN: case OR_PKDA: {
      const double be = J->beta[tokh];
      double db = 0.0;
      for (int i = 0; i < dk; ++i) {
        if (gk) gk[i] = dr[i] + be * Bt[i] * dw[i];
        db += Bt[i] * kt[i] * dw[i];
        dBt[i] = be * kt[i] * dw[i];
      }
      if (BJ->dbeta) BJ->dbeta[tokh] = db;
      if (gv) for (int j = 0; j < dv; ++j) gv[j] = dd[j];
      if (gq) for (int i = 0; i < dk; ++i) gq[i] = dqq[i];
    } break;
    case OR_PLA: {
      const double be = J->beta[tokh];
      double db = 0.0;
      for (int i = 0; i < dk; ++i) {
        if (gk) gk[i] = be * dw[i];
        db += kt[i] * dw[i];
        dBt[i] = qt[i] * dqq[i];
        if (gq) gq[i] = Bt[i] * dqq[i];
      }
      if (BJ->dbeta) BJ->dbeta[tokh] = db;
      if (gv) for (int j = 0; j < dv; ++j) gv[j] = dd[j];
    } break;
    case OR_FG2: case OR_FG2P: {
      const double *bk = J->beta + tokh * dk;
      const double *bv = J->variant == OR_FG2 ? J->beta + tokh * dv : J->write_gate + tokh * dv;
      for (int i = 0; i < dk; ++i) {
        const double sb = sqrt(bk[i]);
        if (gk) gk[i] = sb * (dr[i] + dw[i]);
        if (BJ->dbeta) BJ->dbeta[tokh * dk + i] = kt[i] * (dr[i] + dw[i]) / (2.0 * sb);
        if (gq) gq[i] = dqq[i];
      }
      for (int j = 0; j < dv; ++j) {
        const double sv = sqrt(bv[j]);
        if (gv) gv[j] = sv * dd[j];
        const double g = vt[j] * dd[j] / (2.0 * sv);
        if (J->variant == OR_FG2) {
          if (BJ->dbeta) BJ->dbeta[tokh * dk + j] += g;
        } else if (BJ->dwrite) {
          BJ->dwrite[tokh * dv + j] = g;
        }
      }
    } break;
    case OR_GDN2: {
      const double *et = J->erase + tokh * dk, *gt = J->write_gate + tokh * dv;
      for (int i = 0; i < dk; ++i) {
        if (gk) gk[i] = et[i] * dr[i] + dw[i];
        if (BJ->derase) BJ->derase[tokh * dk + i] = kt[i] * dr[i];
        if (gq) gq[i] = dqq[i];
      }
      for (int j = 0; j < dv; ++j) {
        if (gv) gv[j] = gt[j] * dd[j];
        if (BJ->dwrite) BJ->dwrite[tokh * dv + j] = vt[j] * dd[j];
      }
    } break;
    }
    /* preconditioner: B_t depends on A_t = A_{t-1} + k_t . k_t, and A_t feeds
     * every later token: dA_t (total) = dA_t (own coefficient) + dA_{t+1} */
    if (pre) {
      precond_coef_grad(dk, Ahist + (size_t)(t + 1) * dk, J->x, J->eps, dBt, dAt);
      for (int i = 0; i < dk; ++i) {
        dAcc[i] += dAt[i];
        if (gk) gk[i] += 2.0 * kt[i] * dAcc[i];
      }
    }
  }
#undef ALPHA_OF
  if (BJ->dS0) memcpy(BJ->dS0 + sidx, dS, sizeof(double) * SS);
  if (BJ->dA0 && pre) memcpy(BJ->dA0 + ((size_t)b * H + h) * dk, dAcc, sizeof(double) * (size_t)dk);
  free(S); free(Ahist); free(Bc); free(dS); free(dP); free(dAcc); free(dAt); free(dBt);
  free(alpha); free(r); free(w); free(u); free(qq); free(delta); free(dd); free(dqq);
  free(dr); free(dw);
  return 0;
}

int oracle_backward(int variant, int decay, int B, int T, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *log_alpha, const double *beta, const double *erase,
                    const double *write_gate, const double *S0, const double *A0,
                    double q_scale, double x, double eps, const double *dO, const double *dST,
                    double *dq, double *dkk, double *dvv, double *dla, double *dbeta,
                    double *derase, double *dwrite, double *dS0, double *dA0) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return 1;
  if (variant < OR_DN || variant > OR_FG2P) return 1;
  if (!q || !k || !v) return 1;
  if (decay != OR_DECAY_NONE && !log_alpha) return 1;
  if (variant == OR_GDN2 ? (!erase || !write_gate) : !beta) return 1;
  if (variant == OR_FG2P && !write_gate) return 1;
  if (variant == OR_FG2 && dk != dv) return 1;
  job_t J;
  memset(&J, 0, sizeof(J));
  J.variant = variant; J.decay = decay;
  J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
  J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta;
  J.erase = erase; J.write_gate = write_gate; J.S0 = S0; J.A0 = A0;
  J.q_scale = q_scale; J.x = x; J.eps = eps;
  bjob_t BJ = {&J, dO, dST, dq, dkk, dvv, dla, dbeta, derase, dwrite, dS0, dA0};
  int err = 0;
  for (int unit = 0; unit < B * H; ++unit) {
    const int rc = run_unit_bwd(&BJ, unit);
    if (rc) err = rc;
  }
  return err;
}
