/*
 * ttt_oracle.c - fp64 CPU oracle of the Test-Time-Training (TTT) layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path (the
 * CUDA library and its Python binding) never calls it, shares no code with it
 * and fails loudly when its own CUDA extension is missing.
 *
 * Source of the method: the TTT write-up "大模型最强架构TTT问世！斯坦福UCSD等5年
 * 磨一剑，一夜推翻Transformer" (itmax.cn / aharts.cn, a summary of arXiv
 * 2407.04620).  Its equations were images and did not survive; what follows is
 * stated from the prose, with every reading called out:
 *
 *  - §03.1 "TTT hidden state": the hidden state is the weight W of a model f.
 *    The update rule is one gradient step W_t = W_{t-1} - eta_t * grad l, and
 *    the output rule evaluates f at the UPDATED weight: z_t = f(x_t; W_t).
 *  - §03.5 "self-supervised task": multi-view reconstruction,
 *    l(W; x_t) = || f(theta_K x_t; W) - theta_V x_t ||^2, output f(theta_Q x_t; W).
 *    The projections are outside this layer: it receives K, V, Q already
 *    projected.  Reading: ||.||^2 has no 1/2 and no 1/d, so gradients carry 2.
 *  - §03.6 "mini-batch TTT": G_t = grad l(W_{t'}; x_t) with t' = t - mod(t, b),
 *    i.e. every gradient of a mini-batch is taken at the state left by the
 *    previous mini-batch.  Reading: tokens are 0-indexed, so mini-batch n holds
 *    tokens n*b .. n*b+b-1 and its base is the state after token n*b-1.
 *  - §03.9 "two variants": TTT-Linear f(x) = x W with W square; TTT-MLP has two
 *    layers, hidden width 4x the input, GELU; for stability f carries a layer
 *    norm and a residual: f(x) = x + LN(f_res(x)).  Readings: LN uses the
 *    population (biased) variance and an explicit epsilon; gamma and beta are
 *    fixed layer parameters that the inner loop does not update; GELU is the
 *    exact x * Phi(x); f has no bias.
 *
 * This file implements the PRIMAL form: token by token, every per-token
 * gradient is materialised as a full parameter-sized array and applied with
 * its own step size.  It deliberately does not use the dual form (§03.7), so
 * that agreement between the two is evidence about both.
 *
 * Layouts (row-major, contiguous, float64):
 *   Q, K, V, Z : [B][H][T][d]      eta : [B][H][T]
 *   W0         : [H][P]            W_out : [B][H][P]
 *   gamma, beta: [H][d]
 * with P = d*d for the linear kinds (W[i][j], f(x)_j = sum_i x_i W[i][j]) and
 * P = d*h + h*d for the MLP (W1 [d][h] followed by W2 [h][d]).
 */
#define _DEFAULT_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORACLE_LINEAR = 0, ORACLE_LINEAR_LN = 1, ORACLE_MLP_LN = 2 };

typedef struct {
  int kind;
  int d;
  int h;               /* MLP hidden width; unused for the linear kinds */
  const double *gamma; /* [d], LN scale of this head (LN kinds only) */
  const double *beta;  /* [d], LN shift of this head */
  double eps;
} model_t;

static long param_count(const model_t *m) {
  return m->kind == ORACLE_MLP_LN ? 2L * m->d * m->h : (long)m->d * m->d;
}

/* --- elementary functions ------------------------------------------------ */

/* GELU, exact form x * Phi(x) with Phi the standard normal CDF. */
static double gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }

/* d/dx [x * Phi(x)] = Phi(x) + x * phi(x), phi the standard normal density. */
static double gelu_deriv(double x) {
  const double Phi = 0.5 * (1.0 + erf(x / sqrt(2.0)));
  const double phi = exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
  return Phi + x * phi;
}

/* Layer norm of one row y[d]: xhat = (y - mean) / sqrt(var + eps), with the
 * population variance.  Returns 1/sqrt(var + eps) and fills xhat. */
static double ln_normalise(const double *y, int d, double eps, double *xhat) {
  double mean = 0.0;
  for (int j = 0; j < d; ++j) mean += y[j];
  mean /= d;
  double var = 0.0;
  for (int j = 0; j < d; ++j) var += (y[j] - mean) * (y[j] - mean);
  var /= d;
  const double rstd = 1.0 / sqrt(var + eps);
  for (int j = 0; j < d; ++j) xhat[j] = (y[j] - mean) * rstd;
  return rstd;
}

/* Back-propagate through xhat = LN-normalise(y) with the explicit Jacobian
 * d xhat_i / d y_j = rstd * (delta_ij - 1/d - xhat_i xhat_j / d):
 * dy_j = sum_i dxhat_i * d xhat_i / d y_j. */
static void ln_normalise_backward(const double *xhat, double rstd, int d,
                                  const double *dxhat, double *dy) {
  for (int j = 0; j < d; ++j) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) {
      const double jac = rstd * ((i == j ? 1.0 : 0.0) - 1.0 / d - xhat[i] * xhat[j] / d);
      acc += dxhat[i] * jac;
    }
    dy[j] = acc;
  }
}

/* --- the inner model f ----------------------------------------------------- */

/* Scratch big enough for any one evaluation: 6 rows of max(d, h). */
typedef struct {
  double *a, *s, *y, *xhat, *g1, *g2;
} scratch_t;

static int scratch_init(scratch_t *sc, const model_t *m) {
  const int n = m->h > m->d ? m->h : m->d;
  double *buf = (double *)calloc(6 * (size_t)n, sizeof(double));
  if (!buf) return -1;
  sc->a = buf;
  sc->s = buf + n;
  sc->y = buf + 2 * n;
  sc->xhat = buf + 3 * n;
  sc->g1 = buf + 4 * n;
  sc->g2 = buf + 5 * n;
  return 0;
}

static void scratch_free(scratch_t *sc) { free(sc->a); }

/* out[d] = f(x; W).  Linear: x W.  Linear+LN: x + LN(x W).
 * MLP: x + LN(GELU(x W1) W2). */
static void model_apply(const model_t *m, const double *W, const double *x, double *out,
                        scratch_t *sc) {
  const int d = m->d, h = m->h;
  double *y = sc->y;
  if (m->kind == ORACLE_MLP_LN) {
    const double *W1 = W, *W2 = W + (long)d * h;
    for (int i = 0; i < h; ++i) {
      double acc = 0.0;
      for (int p = 0; p < d; ++p) acc += x[p] * W1[(long)p * h + i];
      sc->s[i] = gelu(acc);
    }
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int i = 0; i < h; ++i) acc += sc->s[i] * W2[(long)i * d + j];
      y[j] = acc;
    }
  } else {
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += x[i] * W[(long)i * d + j];
      y[j] = acc;
    }
  }
  if (m->kind == ORACLE_LINEAR) {
    for (int j = 0; j < d; ++j) out[j] = y[j];
    return;
  }
  ln_normalise(y, d, m->eps, sc->xhat);
  for (int j = 0; j < d; ++j) out[j] = x[j] + (m->gamma[j] * sc->xhat[j] + m->beta[j]);
}

/* Loss l(W; k, v) = || f(k; W) - v ||^2 and, if grad != NULL, its gradient with
 * respect to every parameter of W (same layout as W). */
static double model_loss_grad(const model_t *m, const double *W, const double *k,
                              const double *v, double *grad, scratch_t *sc) {
  const int d = m->d, h = m->h;
  double *a = sc->a, *s = sc->s, *y = sc->y, *xhat = sc->xhat;
  double *dout = sc->g1, *dy = sc->g2;
  double rstd = 0.0;

  /* forward, keeping what the backward needs */
  if (m->kind == ORACLE_MLP_LN) {
    const double *W1 = W, *W2 = W + (long)d * h;
    for (int i = 0; i < h; ++i) {
      double acc = 0.0;
      for (int p = 0; p < d; ++p) acc += k[p] * W1[(long)p * h + i];
      a[i] = acc;
      s[i] = gelu(acc);
    }
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int i = 0; i < h; ++i) acc += s[i] * W2[(long)i * d + j];
      y[j] = acc;
    }
  } else {
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += k[i] * W[(long)i * d + j];
      y[j] = acc;
    }
  }
  double loss = 0.0;
  if (m->kind == ORACLE_LINEAR) {
    for (int j = 0; j < d; ++j) {
      const double r = y[j] - v[j];
      loss += r * r;
      dy[j] = 2.0 * r; /* d l / d y */
    }
  } else {
    rstd = ln_normalise(y, d, m->eps, xhat);
    for (int j = 0; j < d; ++j) {
      const double r = k[j] + (m->gamma[j] * xhat[j] + m->beta[j]) - v[j];
      loss += r * r;
      dout[j] = 2.0 * r * m->gamma[j]; /* d l / d xhat */
    }
    ln_normalise_backward(xhat, rstd, d, dout, dy); /* d l / d y */
  }
  if (!grad) return loss;

  if (m->kind == ORACLE_MLP_LN) {
    const double *W2 = W + (long)d * h;
    double *gW1 = grad, *gW2 = grad + (long)d * h;
    /* y = s W2: dl/dW2[i][j] = s_i dy_j ; dl/ds_i = sum_j W2[i][j] dy_j */
    for (int i = 0; i < h; ++i)
      for (int j = 0; j < d; ++j) gW2[(long)i * d + j] = s[i] * dy[j];
    for (int i = 0; i < h; ++i) {
      double ds = 0.0;
      for (int j = 0; j < d; ++j) ds += W2[(long)i * d + j] * dy[j];
      a[i] = ds * gelu_deriv(a[i]); /* dl/da, overwriting a */
    }
    /* a = k W1: dl/dW1[p][i] = k_p dl/da_i */
    for (int p = 0; p < d; ++p)
      for (int i = 0; i < h; ++i) gW1[(long)p * h + i] = k[p] * a[i];
  } else {
    /* y = k W: dl/dW[i][j] = k_i dy_j */
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) grad[(long)i * d + j] = k[i] * dy[j];
  }
  return loss;
}

/* --- primal mini-batch TTT over one (batch, head) sequence ---------------- */

static int run_sequence(const model_t *m, const double *Q, const double *K, const double *V,
                        const double *eta, const double *W0, int T, int b, double *Z,
                        double *Wout) {
  const int d = m->d;
  const long P = param_count(m);
  double *W = (double *)malloc(sizeof(double) * P);
  double *Wbase = (double *)malloc(sizeof(double) * P);
  double *grad = (double *)malloc(sizeof(double) * P);
  scratch_t sc;
  if (!W || !Wbase || !grad || scratch_init(&sc, m) != 0) {
    free(W);
    free(Wbase);
    free(grad);
    return -2;
  }
  memcpy(W, W0, sizeof(double) * P);
  for (int t = 0; t < T; ++t) {
    if (t % b == 0) memcpy(Wbase, W, sizeof(double) * P); /* t' = t - mod(t, b) */
    const double *k = K + (long)t * d, *v = V + (long)t * d, *q = Q + (long)t * d;
    model_loss_grad(m, Wbase, k, v, grad, &sc); /* G_t at the mini-batch base */
    for (long p = 0; p < P; ++p) W[p] -= eta[t] * grad[p];
    model_apply(m, W, q, Z + (long)t * d, &sc); /* output at the updated W_t */
  }
  memcpy(Wout, W, sizeof(double) * P);
  scratch_free(&sc);
  free(W);
  free(Wbase);
  free(grad);
  return 0;
}

/* --- momentum and decay variant (Titans-style memory update) ------------- */

/* The Titans article (page 4 of the sources, §二.1(2)) adds to the gradient
 * ("surprise") step a momentum on past surprise and a weight decay that forgets.
 * Plainest reading, kept to TTT's mini-batch rule (§03.6; the article calls the
 * update equivalent to mini-batch gradient descent with momentum and weight
 * decay): with S_0 = 0 and t' the base of token t's mini-batch,
 *   S_t = alpha_t S_{t-1} - eta_t grad l(W_{t'}; x_t)
 *   W_t = (1 - lambda_t) W_{t-1} + S_t,     z_t = f(q_t; W_t).
 * alpha = lambda = 0 is TTT itself. */
static int run_sequence_momentum(const model_t *m, const double *Q, const double *K,
                                 const double *V, const double *eta, const double *alpha,
                                 const double *lam, const double *W0, int T, int b, double *Z,
                                 double *Wout, double *Sout) {
  const int d = m->d;
  const long P = param_count(m);
  double *W = (double *)malloc(sizeof(double) * P);
  double *Wbase = (double *)malloc(sizeof(double) * P);
  double *S = (double *)calloc((size_t)P, sizeof(double));
  double *grad = (double *)malloc(sizeof(double) * P);
  scratch_t sc;
  if (!W || !Wbase || !S || !grad || scratch_init(&sc, m) != 0) {
    free(W);
    free(Wbase);
    free(S);
    free(grad);
    return -2;
  }
  memcpy(W, W0, sizeof(double) * P);
  for (int t = 0; t < T; ++t) {
    if (t % b == 0) memcpy(Wbase, W, sizeof(double) * P);
    const double *k = K + (long)t * d, *v = V + (long)t * d, *q = Q + (long)t * d;
    model_loss_grad(m, Wbase, k, v, grad, &sc);
    for (long p = 0; p < P; ++p) {
      S[p] = alpha[t] * S[p] - eta[t] * grad[p];
      W[p] = (1.0 - lam[t]) * W[p] + S[p];
    }
    model_apply(m, W, q, Z + (long)t * d, &sc);
  }
  memcpy(Wout, W, sizeof(double) * P);
  memcpy(Sout, S, sizeof(double) * P);
  scratch_free(&sc);
  free(W);
  free(Wbase);
  free(S);
  free(grad);
  return 0;
}

/* One thread over every unit (the variant is checked at small sizes only).
 * alpha, lam: [B][H][T] like eta; S_out: [B][H][P], the final momentum.
 * Returns 0, -1 on a bad argument, -2 on allocation failure. */
int oracle_ttt_momentum_forward_f64(int kind, const double *Q, const double *K, const double *V,
                                    const double *eta, const double *alpha, const double *lam,
                                    const double *W0, int B, int H, int T, int d, int hidden,
                                    int b, const double *gamma, const double *beta, double eps,
                                    double *Z, double *Wout, double *Sout) {
  if (kind < ORACLE_LINEAR || kind > ORACLE_MLP_LN) return -1;
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0 || T % b != 0) return -1;
  if (kind == ORACLE_MLP_LN && hidden <= 0) return -1;
  if (kind != ORACLE_LINEAR && (!gamma || !beta || !(eps > 0.0))) return -1;
  if ((long)B * H == 0) return 0;
  if (!W0 || !Wout || !Sout || (T > 0 && (!Q || !K || !V || !eta || !alpha || !lam || !Z)))
    return -1;
  model_t m = {kind, d, hidden, NULL, NULL, eps};
  const long P = param_count(&m);
  for (long u = 0; u < (long)B * H; ++u) {
    const int hh = (int)(u % H);
    const long tok = u * (long)T;
    if (kind != ORACLE_LINEAR) {
      m.gamma = gamma + (long)hh * d;
      m.beta = beta + (long)hh * d;
    }
    const int rc = run_sequence_momentum(&m, Q + tok * d, K + tok * d, V + tok * d, eta + tok,
                                         alpha + tok, lam + tok, W0 + (long)hh * P, T, b,
                                         Z + tok * d, Wout + u * P, Sout + u * P);
    if (rc != 0) return rc;
  }
  return 0;
}

/* --- multithreaded driver over (batch, head) units ------------------------- */

typedef struct {
  int kind, B, H, T, d, h, b;
  const double *Q, *K, *V, *eta, *W0, *gamma, *beta;
  double eps;
  double *Z, *Wout;
  atomic_long next;
  atomic_int status;
} job_t;

static void *worker(void *arg) {
  job_t *job = (job_t *)arg;
  const int d = job->d;
  model_t m = {job->kind, d, job->h, NULL, NULL, job->eps};
  const long P = param_count(&m);
  const long units = (long)job->B * job->H;
  for (;;) {
    const long u = atomic_fetch_add(&job->next, 1);
    if (u >= units) break;
    const int hh = (int)(u % job->H);
    const long tok = u * (long)job->T;
    if (job->kind != ORACLE_LINEAR) {
      m.gamma = job->gamma + (long)hh * d;
      m.beta = job->beta + (long)hh * d;
    }
    const int rc = run_sequence(&m, job->Q + tok * d, job->K + tok * d, job->V + tok * d,
                                job->eta + tok, job->W0 + (long)hh * P, job->T, job->b,
                                job->Z + tok * d, job->Wout + u * P);
    if (rc != 0) atomic_store(&job->status, rc);
  }
  return NULL;
}

/* Returns 0 on success, -1 on a bad argument, -2 on allocation failure. */
int oracle_ttt_forward_f64(int kind, const double *Q, const double *K, const double *V,
                           const double *eta, const double *W0, int B, int H, int T, int d,
                           int hidden, int b, const double *gamma, const double *beta,
                           double eps, double *Z, double *Wout, int nthreads) {
  if (kind < ORACLE_LINEAR || kind > ORACLE_MLP_LN) return -1;
  if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0 || T % b != 0) return -1;
  if (kind == ORACLE_MLP_LN && hidden <= 0) return -1;
  if (kind != ORACLE_LINEAR && (!gamma || !beta || !(eps > 0.0))) return -1;
  if ((long)B * H == 0) return 0;
  if (!W0 || !Wout || (T > 0 && (!Q || !K || !V || !eta || !Z))) return -1;
  job_t job;
  job.kind = kind;
  job.B = B;
  job.H = H;
  job.T = T;
  job.d = d;
  job.h = hidden;
  job.b = b;
  job.Q = Q;
  job.K = K;
  job.V = V;
  job.eta = eta;
  job.W0 = W0;
  job.gamma = gamma;
  job.beta = beta;
  job.eps = eps;
  job.Z = Z;
  job.Wout = Wout;
  atomic_init(&job.next, 0);
  atomic_init(&job.status, 0);
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if ((long)nthreads > (long)B * H) nthreads = B * H;
  pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
  if (!tid) return -2;
  int started = 0;
  for (int i = 1; i < nthreads; ++i) {
    if (pthread_create(&tid[i], NULL, worker, &job) != 0) break;
    ++started;
  }
  worker(&job); /* the calling thread works too */
  for (int i = 1; i <= started; ++i) pthread_join(tid[i], NULL);
  free(tid);
  return atomic_load(&job.status);
}

/* Number of worker threads a call with nthreads <= 0 would use. */
int oracle_default_threads(void) { return (int)sysconf(_SC_NPROCESSORS_ONLN); }

/* Per-token loss and gradient of one head, for finite-difference and autograd
 * checks.  grad may be NULL.  Returns the loss, or NAN on a bad argument. */
double oracle_loss_grad_f64(int kind, const double *W, const double *k, const double *v, int d,
                            int hidden, const double *gamma, const double *beta, double eps,
                            double *grad) {
  if (kind < ORACLE_LINEAR || kind > ORACLE_MLP_LN || d <= 0) return NAN;
  if (kind == ORACLE_MLP_LN && hidden <= 0) return NAN;
  model_t m = {kind, d, hidden, gamma, beta, eps};
  scratch_t sc;
  if (scratch_init(&sc, &m) != 0) return NAN;
  const double loss = model_loss_grad(&m, W, k, v, grad, &sc);
  scratch_free(&sc);
  return loss;
}

/* out[d] = f(x; W) for one head.  Returns 0, or -1 on a bad argument. */
int oracle_apply_f64(int kind, const double *W, const double *x, int d, int hidden,
                     const double *gamma, const double *beta, double eps, double *out) {
  if (kind < ORACLE_LINEAR || kind > ORACLE_MLP_LN || d <= 0) return -1;
  if (kind == ORACLE_MLP_LN && hidden <= 0) return -1;
  model_t m = {kind, d, hidden, gamma, beta, eps};
  scratch_t sc;
  if (scratch_init(&sc, &m) != 0) return -2;
  model_apply(&m, W, x, out, &sc);
  scratch_free(&sc);
  return 0;
}
