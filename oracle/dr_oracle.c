/*
 * dr_oracle.c -- plain fp64 CPU oracle for gated delta-rule linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes is the plain token-by-token definition of the recurrence,
 * with no chunking, blocking or reordering:
 *
 *   P_t = S_{t-1} Diag(alpha_t)                         (decay, alpha = exp g)
 *   S_t = P_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T  (erase then write)
 *       = P_t + beta_t (v_t - P_t k_t) k_t^T
 *   o_t = S_t q_t                                        (read after write)
 *
 * S is d_v x d_k.  This is the transpose of the update
 * S_t = (I - beta_t k_t k_t^*) Lambda_t S_{t-1} + beta_t k_t v_t^* printed in
 * "Semidirect Fourier Delta Attention" (gist.science explainer, section
 * "Kernarchitektur") with the phase theta set to zero, which that page states
 * recovers Kimi Delta Attention (KDA); the delta-rule erase-and-write itself
 * is the one the ReWY abstract (paperdot listing) builds on for DeltaNet, GDN
 * and KDA.
 *
 * Gate kinds: none (alpha = 1, DeltaNet), scalar (one log-gate per head and
 * token, GDN), per-channel (one log-gate per key channel, KDA) and phase
 * (SFDA, same explainer, "Kernarchitektur": the complex diagonal
 * Lambda_t = diag(alpha_t e^{i theta_t}) written in real coordinates as a
 * direct sum of 2 x 2 rotation-decay blocks).  For the phase gate the key
 * channels pair up as (2j, 2j+1), one complex coordinate each; g holds
 * log alpha_j at channel 2j and theta_j at channel 2j+1, and the decay maps a
 * state row's pair (x, y) -- the real and imaginary parts of that coordinate --
 * to alpha_j (cos theta_j x - sin theta_j y, sin theta_j x + cos theta_j y).
 * Keys, queries and values stay real, and the erase-and-write is the real
 * rank-one correction above (the reading of the page's update in real
 * coordinates); zero phase gives KDA with both channels of a pair sharing
 * one decay.
 * Beta modes: direct (beta is the input) and Kaczmarz (KLA abstract,
 * thelatestinai.com): beta_t = eta_t / (||k_t||^2 + eps), the input being eta.
 *
 * The backward is a hand-derived reverse-mode pass of the same recurrence,
 * token by token in reverse, with the states re-run forward from checkpoints.
 * For a scalar loss L with dL/do_t = do_t and dL/dS_T = dS_T, per step t
 * (dS holds dL/dS_t on entry):
 *   dS  += do_t q_t^T                 dq_t = S_t^T do_t
 *   w    = dS k_t                     dbeta_t = e_t . w      (e_t = v_t - P_t k_t)
 *   de   = beta_t w                   dv_t = de
 *   dk_t = beta_t dS^T e_t - P_t^T de
 *   dP   = dS - de k_t^T
 *   dg_t[c] = sum_a dP[a,c] P[a,c]    (gradient w.r.t. log alpha; summed over
 *                                      c for a scalar gate)
 *   dS_{t-1} = dP Diag(alpha_t)
 * For the phase gate, with (Px, Py) and (dPx, dPy) a row's pair j of P, dP:
 *   dg_t[2j]   = sum_a (dPx Px + dPy Py)          (d/d log alpha_j)
 *   dg_t[2j+1] = sum_a (dPy Px - dPx Py)          (d/d theta_j)
 *   dS_{t-1} pair = alpha_j (cos theta_j dPx + sin theta_j dPy,
 *                            -sin theta_j dPx + cos theta_j dPy)   (Lambda^T dP)
 * Kaczmarz mode adds the chain through beta = eta/(n+eps), n = ||k||^2:
 *   deta = dbeta/(n+eps),  dk_t += -2 beta dbeta k_t/(n+eps).
 *
 * Layouts (row-major, all fp64):
 *   q, k      [B, T, H, dk]      v, o, dO  [B, T, H, dv]
 *   beta      [B, T, H]          (eta in Kaczmarz mode)
 *   g         [B, T, H] (scalar) or [B, T, H, dk] (per-channel, phase); unused
 *             for none
 *   S0, ST, dST, dS0   [B, H, dv, dk]   (S0/dST may be NULL = zero)
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GATE_NONE 0
#define ORACLE_GATE_SCALAR 1
#define ORACLE_GATE_CHANNEL 2
#define ORACLE_GATE_PHASE 3
#define ORACLE_BETA_DIRECT 0
#define ORACLE_BETA_KACZMARZ 1

typedef struct {
  int B, H, T, dk, dv, gate, beta_mode;
  double eps;
} oproblem;

/* alpha_t for channel c of head (b,h) at token t. */
static double oracle_alpha(const oproblem* p, const double* g, int b, int t, int h,
                           int c) {
  if (p->gate == ORACLE_GATE_NONE) return 1.0;
  size_t row = ((size_t)b * p->T + t) * p->H + h;
  if (p->gate == ORACLE_GATE_SCALAR) return exp(g[row]);
  return exp(g[row * p->dk + c]);
}

/* The decay of token t for head (b,h): alpha[c] for the diagonal gates; for
   the phase gate ac[j] = alpha_j cos theta_j, as[j] = alpha_j sin theta_j. */
static void oracle_decay(const oproblem* p, const double* g, int b, int t, int h,
                         double* alpha, double* ac, double* as) {
  if (p->gate != ORACLE_GATE_PHASE) {
    for (int c = 0; c < p->dk; ++c) alpha[c] = oracle_alpha(p, g, b, t, h, c);
    return;
  }
  size_t row = ((size_t)b * p->T + t) * p->H + h;
  for (int j = 0; j < p->dk / 2; ++j) {
    double al = exp(g[row * p->dk + 2 * j]), th = g[row * p->dk + 2 * j + 1];
    ac[j] = al * cos(th);
    as[j] = al * sin(th);
  }
}

/* Applies the decay to one state row in place (row . Lambda^T). */
static void oracle_decay_row(const oproblem* p, double* Sa, const double* alpha,
                             const double* ac, const double* as) {
  if (p->gate != ORACLE_GATE_PHASE) {
    for (int c = 0; c < p->dk; ++c) Sa[c] *= alpha[c];
    return;
  }
  for (int j = 0; j < p->dk / 2; ++j) {
    double x = Sa[2 * j], y = Sa[2 * j + 1];
    Sa[2 * j] = ac[j] * x - as[j] * y;
    Sa[2 * j + 1] = as[j] * x + ac[j] * y;
  }
}

/* Effective beta_t and the key norm n_t = ||k_t||^2. */
static double oracle_beta(const oproblem* p, const double* beta, const double* kt,
                          size_t row, double* norm_out) {
  double n = 0.0;
  for (int c = 0; c < p->dk; ++c) n += kt[c] * kt[c];
  if (norm_out) *norm_out = n;
  if (p->beta_mode == ORACLE_BETA_KACZMARZ) return beta[row] / (n + p->eps);
  return beta[row];
}

/* One recurrence step in place: S <- P + beta (v - P k) k^T with P = S Lambda^T
   (P = S Diag(alpha) for the diagonal gates).
   If P_out is non-NULL it receives P; e_out receives e = v - P k. */
static void oracle_step(const oproblem* p, double* S, const double* alpha,
                        const double* ac, const double* as, const double* kt,
                        const double* vt, double bt, double* P_out, double* e_out) {
  const int dk = p->dk, dv = p->dv;
  for (int a = 0; a < dv; ++a) {
    double* Sa = S + (size_t)a * dk;
    double pk = 0.0;
    oracle_decay_row(p, Sa, alpha, ac, as);
    for (int c = 0; c < dk; ++c) pk += Sa[c] * kt[c];
    if (P_out) memcpy(P_out + (size_t)a * dk, Sa, sizeof(double) * dk);
    double e = vt[a] - pk;
    if (e_out) e_out[a] = e;
    double s = bt * e;
    for (int c = 0; c < dk; ++c) Sa[c] += s * kt[c];
  }
}

static void oracle_fwd_head(const oproblem* p, int b, int h, const double* q,
                            const double* k, const double* v, const double* beta,
                            const double* g, const double* S0, double* o, double* ST) {
  const int dk = p->dk, dv = p->dv, H = p->H;
  const size_t SS = (size_t)dv * dk;
  double* S = (double*)malloc(sizeof(double) * SS);
  double* alpha = (double*)malloc(sizeof(double) * dk);
  double* ac = (double*)malloc(sizeof(double) * (dk / 2 + 1));
  double* as = (double*)malloc(sizeof(double) * (dk / 2 + 1));
  if (S0)
    memcpy(S, S0 + ((size_t)b * H + h) * SS, sizeof(double) * SS);
  else
    memset(S, 0, sizeof(double) * SS);
  for (int t = 0; t < p->T; ++t) {
    size_t row = ((size_t)b * p->T + t) * H + h;
    const double* qt = q + row * dk;
    const double* kt = k + row * dk;
    const double* vt = v + row * dv;
    oracle_decay(p, g, b, t, h, alpha, ac, as);
    double bt = oracle_beta(p, beta, kt, row, NULL);
    oracle_step(p, S, alpha, ac, as, kt, vt, bt, NULL, NULL);
    double* ot = o + row * dv;
    for (int a = 0; a < dv; ++a) {
      double acc = 0.0;
      const double* Sa = S + (size_t)a * dk;
      for (int c = 0; c < dk; ++c) acc += Sa[c] * qt[c];
      ot[a] = acc;
    }
  }
  if (ST) memcpy(ST + ((size_t)b * H + h) * SS, S, sizeof(double) * SS);
  free(S);
  free(alpha);
  free(ac);
  free(as);
}

/* Checkpoint spacing: 64 tokens, doubled until there are no more checkpoints
   than tokens per segment (keeps memory near 2*sqrt(T) states per head). */
static int oracle_ckpt_len(int T) {
  int L = 64;
  while ((T + L - 1) / L > L) L *= 2;
  return L;
}

static void oracle_bwd_head(const oproblem* p, int b, int h, const double* q,
                            const double* k, const double* v, const double* beta,
                            const double* g, const double* S0, const double* dO,
                            const double* dST, double* dq, double* dk_out, double* dv_out,
                            double* dbeta, double* dg, double* dS0) {
  const int dk = p->dk, dv = p->dv, H = p->H, T = p->T;
  const size_t SS = (size_t)dv * dk;
  const int L = oracle_ckpt_len(T);
  const int nseg = (T + L - 1) / L;
  double* ckpt = (double*)malloc(sizeof(double) * SS * (size_t)(nseg > 0 ? nseg : 1));
  double* Sbuf = (double*)malloc(sizeof(double) * SS * (size_t)(L + 1));
  double* P = (double*)malloc(sizeof(double) * SS);
  double* dS = (double*)malloc(sizeof(double) * SS);
  double* alpha = (double*)malloc(sizeof(double) * dk);
  double* ac = (double*)malloc(sizeof(double) * (dk / 2 + 1));
  double* as = (double*)malloc(sizeof(double) * (dk / 2 + 1));
  double* e = (double*)malloc(sizeof(double) * dv);
  double* w = (double*)malloc(sizeof(double) * dv);
  double* dgc = (double*)malloc(sizeof(double) * dk);

  /* Forward pass recording the state at the start of every segment. */
  double* S = Sbuf; /* scratch for the first pass */
  if (S0)
    memcpy(S, S0 + ((size_t)b * H + h) * SS, sizeof(double) * SS);
  else
    memset(S, 0, sizeof(double) * SS);
  for (int t = 0; t < T; ++t) {
    if (t % L == 0) memcpy(ckpt + (size_t)(t / L) * SS, S, sizeof(double) * SS);
    size_t row = ((size_t)b * T + t) * H + h;
    oracle_decay(p, g, b, t, h, alpha, ac, as);
    double bt = oracle_beta(p, beta, k + row * dk, row, NULL);
    oracle_step(p, S, alpha, ac, as, k + row * dk, v + row * dv, bt, NULL, NULL);
  }

  if (dST)
    memcpy(dS, dST + ((size_t)b * H + h) * SS, sizeof(double) * SS);
  else
    memset(dS, 0, sizeof(double) * SS);

  for (int seg = nseg - 1; seg >= 0; --seg) {
    const int t0 = seg * L;
    const int t1 = (t0 + L < T) ? t0 + L : T;
    /* Re-run the segment forward: Sbuf[j] = state after t0 + j tokens. */
    memcpy(Sbuf, ckpt + (size_t)seg * SS, sizeof(double) * SS);
    for (int t = t0; t < t1; ++t) {
      size_t row = ((size_t)b * T + t) * H + h;
      double* Sn = Sbuf + (size_t)(t - t0 + 1) * SS;
      memcpy(Sn, Sbuf + (size_t)(t - t0) * SS, sizeof(double) * SS);
      oracle_decay(p, g, b, t, h, alpha, ac, as);
      double bt = oracle_beta(p, beta, k + row * dk, row, NULL);
      oracle_step(p, Sn, alpha, ac, as, k + row * dk, v + row * dv, bt, NULL, NULL);
    }
    for (int t = t1 - 1; t >= t0; --t) {
      size_t row = ((size_t)b * T + t) * H + h;
      const double* qt = q + row * dk;
      const double* kt = k + row * dk;
      const double* vt = v + row * dv;
      const double* dot = dO + row * dv;
      const double* Sprev = Sbuf + (size_t)(t - t0) * SS;
      const double* Snew = Sbuf + (size_t)(t - t0 + 1) * SS;
      double n;
      double bt = oracle_beta(p, beta, kt, row, &n);
      oracle_decay(p, g, b, t, h, alpha, ac, as);

      /* o_t = S_t q_t */
      for (int a = 0; a < dv; ++a)
        for (int c = 0; c < dk; ++c) dS[(size_t)a * dk + c] += dot[a] * qt[c];
      double* dqt = dq + row * dk;
      for (int c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int a = 0; a < dv; ++a) acc += Snew[(size_t)a * dk + c] * dot[a];
        dqt[c] = acc;
      }
      /* P = S_{t-1} Lambda^T (S_{t-1} Diag(alpha) for the diagonal gates),
         e = v - P k */
      for (int a = 0; a < dv; ++a) {
        double* Pa = P + (size_t)a * dk;
        memcpy(Pa, Sprev + (size_t)a * dk, sizeof(double) * dk);
        oracle_decay_row(p, Pa, alpha, ac, as);
        double pk = 0.0;
        for (int c = 0; c < dk; ++c) pk += Pa[c] * kt[c];
        e[a] = vt[a] - pk;
      }
      /* S_t = P + beta e k^T */
      double db = 0.0;
      for (int a = 0; a < dv; ++a) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += dS[(size_t)a * dk + c] * kt[c];
        w[a] = acc;
        db += e[a] * acc;
      }
      double* dkt = dk_out + row * dk;
      double* dvt = dv_out + row * dv;
      for (int a = 0; a < dv; ++a) dvt[a] = bt * w[a]; /* de = beta w */
      for (int c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int a = 0; a < dv; ++a)
          acc += bt * dS[(size_t)a * dk + c] * e[a] - P[(size_t)a * dk + c] * dvt[a];
        dkt[c] = acc;
      }
      /* dP = dS - de k^T ; dg ; dS_{t-1} = dP Lambda (dP Diag(alpha)) */
      for (int c = 0; c < dk; ++c) dgc[c] = 0.0;
      if (p->gate == ORACLE_GATE_PHASE) {
        for (int a = 0; a < dv; ++a) {
          for (int j = 0; j < dk / 2; ++j) {
            size_t ix = (size_t)a * dk + 2 * j;
            double dpx = dS[ix] - dvt[a] * kt[2 * j];
            double dpy = dS[ix + 1] - dvt[a] * kt[2 * j + 1];
            double px = P[ix], py = P[ix + 1];
            dgc[2 * j] += dpx * px + dpy * py;
            dgc[2 * j + 1] += dpy * px - dpx * py;
            dS[ix] = ac[j] * dpx + as[j] * dpy;
            dS[ix + 1] = -as[j] * dpx + ac[j] * dpy;
          }
        }
      } else {
        for (int a = 0; a < dv; ++a) {
          for (int c = 0; c < dk; ++c) {
            size_t ix = (size_t)a * dk + c;
            double dp = dS[ix] - dvt[a] * kt[c];
            dgc[c] += dp * P[ix];
            dS[ix] = dp * alpha[c];
          }
        }
      }
      if (p->gate == ORACLE_GATE_CHANNEL || p->gate == ORACLE_GATE_PHASE) {
        for (int c = 0; c < dk; ++c) dg[row * dk + c] = dgc[c];
      } else if (p->gate == ORACLE_GATE_SCALAR) {
        double s = 0.0;
        for (int c = 0; c < dk; ++c) s += dgc[c];
        dg[row] = s;
      }
      if (p->beta_mode == ORACLE_BETA_KACZMARZ) {
        double den = n + p->eps;
        for (int c = 0; c < dk; ++c) dkt[c] += -2.0 * bt * db * kt[c] / den;
        dbeta[row] = db / den;
      } else {
        dbeta[row] = db;
      }
    }
  }
  memcpy(dS0 + ((size_t)b * H + h) * SS, dS, sizeof(double) * SS);
  free(ckpt);
  free(Sbuf);
  free(P);
  free(dS);
  free(alpha);
  free(ac);
  free(as);
  free(e);
  free(w);
  free(dgc);
}

static oproblem make_problem(int B, int H, int T, int dk, int dv, int gate, int beta_mode,
                             double eps) {
  oproblem p;
  p.B = B;
  p.H = H;
  p.T = T;
  p.dk = dk;
  p.dv = dv;
  p.gate = gate;
  p.beta_mode = beta_mode;
  p.eps = eps;
  return p;
}

/* Forward over all heads; OpenMP over (b, h). Returns the thread count used. */
int oracle_fwd(int B, int H, int T, int dk, int dv, int gate, int beta_mode, double eps,
               const double* q, const double* k, const double* v, const double* beta,
               const double* g, const double* S0, double* o, double* ST) {
  oproblem p = make_problem(B, H, T, dk, dv, gate, beta_mode, eps);
  int used = 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < B * H; ++bh) {
#ifdef _OPENMP
    if (bh == 0) used = omp_get_num_threads();
#endif
    oracle_fwd_head(&p, bh / H, bh % H, q, k, v, beta, g, S0, o, ST);
  }
  return used;
}

/* Backward over all heads; OpenMP over (b, h). dg may be NULL for gate none.
   Returns the thread count used. */
int oracle_bwd(int B, int H, int T, int dk, int dv, int gate, int beta_mode, double eps,
               const double* q, const double* k, const double* v, const double* beta,
               const double* g, const double* S0, const double* dO, const double* dST,
               double* dq, double* dk_out, double* dv_out, double* dbeta, double* dg,
               double* dS0) {
  oproblem p = make_problem(B, H, T, dk, dv, gate, beta_mode, eps);
  int used = 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < B * H; ++bh) {
#ifdef _OPENMP
    if (bh == 0) used = omp_get_num_threads();
#endif
    oracle_bwd_head(&p, bh / H, bh % H, q, k, v, beta, g, S0, dO, dST, dq, dk_out, dv_out,
                    dbeta, dg, dS0);
  }
  return used;
}
