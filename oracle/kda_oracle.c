/*
 * kda_oracle.c -- fp64 CPU oracle for the Kimi Delta Attention (KDA) path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (libkda, its kernels or
 * its Python binding) links, loads or calls this file; only tests/, the
 * smoke check and the bench's CPU-baseline leg do.  It shares no code,
 * header, constant or helper with the CUDA path.
 *
 * What it computes, in plain sequential fp64, one token at a time:
 *
 *   Gate -- "NLP--技术报告解读-Kimi-K3" (joezjh.github.io), Model Architecture >
 *   Kimi Delta Attention (KDA) > Lower-bounded decay equation:
 *       g_t^h = g_min * Sigmoid(exp(A_h) * z_t^h),   g_min = -5,
 *   with alpha_t = exp(g_t) the channel-wise retention.
 *
 *   Recurrence -- same page and section, state-update equation:
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *       o~_t = S_t^T q_t        (the output reads the state AFTER the update),
 *   with S in R^{dk x dv}.  The product is evaluated in the order the
 *   equation states it: first Diag(alpha_t) S_{t-1} (row i scaled by
 *   alpha_{t,i}), then the delta projection, which for the rank-one matrix
 *   (I - beta k k^T) applied to S' is  S' - beta k (k^T S').  Adding
 *   beta k v^T gives  S' + k (beta (v - S'^T k))^T.  The query scale is a
 *   plain factor on o (the pages print none; callers pass 1.0).
 *
 * Parity pins for every function here live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- gate */

/* g[r, h, i] = g_min / (1 + exp(-exp(A_log[h]) * z[r, h, i]))  (fp64).
 * z and g are [rows, H, dk] contiguous; A_log is [H]. */
void kda_oracle_gate(int64_t rows, int H, int dk, const double *z,
                     const double *A_log, double g_min, double *g) {
  for (int64_t r = 0; r < rows; ++r) {
    for (int h = 0; h < H; ++h) {
      const double a = exp(A_log[h]);
      const int64_t base = (r * H + h) * (int64_t)dk;
      for (int i = 0; i < dk; ++i) {
        const double x = a * z[base + i];
        g[base + i] = g_min * (1.0 / (1.0 + exp(-x)));
      }
    }
  }
}

/* Gradients of the gate above (chain rule; the pages give the forward only):
 * with x = e^{A_h} z and s = sigmoid(x), dg/dz = g_min s (1 - s) e^{A_h} and
 * dg/dA_h = g_min s (1 - s) x, so
 *   dz = dg g_min s (1 - s) e^{A_h},   dA_log[h] = sum over rows, i of dg g_min s (1 - s) x. */
void kda_oracle_gate_backward(int64_t rows, int H, int dk, const double *z,
                              const double *A_log, double g_min, const double *dg,
                              double *dz, double *dA_log) {
  for (int h = 0; h < H; ++h) dA_log[h] = 0.0;
  for (int64_t r = 0; r < rows; ++r) {
    for (int h = 0; h < H; ++h) {
      const double a = exp(A_log[h]);
      const int64_t base = (r * H + h) * (int64_t)dk;
      for (int i = 0; i < dk; ++i) {
        const double x = a * z[base + i];
        const double s = 1.0 / (1.0 + exp(-x));
        const double d = dg[base + i] * g_min * s * (1.0 - s);
        dz[base + i] = d * a;
        dA_log[h] += d * x;
      }
    }
  }
}

/* ----------------------------------------------------------- recurrence */

/* One (sequence, head): tokens t0 .. t0+L-1 of the packed [Ttot, H, *]
 * arrays, head h.  S is this unit's [dk, dv] state, updated in place.
 * o (may be NULL) receives [Ttot, H, dv] outputs at the same rows. */
static void recurrence_unit(int64_t t0, int64_t L, int h, int H, int dk,
                            int dv, const double *q, const double *k,
                            const double *v, const double *g,
                            const double *beta, double scale, double *S,
                            double *o, double *p) {
  for (int64_t t = t0; t < t0 + L; ++t) {
    const double *qt = q + (t * H + h) * (int64_t)dk;
    const double *kt = k + (t * H + h) * (int64_t)dk;
    const double *vt = v + (t * H + h) * (int64_t)dv;
    const double *gt = g + (t * H + h) * (int64_t)dk;
    const double bt = beta[t * H + h];

    /* S' = Diag(alpha_t) S_{t-1} */
    for (int i = 0; i < dk; ++i) {
      const double a = exp(gt[i]);
      for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
    }
    /* p = S'^T k_t */
    for (int j = 0; j < dv; ++j) p[j] = 0.0;
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) p[j] += S[i * dv + j] * kt[i];
    /* e = beta_t (v_t - p);  S_t = S' + k_t e^T */
    for (int j = 0; j < dv; ++j) p[j] = bt * (vt[j] - p[j]);
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * p[j];
    /* o~_t = scale * S_t^T q_t */
    if (o) {
      double *ot = o + (t * H + h) * (int64_t)dv;
      for (int j = 0; j < dv; ++j) ot[j] = 0.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qt[i];
      for (int j = 0; j < dv; ++j) ot[j] *= scale;
    }
  }
}

typedef struct {
  /* shared, read-only */
  const int64_t *seq_off; /* [num_seqs + 1] token offsets */
  const int32_t *units;   /* [num_units, 2] (seq, head) or NULL = all */
  int64_t num_units;
  int H, dk, dv;
  const double *q, *k, *v, *g, *beta, *S0;
  double scale;
  double *o, *S_out;
  /* work distribution */
  int64_t next;
  pthread_mutex_t lock;
} job_t;

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  double *p = (double *)malloc(sizeof(double) * (size_t)J->dv);
  const int64_t state_sz = (int64_t)J->dk * J->dv;
  for (;;) {
    pthread_mutex_lock(&J->lock);
    const int64_t u = J->next++;
    pthread_mutex_unlock(&J->lock);
    if (u >= J->num_units) break;
    int n, h;
    if (J->units) {
      n = J->units[2 * u];
      h = J->units[2 * u + 1];
    } else {
      n = (int)(u / J->H);
      h = (int)(u % J->H);
    }
    /* the unit's state lives in S_out[n, h] (initialised from S0 or 0) */
    double *S = J->S_out + ((int64_t)n * J->H + h) * state_sz;
    if (J->S0)
      memcpy(S, J->S0 + ((int64_t)n * J->H + h) * state_sz,
             sizeof(double) * (size_t)state_sz);
    else
      memset(S, 0, sizeof(double) * (size_t)state_sz);
    const int64_t t0 = J->seq_off[n];
    const int64_t L = J->seq_off[n + 1] - t0;
    recurrence_unit(t0, L, h, J->H, J->dk, J->dv, J->q, J->k, J->v, J->g,
                    J->beta, J->scale, S, J->o, p);
  }
  free(p);
  return NULL;
}

/* Run the recurrence for every (sequence, head) unit, or for the listed
 * units only.  Layouts (all fp64, contiguous):
 *   q, k, g : [Ttot, H, dk]    v : [Ttot, H, dv]    beta : [Ttot, H]
 *   S0      : [num_seqs, H, dk, dv] or NULL (zero initial state)
 *   o       : [Ttot, H, dv] or NULL          S_out : [num_seqs, H, dk, dv]
 * seq_off holds num_seqs+1 non-decreasing token offsets.  Units not listed
 * leave their o rows and S_out slots untouched.  Returns 0 on success. */
int kda_oracle_forward(int num_seqs, const int64_t *seq_off, int H, int dk,
                       int dv, const double *q, const double *k,
                       const double *v, const double *g, const double *beta,
                       const double *S0, double scale, double *o,
                       double *S_out, const int32_t *units, int64_t num_units,
                       int nthreads) {
  if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !seq_off || !S_out)
    return 1;
  for (int n = 0; n < num_seqs; ++n)
    if (seq_off[n + 1] < seq_off[n]) return 2;
  job_t J;
  J.seq_off = seq_off;
  J.units = units;
  J.num_units = units ? num_units : (int64_t)num_seqs * H;
  J.H = H;
  J.dk = dk;
  J.dv = dv;
  J.q = q;
  J.k = k;
  J.v = v;
  J.g = g;
  J.beta = beta;
  J.S0 = S0;
  J.scale = scale;
  J.o = o;
  J.S_out = S_out;
  J.next = 0;
  pthread_mutex_init(&J.lock, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&J.lock);
  return 0;
}

/* ------------------------------------------------------------- backward */

/* Gradients of a loss through the same recurrence, by reverse-mode
 * differentiation of the steps written above (the pages give the forward
 * only; this is the chain rule applied to it, step by step).  Dense layout,
 * one (b, h) unit at a time, all states of the forward kept:
 *
 *   forward   S'_t = Diag(a_t) S_{t-1},  a_t = exp(g_t)
 *             p_t = S'_t^T k_t,  e_t = beta_t (v_t - p_t)
 *             S_t = S'_t + k_t e_t^T,  o_t = scale S_t^T q_t
 *
 *   backward  with G = dL/dS_t (starting from dL/dS_T = d_final, or 0):
 *             G    += scale q_t do_t^T          dq_t  = scale S_t do_t
 *             de    = G^T k_t                   dk_t  = G e_t + S'_t dp
 *             dv_t  = beta_t de                 dbeta = de . (v_t - p_t)
 *             dp    = -beta_t de                G'    = G + k_t dp^T
 *             da_i  = sum_j G'_ij S_{t-1,ij}    dg_t  = da * a_t
 *             G     = Diag(a_t) G'   (= dL/dS_{t-1});   dS_0 = final G.
 *
 * Inputs q, k, g [B, T, H, dk]; v, dout [B, T, H, dv]; beta [B, T, H];
 * S0, dfinal [B, H, dk, dv] or NULL (zeros).  Outputs of the same shapes:
 * dq, dk, dg, dv, dbeta, dS0 (dS0 may be NULL).  Returns 0, or -1 when out of
 * memory. */
int kda_oracle_backward(int B, int64_t T, int H, int dk, int dv, const double *q,
                        const double *k, const double *v, const double *g,
                        const double *beta, const double *S0, const double *dout,
                        const double *dfinal, double scale, double *dq, double *dk_out,
                        double *dv_out, double *dg, double *dbeta, double *dS0) {
  const int64_t SZ = (int64_t)dk * dv;
  double *St = (double *)malloc(sizeof(double) * (size_t)((T + 1) * SZ));
  double *G = (double *)malloc(sizeof(double) * (size_t)SZ);
  double *Sp = (double *)malloc(sizeof(double) * (size_t)SZ);
  double *p = (double *)malloc(sizeof(double) * (size_t)dv);
  double *e = (double *)malloc(sizeof(double) * (size_t)dv);
  double *de = (double *)malloc(sizeof(double) * (size_t)dv);
  double *dp = (double *)malloc(sizeof(double) * (size_t)dv);
  if (!St || !G || !Sp || !p || !e || !de || !dp) {
    free(St); free(G); free(Sp); free(p); free(e); free(de); free(dp);
    return -1;
  }
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < H; ++h) {
      const int64_t unit = (int64_t)b * H + h;
      /* forward, keeping S_0 .. S_T */
      for (int64_t x = 0; x < SZ; ++x) St[x] = S0 ? S0[unit * SZ + x] : 0.0;
      for (int64_t t = 0; t < T; ++t) {
        const int64_t r = (int64_t)b * T + t;
        const double *kt = k + (r * H + h) * (int64_t)dk;
        const double *vt = v + (r * H + h) * (int64_t)dv;
        const double *gt = g + (r * H + h) * (int64_t)dk;
        const double bt = beta[r * H + h];
        const double *prev = St + t * SZ;
        double *cur = St + (t + 1) * SZ;
        for (int i = 0; i < dk; ++i) {
          const double a = exp(gt[i]);
          for (int j = 0; j < dv; ++j) cur[i * dv + j] = a * prev[i * dv + j];
        }
        for (int j = 0; j < dv; ++j) p[j] = 0.0;
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) p[j] += cur[i * dv + j] * kt[i];
        for (int j = 0; j < dv; ++j) e[j] = bt * (vt[j] - p[j]);
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) cur[i * dv + j] += kt[i] * e[j];
      }
      /* backward */
      for (int64_t x = 0; x < SZ; ++x) G[x] = dfinal ? dfinal[unit * SZ + x] : 0.0;
      for (int64_t t = T - 1; t >= 0; --t) {
        const int64_t r = (int64_t)b * T + t;
        const double *qt = q + (r * H + h) * (int64_t)dk;
        const double *kt = k + (r * H + h) * (int64_t)dk;
        const double *vt = v + (r * H + h) * (int64_t)dv;
        const double *gt = g + (r * H + h) * (int64_t)dk;
        const double *dot = dout + (r * H + h) * (int64_t)dv;
        const double bt = beta[r * H + h];
        const double *pre = St + t * SZ, *post = St + (t + 1) * SZ;
        double *dqt = dq + (r * H + h) * (int64_t)dk;
        double *dkt = dk_out + (r * H + h) * (int64_t)dk;
        double *dvt = dv_out + (r * H + h) * (int64_t)dv;
        double *dgt = dg + (r * H + h) * (int64_t)dk;
        /* output: o_t = scale S_t^T q_t */
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) G[i * dv + j] += scale * qt[i] * dot[j];
        for (int i = 0; i < dk; ++i) {
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) acc += post[i * dv + j] * dot[j];
          dqt[i] = scale * acc;
        }
        /* recompute S'_t, p_t, e_t */
        for (int i = 0; i < dk; ++i) {
          const double a = exp(gt[i]);
          for (int j = 0; j < dv; ++j) Sp[i * dv + j] = a * pre[i * dv + j];
        }
        for (int j = 0; j < dv; ++j) p[j] = 0.0;
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) p[j] += Sp[i * dv + j] * kt[i];
        for (int j = 0; j < dv; ++j) e[j] = bt * (vt[j] - p[j]);
        /* S_t = S' + k e^T */
        for (int j = 0; j < dv; ++j) de[j] = 0.0;
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) de[j] += G[i * dv + j] * kt[i];
        for (int i = 0; i < dk; ++i) {
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) acc += G[i * dv + j] * e[j];
          dkt[i] = acc;
        }
        /* e = beta (v - p) */
        double db = 0.0;
        for (int j = 0; j < dv; ++j) {
          dvt[j] = bt * de[j];
          db += de[j] * (vt[j] - p[j]);
          dp[j] = -bt * de[j];
        }
        dbeta[r * H + h] = db;
        /* p = S'^T k: G' = G + k dp^T, dk += S' dp */
        for (int i = 0; i < dk; ++i) {
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) {
            G[i * dv + j] += kt[i] * dp[j];
            acc += Sp[i * dv + j] * dp[j];
          }
          dkt[i] += acc;
        }
        /* S' = Diag(a) S_{t-1} */
        for (int i = 0; i < dk; ++i) {
          const double a = exp(gt[i]);
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) {
            acc += G[i * dv + j] * pre[i * dv + j];
            G[i * dv + j] *= a;
          }
          dgt[i] = acc * a;
        }
      }
      if (dS0)
        for (int64_t x = 0; x < SZ; ++x) dS0[unit * SZ + x] = G[x];
    }
  }
  free(St); free(G); free(Sp); free(p); free(e); free(de); free(dp);
  return 0;
}

