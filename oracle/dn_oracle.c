/*
 * fp64 CPU oracle of the gated delta-rule recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. It shares no code with
 * the CUDA path and is deliberately plain: one sequential loop over tokens per
 * (batch, head), in double precision, written straight from the definitions.
 *
 * Definitions followed (key-major state S in R^{dk x dv}):
 *   decay     S_bar = Diag(alpha_t) S_{t-1}
 *             scalar alpha: Gated DeltaNet forget gate (FG2-GDN page, section 1;
 *             Sparse Delta Memory page, "Gated Delta Updates", forget gate applied
 *             before the delta step); vector alpha in R^dk: KDA channel-wise decay
 *             (FG2-GDN page, section 1).
 *   write key w_t = beta^k_t (.) d_t (.) k_t
 *             vector beta^k: FG2-GDN+ erase strength (FG2-GDN page, section 2.B);
 *             d_t: OSDN preconditioner applied as a write-key scaling
 *             (OSDN page, section 2.1, the right-preconditioning identity).
 *   residual  u_t = beta^v_t (.) v_t - S_bar^T k_t
 *             the prediction uses the raw key k_t (OSDN page, section 2.1: the
 *             residual v - S k keeps the unscaled key); beta^v is the FG2-GDN+
 *             write strength (FG2-GDN page, section 2.B).
 *   update    S_t = S_bar + w_t u_t^T
 *             = (I - w_t k_t^T) Diag(alpha_t) S_{t-1} + w_t (beta^v_t (.) v_t)^T,
 *             the delta rule as one online-gradient step on 0.5 ||S k - v||^2
 *             (OSDN page, section 1), transposed to the key-major orientation.
 *   readout   o_t = S_t^T q_t  (after the update, no 1/sqrt(dk) scaling), or, with pre_read,
 *             o_t = S_{t-1}^T q_t: the state before token t's decay and write (the read of the
 *             delta-mem page, section 2.C, r_t = S_{t-1} q_t, transposed to key-major).
 *
 * Gate widths: 0 = absent (the gate is 1), 1 = one value per token, n = one value
 * per channel (n = dk for alpha, beta^k, d; n = dv for beta^v).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static inline double gate(const double* g, int width, int t, int i) {
  if (width == 0) return 1.0;
  if (width == 1) return g[t];
  return g[(int64_t)t * width + i];
}

/*
 * One (batch, head) sequence.
 *   q, k: [T][dk]   v: [T][dv]   gates: [T][width]
 *   S:    [dk][dv]  in: initial state, out: final state
 *   o:    [T][dv]
 * Returns 0, or -1 on a bad argument / allocation failure.
 */
int dn_oracle_head(int T, int dk, int dv, const double* q, const double* k, const double* v,
                   const double* alpha, int alpha_w, const double* beta_k, int bk_w,
                   const double* beta_v, int bv_w, const double* key_scale, int d_w, double* S,
                   double* o, int pre_read) {
  if (T < 0 || dk <= 0 || dv <= 0 || !S) return -1;
  if (!(alpha_w == 0 || alpha_w == 1 || alpha_w == dk)) return -1;
  if (!(bk_w == 0 || bk_w == 1 || bk_w == dk)) return -1;
  if (!(bv_w == 0 || bv_w == 1 || bv_w == dv)) return -1;
  if (!(d_w == 0 || d_w == 1 || d_w == dk)) return -1;
  double* w = (double*)malloc(sizeof(double) * (size_t)dk);
  double* u = (double*)malloc(sizeof(double) * (size_t)dv);
  if (!w || !u) {
    free(w);
    free(u);
    return -1;
  }
  for (int t = 0; t < T; ++t) {
    const double* kt = k + (int64_t)t * dk;
    const double* qt = q + (int64_t)t * dk;
    const double* vt = v + (int64_t)t * dv;
    double* ot = o + (int64_t)t * dv;
    if (pre_read) {
      /* o_t = S_{t-1}^T q_t, before this token's decay and write */
      for (int j = 0; j < dv; ++j) ot[j] = 0.0;
      for (int i = 0; i < dk; ++i) {
        const double* Si = S + (int64_t)i * dv;
        const double qpre = qt[i];
        for (int j = 0; j < dv; ++j) ot[j] += Si[j] * qpre;
      }
    }
    /* S_bar = Diag(alpha_t) S_{t-1}: row i of S scales by alpha_t[i] */
    for (int i = 0; i < dk; ++i) {
      double a = gate(alpha, alpha_w, t, i);
      double* Si = S + (int64_t)i * dv;
      for (int j = 0; j < dv; ++j) Si[j] *= a;
    }
    /* w_t = beta^k (.) d (.) k */
    for (int i = 0; i < dk; ++i) w[i] = gate(beta_k, bk_w, t, i) * gate(key_scale, d_w, t, i) * kt[i];
    /* u_t = beta^v (.) v - S_bar^T k */
    for (int j = 0; j < dv; ++j) u[j] = gate(beta_v, bv_w, t, j) * vt[j];
    for (int i = 0; i < dk; ++i) {
      const double* Si = S + (int64_t)i * dv;
      double ki = kt[i];
      for (int j = 0; j < dv; ++j) u[j] -= Si[j] * ki;
    }
    /* S_t = S_bar + w u^T */
    for (int i = 0; i < dk; ++i) {
      double* Si = S + (int64_t)i * dv;
      double wi = w[i];
      for (int j = 0; j < dv; ++j) Si[j] += wi * u[j];
    }
    if (pre_read) continue;
    /* o_t = S_t^T q_t */
    for (int j = 0; j < dv; ++j) ot[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
      const double* Si = S + (int64_t)i * dv;
      double qi = qt[i];
      for (int j = 0; j < dv; ++j) ot[j] += Si[j] * qi;
    }
  }
  free(w);
  free(u);
  return 0;
}

/*
 * NH independent heads, each laid out contiguously ([NH][T][...], [NH][dk][dv]).
 * A gate pointer may be NULL exactly when its width is 0. Heads run in parallel
 * on `nthreads` OpenMP threads (<= 0: the OpenMP default). Returns 0 or -1.
 */
int dn_oracle_heads(int NH, int T, int dk, int dv, const double* q, const double* k,
                    const double* v, const double* alpha, int alpha_w, const double* beta_k,
                    int bk_w, const double* beta_v, int bv_w, const double* key_scale, int d_w,
                    double* S, double* o, int pre_read, int nthreads) {
  if (NH < 0) return -1;
  int bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int h = 0; h < NH; ++h) {
    int64_t tk = (int64_t)h * T * dk, tv = (int64_t)h * T * dv;
    int rc = dn_oracle_head(
        T, dk, dv, q + tk, k + tk, v + tv, alpha ? alpha + (int64_t)h * T * alpha_w : NULL, alpha_w,
        beta_k ? beta_k + (int64_t)h * T * bk_w : NULL, bk_w,
        beta_v ? beta_v + (int64_t)h * T * bv_w : NULL, bv_w,
        key_scale ? key_scale + (int64_t)h * T * d_w : NULL, d_w, S + (int64_t)h * dk * dv, o + tv,
        pre_read);
    bad |= (rc != 0);
  }
  return bad ? -1 : 0;
}

/*
 * OSDN phase 1: the diagonal preconditioner sequence of one (batch, head)
 * (OSDN page, section 2.2 "decoupled hypergradient feedback" and section 2.3
 * "adaptive preconditioner forgetting").
 *
 * The per-token surrogate of the preconditioner is, in closed form,
 *   h_t(d) = ((1 - beta_t <d, k_t (.) k_t>)^2 - 1) / (2 ||k_t||^2),
 * whose gradient in d is
 *   grad h_t(d) = -beta_t (1 - beta_t <d, k_t (.) k_t>) (k_t (.) k_t) / ||k_t||^2.
 * Token t is written with the preconditioner d_t (the key scale d of the main
 * recurrence), then one online-gradient-descent step with retention r_t follows:
 *   d_{t+1} = r_t d_t - eta grad h_t(d_t)
 * (r_t = 1 without retention). A token with k_t = 0 has no gradient and leaves
 * d unchanged apart from the retention.
 *
 *   k: [T][dk]  beta: [T]  r: [T] or NULL  d: [dk] in: d_0, out: d_T
 *   dseq: [T][dk] out: d_t for every token
 */
int dn_oracle_osdn_head(int T, int dk, const double* k, const double* beta, const double* r,
                        double eta, double* d, double* dseq) {
  if (T < 0 || dk <= 0 || !d || !dseq || (T > 0 && (!k || !beta))) return -1;
  for (int t = 0; t < T; ++t) {
    const double* kt = k + (int64_t)t * dk;
    double* out = dseq + (int64_t)t * dk;
    double dot = 0.0, nrm = 0.0;
    for (int i = 0; i < dk; ++i) {
      out[i] = d[i];
      dot += d[i] * kt[i] * kt[i];
      nrm += kt[i] * kt[i];
    }
    const double rt = r ? r[t] : 1.0;
    const double g = 1.0 - beta[t] * dot;
    for (int i = 0; i < dk; ++i) {
      const double grad = nrm > 0.0 ? -beta[t] * g * kt[i] * kt[i] / nrm : 0.0;
      d[i] = rt * d[i] - eta * grad;
    }
  }
  return 0;
}

/* NH heads of OSDN phase 1, laid out contiguously ([NH][T][dk], [NH][T], [NH][dk]). */
int dn_oracle_osdn_heads(int NH, int T, int dk, const double* k, const double* beta, const double* r,
                         double eta, double* d, double* dseq, int nthreads) {
  if (NH < 0) return -1;
  int bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int h = 0; h < NH; ++h) {
    int rc = dn_oracle_osdn_head(T, dk, k + (int64_t)h * T * dk, beta + (int64_t)h * T,
                                 r ? r + (int64_t)h * T : NULL, eta, d + (int64_t)h * dk,
                                 dseq + (int64_t)h * T * dk);
    bad |= (rc != 0);
  }
  return bad ? -1 : 0;
}

/*
 * Reverse mode of dn_oracle_head: the gradients of a scalar loss
 *   L = sum_t <dO_t, o_t> + <dS_T, S_T>
 * with respect to every input, for one (batch, head). This is the chain rule
 * applied to the per-token steps above, walked from the last token to the first
 * (the training pass the FG2-GDN page, section 3 item 2, says the chunked form
 * serves; the pages print no backward, so it is derived here from the forward).
 *
 * Per token, with S_prev = S_{t-1}, S_bar = Diag(alpha_t) S_prev,
 * u = beta^v (.) v - S_bar^T k, S_t = S_bar + w u^T, and dS the adjoint of S_t:
 *   post read-out:  dS += q dO^T,  dq = S_t dO          (o_t = S_t^T q_t)
 *   dw = dS u,  du = dS^T w
 *   dS_bar = dS - k du^T                    (S_t = S_bar + w u^T, u = ... - S_bar^T k)
 *   dk = (beta^k (.) d) (.) dw - S_bar du
 *   dv = beta^v (.) du,  dbeta^v = v (.) du,  dbeta^k = d (.) k (.) dw,  dd = beta^k (.) k (.) dw
 *   dalpha_i = sum_j dS_bar_ij S_prev_ij
 *   dS_prev = Diag(alpha_t) dS_bar
 *   pre read-out:   dq = S_prev dO,  dS_prev += q dO^T   (o_t = S_{t-1}^T q_t)
 * A gate of width 1 gets the sum of its per-channel gradient. dS starts at dS_T
 * (NULL: zero) and ends as dS0.
 *
 * The forward states are not reversed algebraically (dividing by alpha and undoing
 * the erase is ill-conditioned): S is kept every `ck` tokens and each block of
 * states is recomputed from its checkpoint with the forward steps.
 *
 *   q, k, dq, dk: [T][dk]   v, dO, dv: [T][dv]   gates and their gradients: [T][width]
 *   S0, dS0: [dk][dv]  (S0 NULL: zero; dS_T NULL: zero)
 * Gradient pointers of absent gates (width 0) are ignored. Returns 0 or -1.
 */
static void fwd_token(int dk, int dv, const double* qt, const double* kt, const double* vt,
                      const double* alpha, int alpha_w, const double* beta_k, int bk_w,
                      const double* beta_v, int bv_w, const double* key_scale, int d_w, int t,
                      const double* S_prev, double* S_bar, double* w, double* u, double* S_t) {
  (void)qt;
  for (int i = 0; i < dk; ++i) {
    const double decay = gate(alpha, alpha_w, t, i);
    for (int j = 0; j < dv; ++j) S_bar[(int64_t)i * dv + j] = decay * S_prev[(int64_t)i * dv + j];
  }
  for (int i = 0; i < dk; ++i) {
    const double bkd = gate(beta_k, bk_w, t, i) * gate(key_scale, d_w, t, i);
    w[i] = bkd * kt[i];
  }
  for (int j = 0; j < dv; ++j) u[j] = vt[j] * gate(beta_v, bv_w, t, j);
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) u[j] -= S_bar[(int64_t)i * dv + j] * kt[i];
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) S_t[(int64_t)i * dv + j] = S_bar[(int64_t)i * dv + j] + w[i] * u[j];
}

static void gate_grad(double* dg, int width, int t, int i, double x) {
  if (!dg || width == 0) return;
  if (width == 1)
    dg[t] += x;
  else
    dg[(int64_t)t * width + i] += x;
}

int dn_oracle_bwd_head(int T, int dk, int dv, const double* q, const double* k, const double* v,
                       const double* alpha, int alpha_w, const double* beta_k, int bk_w,
                       const double* beta_v, int bv_w, const double* key_scale, int d_w,
                       const double* S0, const double* dO, const double* dS_T, int pre_read,
                       double* dq, double* dkey, double* dval, double* dalpha, double* dbeta_k,
                       double* dbeta_v, double* dkey_scale, double* dS0) {
  if (T < 0 || dk <= 0 || dv <= 0 || !dS0) return -1;
  if (!(alpha_w == 0 || alpha_w == 1 || alpha_w == dk)) return -1;
  if (!(bk_w == 0 || bk_w == 1 || bk_w == dk)) return -1;
  if (!(bv_w == 0 || bv_w == 1 || bv_w == dv)) return -1;
  if (!(d_w == 0 || d_w == 1 || d_w == dk)) return -1;
  const int ck = 64;
  const int nblk = (T + ck - 1) / ck;
  const size_t m = (size_t)dk * dv;
  double* cks = (double*)malloc(sizeof(double) * m * (size_t)(nblk > 0 ? nblk : 1));
  double* states = (double*)malloc(sizeof(double) * m * (size_t)(ck + 1));
  double* S_bar = (double*)malloc(sizeof(double) * m);
  double* S_t = (double*)malloc(sizeof(double) * m);
  double* dS = (double*)malloc(sizeof(double) * m);
  double* w = (double*)malloc(sizeof(double) * (size_t)dk);
  double* u = (double*)malloc(sizeof(double) * (size_t)dv);
  double* dw = (double*)malloc(sizeof(double) * (size_t)dk);
  double* du = (double*)malloc(sizeof(double) * (size_t)dv);
  int rc = 0;
  if (!cks || !states || !S_bar || !S_t || !dS || !w || !u || !dw || !du) {
    rc = -1;
    goto done;
  }
  if (dalpha && alpha_w) memset(dalpha, 0, sizeof(double) * (size_t)T * alpha_w);
  if (dbeta_k && bk_w) memset(dbeta_k, 0, sizeof(double) * (size_t)T * bk_w);
  if (dbeta_v && bv_w) memset(dbeta_v, 0, sizeof(double) * (size_t)T * bv_w);
  if (dkey_scale && d_w) memset(dkey_scale, 0, sizeof(double) * (size_t)T * d_w);

  /* forward: the state entering every block of ck tokens */
  for (size_t e = 0; e < m; ++e) S_t[e] = S0 ? S0[e] : 0.0;
  for (int blk = 0; blk < nblk; ++blk) {
    memcpy(cks + (size_t)blk * m, S_t, sizeof(double) * m);
    const int t1 = (blk + 1) * ck < T ? (blk + 1) * ck : T;
    for (int t = blk * ck; t < t1; ++t) {
      memcpy(states, S_t, sizeof(double) * m);
      fwd_token(dk, dv, q + (int64_t)t * dk, k + (int64_t)t * dk, v + (int64_t)t * dv, alpha, alpha_w,
                beta_k, bk_w, beta_v, bv_w, key_scale, d_w, t, states, S_bar, w, u, S_t);
    }
  }

  /* reverse */
  for (size_t e = 0; e < m; ++e) dS[e] = dS_T ? dS_T[e] : 0.0;
  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * ck, t1 = (blk + 1) * ck < T ? (blk + 1) * ck : T;
    /* states[s] = S_{t0 + s - 1}, the state before token t0 + s */
    memcpy(states, cks + (size_t)blk * m, sizeof(double) * m);
    for (int t = t0; t < t1 - 1; ++t)
      fwd_token(dk, dv, q + (int64_t)t * dk, k + (int64_t)t * dk, v + (int64_t)t * dv, alpha, alpha_w,
                beta_k, bk_w, beta_v, bv_w, key_scale, d_w, t, states + (size_t)(t - t0) * m, S_bar, w, u,
                states + (size_t)(t - t0 + 1) * m);
    for (int t = t1 - 1; t >= t0; --t) {
      const double* qt = q + (int64_t)t * dk;
      const double* kt = k + (int64_t)t * dk;
      const double* vt = v + (int64_t)t * dv;
      const double* dOt = dO + (int64_t)t * dv;
      const double* S_prev = states + (size_t)(t - t0) * m;
      fwd_token(dk, dv, qt, kt, vt, alpha, alpha_w, beta_k, bk_w, beta_v, bv_w, key_scale, d_w, t, S_prev,
                S_bar, w, u, S_t);
      double* dqt = dq + (int64_t)t * dk;
      double* dkt = dkey + (int64_t)t * dk;
      double* dvt = dval + (int64_t)t * dv;
      const double* S_read = pre_read ? S_prev : S_t;
      /* dq = S_read dO */
      for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += S_read[(int64_t)i * dv + j] * dOt[j];
        dqt[i] = acc;
      }
      if (!pre_read)
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) dS[(int64_t)i * dv + j] += qt[i] * dOt[j];
      /* dw = dS u, du = dS^T w */
      for (int i = 0; i < dk; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += dS[(int64_t)i * dv + j] * u[j];
        dw[i] = acc;
      }
      for (int j = 0; j < dv; ++j) du[j] = 0.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) du[j] += dS[(int64_t)i * dv + j] * w[i];
      /* dk = (beta^k d) dw - S_bar du; gate gradients of the write key */
      for (int i = 0; i < dk; ++i) {
        const double bk = gate(beta_k, bk_w, t, i), dd = gate(key_scale, d_w, t, i);
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) acc += S_bar[(int64_t)i * dv + j] * du[j];
        dkt[i] = bk * dd * dw[i] - acc;
        gate_grad(dbeta_k, bk_w, t, i, dd * kt[i] * dw[i]);
        gate_grad(dkey_scale, d_w, t, i, bk * kt[i] * dw[i]);
      }
      /* dv = beta^v du, dbeta^v = v du */
      for (int j = 0; j < dv; ++j) {
        dvt[j] = gate(beta_v, bv_w, t, j) * du[j];
        gate_grad(dbeta_v, bv_w, t, j, vt[j] * du[j]);
      }
      /* dS_bar = dS - k du^T; dalpha_i = <row i of dS_bar, row i of S_prev>; dS_prev = Diag(alpha) dS_bar */
      for (int i = 0; i < dk; ++i) {
        const double decay = gate(alpha, alpha_w, t, i);
        double da = 0.0;
        for (int j = 0; j < dv; ++j) {
          const double dsb = dS[(int64_t)i * dv + j] - kt[i] * du[j];
          da += dsb * S_prev[(int64_t)i * dv + j];
          dS[(int64_t)i * dv + j] = decay * dsb;
        }
        gate_grad(dalpha, alpha_w, t, i, da);
      }
      if (pre_read)
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) dS[(int64_t)i * dv + j] += qt[i] * dOt[j];
    }
  }
  memcpy(dS0, dS, sizeof(double) * m);
done:
  free(cks);
  free(states);
  free(S_bar);
  free(S_t);
  free(dS);
  free(w);
  free(u);
  free(dw);
  free(du);
  return rc;
}

/* NH heads of the reverse pass, each laid out contiguously like dn_oracle_heads. */
int dn_oracle_bwd_heads(int NH, int T, int dk, int dv, const double* q, const double* k, const double* v,
                        const double* alpha, int alpha_w, const double* beta_k, int bk_w, const double* beta_v,
                        int bv_w, const double* key_scale, int d_w, const double* S0, const double* dO,
                        const double* dS_T, int pre_read, double* dq, double* dkey, double* dval, double* dalpha,
                        double* dbeta_k, double* dbeta_v, double* dkey_scale, double* dS0, int nthreads) {
  if (NH < 0) return -1;
  int bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int h = 0; h < NH; ++h) {
    const int64_t tk = (int64_t)h * T * dk, tv = (int64_t)h * T * dv, sm = (int64_t)h * dk * dv;
#define DN_G(p, w) ((p) ? (p) + (int64_t)h * T * (w) : NULL)
    int rc = dn_oracle_bwd_head(T, dk, dv, q + tk, k + tk, v + tv, DN_G(alpha, alpha_w), alpha_w,
                                DN_G(beta_k, bk_w), bk_w, DN_G(beta_v, bv_w), bv_w, DN_G(key_scale, d_w), d_w,
                                S0 ? S0 + sm : NULL, dO + tv, dS_T ? dS_T + sm : NULL, pre_read, dq + tk,
                                dkey + tk, dval + tv, DN_G(dalpha, alpha_w), DN_G(dbeta_k, bk_w),
                                DN_G(dbeta_v, bv_w), DN_G(dkey_scale, d_w), dS0 + sm);
#undef DN_G
    bad |= (rc != 0);
  }
  return bad ? -1 : 0;
}

/* Number of threads an OpenMP parallel region would use (for reporting). */
int dn_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
