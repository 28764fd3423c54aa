/*
 * mlstm_oracle.c -- fp64 CPU oracle for the mLSTM forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference arm of bench.py may load this file's library.  The
 * product path (the CUDA library under mlstm_chunkwise_b200/) never calls it
 * and shares no code, header, table or helper with it.
 *
 * What it computes.  "Tiled Flash Linear Attention: More Efficient Linear RNN
 * and xLSTM Kernels" (abstract) applies its kernels to the xLSTM with matrix
 * memory, the mLSTM; "xLSTM: the NX-AI repository behind the extended LSTM
 * architecture" (section "Exponential gating, matrix memory, and why the
 * kernels decide everything") names its ingredients: exponential gating with
 * normalisation and stabilisation, and a matrix-valued memory updated by a
 * matrix operation.  The pages print no formula, so this file follows the
 * recurrence stated in the benchmark spec, token by token, for each
 * (batch, head), in fp64:
 *
 *   lf_t = logsigmoid(f~_t)                 (forget gate, log domain)
 *   li_t = i~_t             (exp mode)      (input gate, log domain)
 *        = logsigmoid(i~_t) (sigmoid mode)
 *   m_t  = max(lf_t + m_{t-1}, li_t)        (max-state stabiliser)
 *   C_t  = e^{lf_t + m_{t-1} - m_t} C_{t-1} + e^{li_t - m_t} (s k_t) v_t^T
 *   n_t  = e^{lf_t + m_{t-1} - m_t} n_{t-1} + e^{li_t - m_t} (s k_t)
 *   h_t  = C_t^T q_t / max(|n_t^T q_t|, e^{-m_t}),      s = 1/sqrt(d_qk)
 *
 * C is stored as [d_qk, d_v] (the transpose of v k^T), so h = C^T q.
 * With no initial state, C_0 = 0, n_0 = 0 and m_0 = 0.  Initial states are
 * given in the frame m_0.
 *
 * There is no blocking, chunking or reordering: the sums run in token order.
 * Parallelism (OpenMP) is over independent (batch, head) pairs only.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_GATE_EXP 0
#define ORACLE_GATE_SIGMOID 1

/* log(sigmoid(x)) = -log(1 + e^{-x}), written so that neither branch
 * overflows. */
static double oracle_logsigmoid(double x) {
  if (x >= 0.0) return -log1p(exp(-x));
  return x - log1p(exp(x));
}

/*
 * Runs the recurrence above for every (b, h).
 *
 * Inputs (row-major, fp64):
 *   Q, K  [B, NH, T, DK]     V [B, NH, T, DV]
 *   i_pre, f_pre [B, NH, T]  (gate pre-activations)
 *   C0 [B, NH, DK, DV], n0 [B, NH, DK], m0 [B, NH]: all NULL (zero state) or
 *   all given.
 * Outputs (any may be NULL except H):
 *   H [B, NH, T, DV]
 *   C_T, n_T, m_T: final state, same layouts as C0, n0, m0
 *   den_out [B, NH, T]: the denominator max(|n_t^T q_t|, e^{-m_t})
 *   m_out   [B, NH, T]: the stabiliser m_t
 *   snap_every > 0 with C_snap [B, NH, T/snap_every, DK, DV],
 *   n_snap [..., DK], m_snap [...]: the state entering token j*snap_every,
 *   i.e. after j*snap_every tokens (j = 0 gives the initial state).
 * Returns 0, or -1 on a bad argument.
 */
int mlstm_oracle_recurrent(const double* Q, const double* K, const double* V,
                           const double* i_pre, const double* f_pre,
                           const double* C0, const double* n0, const double* m0,
                           int B, int NH, int T, int DK, int DV, int gate_mode,
                           double* H, double* C_T, double* n_T, double* m_T,
                           double* den_out, double* m_out, int snap_every,
                           double* C_snap, double* n_snap, double* m_snap) {
  if (B <= 0 || NH <= 0 || T < 0 || DK <= 0 || DV <= 0) return -1;
  if (!Q || !K || !V || !i_pre || !f_pre || !H) return -1;
  if (!((C0 && n0 && m0) || (!C0 && !n0 && !m0))) return -1;
  if (gate_mode != ORACLE_GATE_EXP && gate_mode != ORACLE_GATE_SIGMOID) return -1;
  if (snap_every > 0 && (T % snap_every != 0 || !C_snap || !n_snap || !m_snap)) return -1;

  const double s = 1.0 / sqrt((double)DK);
  const long BH = (long)B * NH;
  int bad = 0;

#pragma omp parallel for schedule(dynamic, 1)
  for (long bh = 0; bh < BH; ++bh) {
    double* C = (double*)malloc(sizeof(double) * (size_t)DK * DV);
    double* n = (double*)malloc(sizeof(double) * (size_t)DK);
    double* ks = (double*)malloc(sizeof(double) * (size_t)DK);
    double* num = (double*)malloc(sizeof(double) * (size_t)DV);
    if (!C || !n || !ks || !num) {
      free(C); free(n); free(ks); free(num);
#pragma omp atomic write
      bad = 1;
      continue;
    }
    double m;
    if (C0) {
      memcpy(C, C0 + bh * DK * DV, sizeof(double) * (size_t)DK * DV);
      memcpy(n, n0 + bh * DK, sizeof(double) * (size_t)DK);
      m = m0[bh];
    } else {
      memset(C, 0, sizeof(double) * (size_t)DK * DV);
      memset(n, 0, sizeof(double) * (size_t)DK);
      m = 0.0;
    }
    const double* q_bh = Q + bh * (long)T * DK;
    const double* k_bh = K + bh * (long)T * DK;
    const double* v_bh = V + bh * (long)T * DV;
    for (int t = 0; t < T; ++t) {
      if (snap_every > 0 && t % snap_every == 0) {
        long j = bh * (T / snap_every) + t / snap_every;
        memcpy(C_snap + j * DK * DV, C, sizeof(double) * (size_t)DK * DV);
        memcpy(n_snap + j * DK, n, sizeof(double) * (size_t)DK);
        m_snap[j] = m;
      }
      const double* q = q_bh + (long)t * DK;
      const double* k = k_bh + (long)t * DK;
      const double* v = v_bh + (long)t * DV;
      const double lf = oracle_logsigmoid(f_pre[bh * T + t]);
      const double li = (gate_mode == ORACLE_GATE_EXP) ? i_pre[bh * T + t]
                                                       : oracle_logsigmoid(i_pre[bh * T + t]);
      const double m_new = fmax(lf + m, li);
      const double fa = exp(lf + m - m_new);
      const double ia = exp(li - m_new);
      /* memory update: C <- fa C + ia (s k) v^T, n <- fa n + ia (s k) */
      for (int a = 0; a < DK; ++a) {
        ks[a] = s * k[a];
        n[a] = fa * n[a] + ia * ks[a];
        double* Ca = C + (long)a * DV;
        for (int j = 0; j < DV; ++j) Ca[j] = fa * Ca[j] + ia * ks[a] * v[j];
      }
      /* readout: h = C^T q / max(|n^T q|, e^{-m}) */
      double den = 0.0;
      for (int j = 0; j < DV; ++j) num[j] = 0.0;
      for (int a = 0; a < DK; ++a) {
        den += n[a] * q[a];
        const double* Ca = C + (long)a * DV;
        for (int j = 0; j < DV; ++j) num[j] += Ca[j] * q[a];
      }
      const double denom = fmax(fabs(den), exp(-m_new));
      double* h = H + (bh * (long)T + t) * DV;
      for (int j = 0; j < DV; ++j) h[j] = num[j] / denom;
      if (den_out) den_out[bh * T + t] = denom;
      if (m_out) m_out[bh * T + t] = m_new;
      m = m_new;
    }
    if (C_T) memcpy(C_T + bh * DK * DV, C, sizeof(double) * (size_t)DK * DV);
    if (n_T) memcpy(n_T + bh * DK, n, sizeof(double) * (size_t)DK);
    if (m_T) m_T[bh] = m;
    free(C); free(n); free(ks); free(num);
  }
  return bad ? -1 : 0;
}

/*
 * The sigmoid-input-gate variant with reduced computation.  "Tiled Flash
 * Linear Attention: More Efficient Linear RNN and xLSTM Kernels" (abstract)
 * introduces an mLSTM variant with a sigmoid input gate that needs less
 * computation; the page does not define it further.  Reading: with both gates
 * sigmoids every gate value lies in (0, 1), the memory cannot grow without
 * bound, and the variant drops the max-state stabiliser and the normaliser:
 *
 *   C_t = sigmoid(f~_t) C_{t-1} + sigmoid(i~_t) (s k_t) v_t^T
 *   h_t = C_t^T q_t                           (no normaliser, no division)
 *
 * This is that definition written out, token by token, in fp64, with no
 * stabiliser.  n_t = sigmoid(f~_t) n_{t-1} + sigmoid(i~_t) (s k_t) is carried
 * only so that the final state can be compared with the other modes' (it
 * does not enter h).  The initial state (C0, n0) is given in the frame m0, as
 * in the other modes: the recurrence starts from e^{m0} C0 and e^{m0} n0.
 * The final state is returned unstabilised (the frame m = 0).
 *
 * Inputs as mlstm_oracle_recurrent; outputs H [B, NH, T, DV] and, where not
 * NULL, C_T [B, NH, DK, DV] and n_T [B, NH, DK].
 */
static double oracle_sigmoid(double x) {
  if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
  const double e = exp(x);
  return e / (1.0 + e);
}

int mlstm_oracle_sigmoid_plain(const double* Q, const double* K, const double* V,
                               const double* i_pre, const double* f_pre, const double* C0,
                               const double* n0, const double* m0, int B, int NH, int T, int DK,
                               int DV, double* H, double* C_T, double* n_T) {
  if (B < 1 || NH < 1 || T < 0 || DK < 1 || DV < 1 || !H) return -1;
  if (!((C0 && n0 && m0) || (!C0 && !n0 && !m0))) return -1;
  const double s = 1.0 / sqrt((double)DK);
  const long BH = (long)B * NH;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (long bh = 0; bh < BH; ++bh) {
    double* C = (double*)calloc((size_t)DK * DV, sizeof(double));
    double* n = (double*)calloc((size_t)DK, sizeof(double));
    if (!C || !n) {
      bad = 1;
      free(C); free(n);
      continue;
    }
    if (C0) {
      const double sc = exp(m0[bh]);
      for (long a = 0; a < (long)DK * DV; ++a) C[a] = sc * C0[bh * DK * DV + a];
      for (int a = 0; a < DK; ++a) n[a] = sc * n0[bh * DK + a];
    }
    for (int t = 0; t < T; ++t) {
      const double f = oracle_sigmoid(f_pre[bh * T + t]);
      const double ig = oracle_sigmoid(i_pre[bh * T + t]);
      const double* k = K + ((long)bh * T + t) * DK;
      const double* v = V + ((long)bh * T + t) * DV;
      const double* q = Q + ((long)bh * T + t) * DK;
      for (int a = 0; a < DK; ++a) {
        const double wk = ig * s * k[a];
        for (int j = 0; j < DV; ++j) C[a * DV + j] = f * C[a * DV + j] + wk * v[j];
        n[a] = f * n[a] + wk;
      }
      double* h = H + ((long)bh * T + t) * DV;
      for (int j = 0; j < DV; ++j) h[j] = 0.0;
      for (int a = 0; a < DK; ++a)
        for (int j = 0; j < DV; ++j) h[j] += C[a * DV + j] * q[a];
    }
    if (C_T) memcpy(C_T + bh * DK * DV, C, sizeof(double) * (size_t)DK * DV);
    if (n_T) memcpy(n_T + bh * DK, n, sizeof(double) * (size_t)DK);
    free(C); free(n);
  }
  return bad ? -1 : 0;
}

/* Number of OpenMP threads a parallel region of this library uses. */
int mlstm_oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
