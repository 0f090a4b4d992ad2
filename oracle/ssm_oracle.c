/*
 * ssm_oracle.c -- float64 CPU oracle for the Mamba-1 selective scan (S6) with a causal depthwise
 * conv1d + SiLU in front of it and a SiLU(z) output gate behind it, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY. This file exists so that the tests, the smoke check and the
 * benchmark's CPU-baseline leg can compare the CUDA kernels against a plain, sequential,
 * obviously correct restatement of the method. The product path never links or calls it, and
 * it shares no code, header, table or constant with the CUDA library.
 *
 * Every quantity is a double. Inputs are whatever the caller passes (the tests pass the exact
 * values the GPU sees, e.g. bf16-rounded numbers promoted to double). Loops run in the order the
 * definitions are written: batch -> channel -> time -> state. The only parallelism is over
 * independent channels (forward) or batch elements (backward); it never changes an arithmetic
 * order.
 *
 * Sources restated here (page title, then section):
 *  [SSMK]  "Sequence and state-space models" (docs.algenta.ai), section `state_space_models`:
 *          ssm_discretize_zoh, ssm_discretize_b, ssm_recurrence_step, ssm_output_step,
 *          mamba_delta_softplus.
 *  [SSM]   "state-space models" (aarnphm.xyz): "From continuous time to tokens" (zero-order hold),
 *          "One recurrence, one convolution" (h_{-1} = 0), "Mamba" (selective Delta_t, B_t, C_t;
 *          fixed diagonal A).
 *  [GLOSS] "State-Space Models & Long-Context Sequence Architectures (Mamba)" (chipfoundryservices
 *          glossary): "Mathematical Formulation" (h' = Ah + Bx, y = Ch + Dx; ZOH A-bar, B-bar),
 *          "Lab 2" (the stable softplus form).
 *  [TL]    "Selective Mamba", TorchLean Runtime.Autograd.Model.Mamba: Parameters (convKernel rows
 *          newest-first, convBias before the content SiLU, logA with A = -exp(logA), dSkip on the
 *          activated feature, zProj gate), State (zero-padded history), zeroState, step.
 *  [RT]    rustytorch commit log, "Real S6 forward" (conv -> SiLU -> softplus delta -> scan ->
 *          D skip -> SiLU(z) gate) and "Hand-written VJP" (reverse-time recurrence over the cached
 *          h trajectory; dA_log = dA * A).
 *
 * Readings taken where the pages leave a step open:
 *  - B-bar is the exact zero-order hold (A-bar - 1)/A * B ([SSMK] ssm_discretize_b, [SSM], [GLOSS]),
 *    not the first-order Delta*B. A = -exp(A_log) is never 0, so the a == 0 fallback is unreachable.
 *  - (A-bar - 1) is evaluated as expm1(Delta*A) so that small Delta*A does not cancel.
 *  - softplus has no large-argument cut-off; the pages give none.
 *  - Delta = dt + dt_bias, then softplus when delta_softplus != 0 (dt_bias may be absent = 0).
 *  - Without a conv (conv_w == NULL) the input x is u itself.
 *  - State carry ([TL] State, step, runArray): h0 is the state after the previous chunk (NULL =
 *    zeroState), conv_hist holds the previous chunk's last K-1 pre-conv inputs newest-first
 *    (history[0] is the most recent token; NULL = zero padding). The page keeps up to K entries
 *    after a step, but a step only ever reads the K-1 newest of them together with the new token,
 *    so K-1 entries carry everything the next chunk needs. h_last / conv_hist_out are the same
 *    objects after this chunk; an empty chunk (L = 0) returns them unchanged.
 *  - euler = 1 selects Mamba's first-order input discretisation B-bar = Delta * B
 *    ([SSMK] mamba_selective_scan_step; [TL] step); A-bar stays exp(Delta * A).
 *
 * Also here: the Mamba-2 state-space-duality recurrence ([SSM] "Mamba-2 and state-space
 * duality"), ssm_oracle_ssd_fwd at the end of the file, with its own readings listed there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- scalar pieces ---------------------------------------------------------------------- */

/* softplus(v) = log(1 + e^v) in the overflow-free form log1p(e^{-|v|}) + max(v, 0)
 * ([SSMK] mamba_delta_softplus; [GLOSS] Lab 2 softplus). */
double ssm_oracle_softplus(double v) { return log1p(exp(-fabs(v))) + (v > 0.0 ? v : 0.0); }

/* logistic sigmoid, written so that neither branch overflows. */
double ssm_oracle_sigmoid(double v) {
  if (v >= 0.0) return 1.0 / (1.0 + exp(-v));
  double e = exp(v);
  return e / (1.0 + e);
}

/* SiLU(v) = v * sigmoid(v) ([TL] content SiLU and the zProj gate; [RT] "conv1d -> SiLU"). */
double ssm_oracle_silu(double v) { return v * ssm_oracle_sigmoid(v); }

/* Exact zero-order hold of one diagonal entry: A-bar = exp(Delta*A), B-bar = (A-bar - 1)/A * B
 * ([SSMK] ssm_discretize_zoh / ssm_discretize_b; [SSM] "From continuous time to tokens";
 * [GLOSS] "Mathematical Formulation"). The a == 0 case falls back to Delta*B as [SSMK] states. */
void ssm_oracle_zoh(double A, double B, double delta, double *Abar, double *Bbar) {
  *Abar = exp(delta * A);
  *Bbar = (A == 0.0) ? delta * B : expm1(delta * A) / A * B;
}

/* ---- causal depthwise conv1d + SiLU ------------------------------------------------------- */

/* One channel: c_t = b + sum_{k<K} w[k] * x[t-k] with x[t<0] = 0 (tap 0 multiplies the current
 * token; history newest-first and zero-padded), u_t = SiLU(c_t). [TL] convKernel / convBias /
 * State.history; [RT] "causal depthwise conv1d -> SiLU". Writes c (may be NULL) and u. */
static void conv_silu_channel(const double *x, const double *w, double b, int64_t L, int64_t K,
                              const double *hist, double *c, double *u) {
  for (int64_t t = 0; t < L; t++) {
    double acc = b;
    for (int64_t k = 0; k < K; k++) {
      if (t - k >= 0)
        acc += w[k] * x[t - k];
      else if (hist)
        acc += w[k] * hist[k - t - 1]; /* x_{t-k} with t-k < 0 is history[k-t-1] */
    }
    if (c) c[t] = acc;
    u[t] = ssm_oracle_silu(acc);
  }
}

/* The K-1 newest pre-conv inputs after this chunk, newest-first, continuing the input history. */
static void conv_hist_after(const double *x, const double *hist, int64_t L, int64_t K, double *out) {
  for (int64_t j = 0; j < K - 1; j++) {
    const int64_t t = L - 1 - j;
    out[j] = (t >= 0) ? x[t] : (hist ? hist[j - L] : 0.0);
  }
}

/* x, u: (Bt, Dn, L); w: [Dn, K] newest-first; b: [Dn] or NULL (zero). */
void ssm_oracle_conv1d_silu(const double *x, const double *w, const double *b, int64_t Bt,
                            int64_t Dn, int64_t L, int64_t K, double *u) {
  for (int64_t bi = 0; bi < Bt; bi++)
    for (int64_t d = 0; d < Dn; d++) {
      const int64_t off = (bi * Dn + d) * L;
      conv_silu_channel(x + off, w + d * K, b ? b[d] : 0.0, L, K, NULL, NULL, u + off);
    }
}

/* ---- forward ------------------------------------------------------------------------------ */

/* Forward of one channel (batch element bi, channel d). Layouts: x, dt, z, out: (Bt, Dn, L);
 * B, C: (Bt, N, L); A_log: [Dn, N]; D, dt_bias, conv_b: [Dn]; conv_w: [Dn, K]. */
static void fwd_channel(const double *x, const double *dt, const double *dt_bias,
                        const double *A_log, const double *B, const double *C, const double *D,
                        const double *z, const double *conv_w, const double *conv_b, int64_t Dn,
                        int64_t N, int64_t L, int64_t K, int delta_softplus, int euler,
                        const double *h0, const double *conv_hist, int64_t bi, int64_t d,
                        double *out, double *u_out, double *y_out, double *h_last,
                        double *conv_hist_out, double *h, double *u) {
  const int64_t off = (bi * Dn + d) * L;
  const double *Bb = B + bi * N * L, *Cb = C + bi * N * L;
  const int64_t ch = bi * Dn + d;
  const double *hist = (conv_hist && K > 1) ? conv_hist + ch * (K - 1) : NULL;

  /* u: conv + SiLU, or x itself when there is no conv. */
  if (conv_w)
    conv_silu_channel(x + off, conv_w + d * K, conv_b ? conv_b[d] : 0.0, L, K, hist, NULL, u);
  else
    for (int64_t t = 0; t < L; t++) u[t] = x[off + t];

  /* h_{-1} = 0 ([SSM]; [TL] zeroState), or the carried state */
  for (int64_t n = 0; n < N; n++) h[n] = h0 ? h0[ch * N + n] : 0.0;
  for (int64_t t = 0; t < L; t++) {
    const double v = dt[off + t] + (dt_bias ? dt_bias[d] : 0.0);
    const double delta = delta_softplus ? ssm_oracle_softplus(v) : v;
    double y = 0.0;
    for (int64_t n = 0; n < N; n++) {
      const double A = -exp(A_log[d * N + n]); /* [TL] logA; [RT] A = -exp(A_log) */
      double Abar, Bbar;
      ssm_oracle_zoh(A, Bb[n * L + t], delta, &Abar, &Bbar);
      if (euler) Bbar = delta * Bb[n * L + t]; /* [SSMK] mamba_selective_scan_step */
      h[n] = Abar * h[n] + Bbar * u[t]; /* [SSMK] ssm_recurrence_step */
      y += Cb[n * L + t] * h[n];        /* [SSMK] ssm_output_step */
    }
    y += (D ? D[d] : 0.0) * u[t]; /* [TL] dSkip on the activated feature; [GLOSS] D x */
    if (y_out) y_out[off + t] = y;
    if (u_out) u_out[off + t] = u[t];
    out[off + t] = z ? y * ssm_oracle_silu(z[off + t]) : y; /* [TL] zProj gate; [RT] SiLU(z) */
  }
  if (h_last)
    for (int64_t n = 0; n < N; n++) h_last[ch * N + n] = h[n];
  if (conv_hist_out && K > 1) conv_hist_after(x + off, hist, L, K, conv_hist_out + ch * (K - 1));
}

/* Whole forward. Nullable: dt_bias, D, z, conv_w (then x is u), conv_b, h0 ((Bt, Dn, N) carried
 * state), conv_hist ((Bt, Dn, K-1) carried inputs, newest-first), u_out, y_out (pre-gate output
 * including D*u), h_last ((Bt, Dn, N) state after the chunk), conv_hist_out ((Bt, Dn, K-1)).
 * n_threads <= 0 means "all". Returns 0, or -1 on allocation failure. */
int ssm_oracle_fwd(const double *x, const double *dt, const double *dt_bias, const double *A_log,
                   const double *B, const double *C, const double *D, const double *z,
                   const double *conv_w, const double *conv_b, int64_t Bt, int64_t Dn, int64_t N,
                   int64_t L, int64_t K, int delta_softplus, int euler, const double *h0,
                   const double *conv_hist, double *out, double *u_out, double *y_out,
                   double *h_last, double *conv_hist_out, int n_threads) {
  int failed = 0;
  const int64_t channels = Bt * Dn;
#ifdef _OPENMP
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel num_threads(n_threads) reduction(| : failed)
#endif
  {
    double *h = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    double *u = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    if (!h || !u) failed = 1;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int64_t ch = 0; ch < channels; ch++)
      if (h && u)
        fwd_channel(x, dt, dt_bias, A_log, B, C, D, z, conv_w, conv_b, Dn, N, L, K,
                    delta_softplus, euler, h0, conv_hist, ch / Dn, ch % Dn, out, u_out, y_out,
                    h_last, conv_hist_out, h, u);
    free(h);
    free(u);
  }
  (void)n_threads;
  return failed ? -1 : 0;
}

/* ---- backward ----------------------------------------------------------------------------- */

/*
 * Vector-Jacobian product of ssm_oracle_fwd ([RT] "Hand-written VJP": a reverse-time recurrence
 * over the cached h trajectory). With x_t = Delta_t * A, a = A-bar, bb = B-bar, lambda_t = dL/dh_t:
 *
 *   dy_t       = dout_t * SiLU(z_t)                      (dy_t = dout_t without a gate)
 *   dz_t       = dout_t * y_t * s(z_t)(1 + z_t(1 - s(z_t)))      s = sigmoid
 *   lambda_t   = dy_t * C_t + a_{t+1} * lambda_{t+1},    lambda_L = 0
 *   dC_t[n]   += dy_t * h_t[n]                           (summed over channels d)
 *   dB_t[n]   += lambda_t[n] * u_t * (a - 1)/A           (summed over channels d)
 *   dDelta_t   = sum_n lambda_t[n] * a * (A * h_{t-1}[n] + B_t[n] * u_t)
 *   dA_n      += lambda_t[n] * (h_{t-1}[n] * Delta_t * a + u_t * B_t[n] * (x a - (a - 1)) / A^2)
 *   dA_log     = dA * A                                  ([RT] VJP commit)
 *   du_t       = D * dy_t + sum_n lambda_t[n] * bb_t[n];  dD += dy_t * u_t
 *   dv_t       = dDelta_t * s(v_t) (softplus) or dDelta_t;  ddt_t = dv_t;  ddt_bias += dv_t
 *   dc_t       = du_t * s(c_t)(1 + c_t(1 - s(c_t)))      (conv pre-activation)
 *   dx_j       = sum_k w[k] * dc_{j+k};  dw[k] = sum_t dc_t x_{t-k};  dconv_b = sum_t dc_t
 *   dh0        = a_0 * lambda_0                          (gradient of the carried state)
 *   dh_last (input) is the gradient arriving at the state after the chunk (from the next chunk's
 *   dh0): it enters as lambda_{L-1} = dy C + dh_last. The carried inputs' output history needs no
 *   such term here: its gradient is the next chunk's dhist added to dx of the last K-1 steps.
 *   dhist_j    = sum_{k > j} w[k] * dc_{k-j-1}           (gradient of the carried inputs x_{-1-j})
 *
 * With euler = 1 (B-bar = Delta * B): bb = Delta B, dB_t[n] += lambda u Delta,
 * dDelta_t = sum_n lambda (A a h_{t-1} + B u), dA_n += lambda Delta a h_{t-1}.
 *
 * Without a conv, dx = du. Every output is overwritten (not accumulated into). Nullable outputs
 * are skipped. Parallel over batch elements only; each batch element runs its channels in order
 * and the per-channel parameter gradients are summed over batch elements afterwards, in order.
 */
int ssm_oracle_bwd(const double *x, const double *dt, const double *dt_bias, const double *A_log,
                   const double *B, const double *C, const double *D, const double *z,
                   const double *conv_w, const double *conv_b, int64_t Bt, int64_t Dn, int64_t N,
                   int64_t L, int64_t K, int delta_softplus, int euler, const double *h0,
                   const double *conv_hist, const double *dout, const double *dh_last, double *dx, double *ddt,
                   double *dA_log, double *dB, double *dC, double *dD, double *ddt_bias,
                   double *dz, double *dconv_w, double *dconv_b, double *dh0, double *dconv_hist,
                   int n_threads) {
  /* per-batch-element partials of the per-channel parameter gradients */
  const size_t nb = (size_t)(Bt > 0 ? Bt : 1);
  double *pA = (double *)calloc(nb * (size_t)(Dn * N), sizeof(double));
  double *pD = (double *)calloc(nb * (size_t)Dn, sizeof(double));
  double *pdtb = (double *)calloc(nb * (size_t)Dn, sizeof(double));
  double *pcw = (double *)calloc(nb * (size_t)(Dn * (K > 0 ? K : 1)), sizeof(double));
  double *pcb = (double *)calloc(nb * (size_t)Dn, sizeof(double));
  int failed = (!pA || !pD || !pdtb || !pcw || !pcb);
  if (failed) goto done;

#ifdef _OPENMP
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for num_threads(n_threads) schedule(dynamic, 1) reduction(| : failed)
#endif
  for (int64_t bi = 0; bi < Bt; bi++) {
    const size_t LN = (size_t)(L * N);
    double *c = (double *)malloc(sizeof(double) * (size_t)L);
    double *u = (double *)malloc(sizeof(double) * (size_t)L);
    double *v = (double *)malloc(sizeof(double) * (size_t)L);
    double *dl = (double *)malloc(sizeof(double) * (size_t)L);
    double *y = (double *)malloc(sizeof(double) * (size_t)L);
    double *dy = (double *)malloc(sizeof(double) * (size_t)L);
    double *dc = (double *)malloc(sizeof(double) * (size_t)L);
    double *a = (double *)malloc(sizeof(double) * LN);
    double *em1 = (double *)malloc(sizeof(double) * LN);
    double *bb = (double *)malloc(sizeof(double) * LN);
    double *h = (double *)malloc(sizeof(double) * LN);
    double *A = (double *)malloc(sizeof(double) * (size_t)N);
    double *lam = (double *)malloc(sizeof(double) * (size_t)N);
    double *dA = (double *)malloc(sizeof(double) * (size_t)N);
    if (!c || !u || !v || !dl || !y || !dy || !dc || !a || !em1 || !bb || !h || !A || !lam || !dA) {
      failed = 1;
    } else {
      const double *Bb = B + bi * N * L, *Cb = C + bi * N * L;
      double *dBb = dB ? dB + bi * N * L : NULL, *dCb = dC ? dC + bi * N * L : NULL;
      if (dBb) memset(dBb, 0, sizeof(double) * LN);
      if (dCb) memset(dCb, 0, sizeof(double) * LN);
      for (int64_t d = 0; d < Dn; d++) {
        const int64_t off = (bi * Dn + d) * L;
        const int64_t chn = bi * Dn + d;
        const double Dd = D ? D[d] : 0.0;
        const double *hist = (conv_hist && K > 1) ? conv_hist + chn * (K - 1) : NULL;
        /* forward recompute with the whole trajectory kept */
        if (conv_w)
          conv_silu_channel(x + off, conv_w + d * K, conv_b ? conv_b[d] : 0.0, L, K, hist, c, u);
        else
          for (int64_t t = 0; t < L; t++) u[t] = x[off + t];
        for (int64_t n = 0; n < N; n++) A[n] = -exp(A_log[d * N + n]);
        for (int64_t t = 0; t < L; t++) {
          v[t] = dt[off + t] + (dt_bias ? dt_bias[d] : 0.0);
          dl[t] = delta_softplus ? ssm_oracle_softplus(v[t]) : v[t];
          double yt = 0.0;
          for (int64_t n = 0; n < N; n++) {
            const size_t i = (size_t)(t * N + n);
            a[i] = exp(dl[t] * A[n]);
            em1[i] = expm1(dl[t] * A[n]);
            bb[i] = euler ? dl[t] * Bb[n * L + t] : em1[i] / A[n] * Bb[n * L + t];
            h[i] = a[i] * (t > 0 ? h[i - (size_t)N] : (h0 ? h0[chn * N + n] : 0.0)) + bb[i] * u[t];
            yt += Cb[n * L + t] * h[i];
          }
          y[t] = yt + Dd * u[t];
        }
        /* output gate */
        for (int64_t t = 0; t < L; t++) {
          if (z) {
            const double zz = z[off + t], s = ssm_oracle_sigmoid(zz);
            dy[t] = dout[off + t] * zz * s;
            if (dz) dz[off + t] = dout[off + t] * y[t] * s * (1.0 + zz * (1.0 - s));
          } else {
            dy[t] = dout[off + t];
          }
        }
        /* reverse-time adjoint recurrence */
        for (int64_t n = 0; n < N; n++) {
          lam[n] = dh_last ? dh_last[chn * N + n] : 0.0;
          dA[n] = 0.0;
        }
        double accD = 0.0, accdtb = 0.0;
        for (int64_t t = L - 1; t >= 0; t--) {
          double du = Dd * dy[t];
          double ddelta = 0.0;
          accD += dy[t] * u[t];
          for (int64_t n = 0; n < N; n++) {
            const size_t i = (size_t)(t * N + n);
            const double anext = (t + 1 < L) ? a[i + (size_t)N] : 1.0; /* lambda_L := dh_last */
            lam[n] = dy[t] * Cb[n * L + t] + anext * lam[n];
            const double hprev = t > 0 ? h[i - (size_t)N] : (h0 ? h0[chn * N + n] : 0.0);
            const double Bt_n = Bb[n * L + t];
            const double xx = dl[t] * A[n];
            if (dCb) dCb[n * L + t] += dy[t] * h[i];
            if (euler) {
              if (dBb) dBb[n * L + t] += lam[n] * u[t] * dl[t];
              ddelta += lam[n] * (A[n] * a[i] * hprev + Bt_n * u[t]);
              dA[n] += lam[n] * dl[t] * a[i] * hprev;
            } else {
              if (dBb) dBb[n * L + t] += lam[n] * u[t] * em1[i] / A[n];
              ddelta += lam[n] * a[i] * (A[n] * hprev + Bt_n * u[t]);
              dA[n] += lam[n] * (hprev * dl[t] * a[i] +
                                 u[t] * Bt_n * (xx * a[i] - em1[i]) / (A[n] * A[n]));
            }
            du += lam[n] * bb[i];
          }
          const double dv = delta_softplus ? ddelta * ssm_oracle_sigmoid(v[t]) : ddelta;
          if (ddt) ddt[off + t] = dv;
          accdtb += dv;
          if (conv_w) {
            const double s = ssm_oracle_sigmoid(c[t]);
            dc[t] = du * s * (1.0 + c[t] * (1.0 - s));
          } else {
            dc[t] = du;
          }
        }
        /* gradient of the carried state: h0 enters only through h_0 = a_0 h0 + ... */
        if (dh0)
          for (int64_t n = 0; n < N; n++) dh0[chn * N + n] = (L > 0) ? a[(size_t)n] * lam[n] : lam[n];
        /* conv backward (or identity) */
        if (conv_w) {
          const double *w = conv_w + d * K;
          if (dconv_hist && K > 1)
            for (int64_t j = 0; j < K - 1; j++) {
              double acc = 0.0; /* x_{-1-j} feeds c_t through tap k = t + 1 + j */
              for (int64_t t = 0; t < L; t++)
                if (t + 1 + j < K) acc += w[t + 1 + j] * dc[t];
              dconv_hist[chn * (K - 1) + j] = acc;
            }
          if (dx)
            for (int64_t j = 0; j < L; j++) {
              double acc = 0.0;
              for (int64_t k = 0; k < K; k++)
                if (j + k < L) acc += w[k] * dc[j + k];
              dx[off + j] = acc;
            }
          double accb = 0.0;
          for (int64_t k = 0; k < K; k++) {
            double acc = 0.0;
            for (int64_t t = 0; t < L; t++) {
              if (t - k >= 0)
                acc += dc[t] * x[off + t - k];
              else if (hist)
                acc += dc[t] * hist[k - t - 1];
            }
            pcw[(size_t)bi * (size_t)(Dn * K) + (size_t)(d * K + k)] = acc;
          }
          for (int64_t t = 0; t < L; t++) accb += dc[t];
          pcb[(size_t)bi * (size_t)Dn + (size_t)d] = accb;
        } else if (dx) {
          for (int64_t t = 0; t < L; t++) dx[off + t] = dc[t];
        }
        for (int64_t n = 0; n < N; n++)
          pA[(size_t)bi * (size_t)(Dn * N) + (size_t)(d * N + n)] = dA[n] * A[n];
        pD[(size_t)bi * (size_t)Dn + (size_t)d] = accD;
        pdtb[(size_t)bi * (size_t)Dn + (size_t)d] = accdtb;
      }
    }
    free(c); free(u); free(v); free(dl); free(y); free(dy); free(dc);
    free(a); free(em1); free(bb); free(h); free(A); free(lam); free(dA);
  }
  if (failed) goto done;

  /* sum the per-batch-element partials over batch elements, in order */
  for (int64_t d = 0; d < Dn; d++) {
    double sD = 0.0, sdtb = 0.0, scb = 0.0;
    for (int64_t bi = 0; bi < Bt; bi++) {
      sD += pD[(size_t)bi * (size_t)Dn + (size_t)d];
      sdtb += pdtb[(size_t)bi * (size_t)Dn + (size_t)d];
      scb += pcb[(size_t)bi * (size_t)Dn + (size_t)d];
    }
    if (dD) dD[d] = sD;
    if (ddt_bias) ddt_bias[d] = sdtb;
    if (dconv_b && conv_w) dconv_b[d] = scb;
    for (int64_t n = 0; n < N; n++) {
      double s = 0.0;
      for (int64_t bi = 0; bi < Bt; bi++) s += pA[(size_t)bi * (size_t)(Dn * N) + (size_t)(d * N + n)];
      if (dA_log) dA_log[d * N + n] = s;
    }
    if (dconv_w && conv_w)
      for (int64_t k = 0; k < K; k++) {
        double s = 0.0;
        for (int64_t bi = 0; bi < Bt; bi++) s += pcw[(size_t)bi * (size_t)(Dn * K) + (size_t)(d * K + k)];
        dconv_w[d * K + k] = s;
      }
  }
done:
  free(pA); free(pD); free(pdtb); free(pcw); free(pcb);
  (void)n_threads;
  return failed ? -1 : 0;
}


/* ---- Mamba-2 state-space duality (SSD) ----------------------------------------------------
 *
 * [SSM] "Mamba-2 and state-space duality": within a head the transition is a scalar multiple of
 * the identity, A-bar_t = a_t I, and unrolling gives y_t = sum_{s<=t} (C_t . B-bar_s)
 * (prod_{k=s+1..t} a_k) x_s, i.e. Y = (L o Q K^T) V with L_ts = prod_{k=s+1..t} a_k (s <= t).
 * This oracle runs the recurrence that unrolls to that sum, one head at a time:
 *   h_t = a_t h_{t-1} + B-bar_t x_t^T     (h is N x P: state index n, head-channel index p)
 *   y_t = h_t^T C_t + D_h x_t
 * Readings taken where the page leaves a step open:
 *  - a_t and B-bar_t come from the same discretisation as the selective scan, with one A per
 *    head: Delta_t = softplus(dt_t + dt_bias[h]) (or dt_t + dt_bias[h] when delta_softplus == 0),
 *    A_h = -exp(A_log[h]), a_t = exp(Delta_t A_h), B-bar_t = beta_t B_t with beta_t =
 *    expm1(Delta_t A_h) / A_h (exact zero-order hold) or Delta_t (euler = 1).
 *  - B_t and C_t (N values) are shared by all heads of a batch element, as the selective scan
 *    shares them across channels; x_t of a head has P values; D_h is one skip weight per head.
 *  - h0 (NULL = 0) is the state before step 0; h_last receives the state after step L-1.
 * Layouts: x, y (Bt, H, L, P); dt (Bt, H, L); B, C (Bt, L, N); A_log, dt_bias, D [H];
 * h0, h_last (Bt, H, N, P). Returns 0, or -1 if the state buffer cannot be allocated.
 */
int ssm_oracle_ssd_fwd(const double *x, const double *dt, const double *dt_bias,
                       const double *A_log, const double *B, const double *C, const double *D,
                       int64_t Bt, int64_t H, int64_t L, int64_t P, int64_t N, int delta_softplus,
                       int euler, const double *h0, double *y, double *h_last, int n_threads) {
  int failed = 0;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
  for (int64_t bh = 0; bh < Bt * H; bh++) {
    const int64_t b = bh / H, hd = bh % H;
    double *st = (double *)malloc(sizeof(double) * (size_t)(N * P));
    if (!st) {
      failed |= 1;
      continue;
    }
    for (int64_t i = 0; i < N * P; i++) st[i] = h0 ? h0[bh * N * P + i] : 0.0;
    const double A = -exp(A_log[hd]);
    const double bias = dt_bias ? dt_bias[hd] : 0.0;
    const double Dh = D ? D[hd] : 0.0;
    for (int64_t t = 0; t < L; t++) {
      const double v = dt[bh * L + t] + bias;
      const double delta = delta_softplus ? ssm_oracle_softplus(v) : v;
      const double a = exp(delta * A);
      const double beta = euler ? delta : expm1(delta * A) / A;
      const double *xt = x + (bh * L + t) * P;
      const double *Bt_ = B + (b * L + t) * N;
      const double *Ct = C + (b * L + t) * N;
      for (int64_t n = 0; n < N; n++)
        for (int64_t p = 0; p < P; p++) st[n * P + p] = a * st[n * P + p] + beta * Bt_[n] * xt[p];
      double *yt = y + (bh * L + t) * P;
      for (int64_t p = 0; p < P; p++) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; n++) acc += Ct[n] * st[n * P + p];
        yt[p] = acc + Dh * xt[p];
      }
    }
    if (h_last)
      for (int64_t i = 0; i < N * P; i++) h_last[bh * N * P + i] = st[i];
    free(st);
  }
  return failed ? -1 : 0;
}
