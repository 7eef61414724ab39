/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the Gated DeltaNet hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * Every result is computed token by token, exactly in the order the pages state
 * the method, in double precision.  Inputs may be given as float32 (the values a
 * bf16/fp32 GPU run sees, exact in float32) or as float64 (the pins use exact
 * fp64 fixtures).
 *
 * Sources (page title, section / equation):
 *  - "Qwen3.5" (rainlin-net), section "GDN详解": the five-step recurrence
 *       S' = alpha*S ; kv = S'^T k ; delta = beta*(v - kv) ; S = S' + k delta^T ;
 *       o = S^T q
 *    and the module skeleton's gate lines beta = sigmoid(b),
 *       g = -exp(A_log) * softplus(a + dt_bias), computed in fp32 there.
 *  - "从 Full Attention 到 Gated DeltaNet" (dingfen), section 9: alpha = e^g,
 *    softplus(x) = log(1 + e^x); section 10: x -> CausalConv1D -> SiLU -> q,k,v.
 *  - "gated-deltanet-qwen3.5" (wanger-sjtu), architecture diagram: decode reads
 *    and updates conv_states and recurrent_states.
 *  - "Gated DeltaNet-2" (zhichai), section "新更新公式": S_bar = D S,
 *    r = S_bar^T e, S = S_bar + k (z - r)^T with e = b (.) k, z = w (.) v;
 *    section "标量绑定的数学表达": the KDA update (I - beta k k^T) D S + beta k v^T;
 *    section "Gate-aware 反向传播": gradients with the channel gates inside the
 *    accumulations.
 *  - "gated-deltanet-qwen3.5" (wanger-sjtu), section "输出门控与 RMSNorm":
 *    RMSNormGated(core_attn_out, z).
 *
 * Readings where the pages are silent (this file's choices, stated here):
 *  - L2 normalisation of q and k is x / sqrt(sum x^2 + 1e-6); q is then scaled
 *    by `scale` (1/sqrt(d_k) by default).
 *  - Grouped heads: value head hv reads key/query head hv / (Hv/Hk).
 *  - Storage of the state is [d_k][d_v] (key index first), o = S^T q.
 *  - softplus is evaluated exactly as log1p(exp(x)), rewritten for x > 0 as
 *    x + log1p(exp(-x)) (the same number, no overflow).
 *  - Decode conv: torch-style causal cross-correlation over the window
 *    [cs0, cs1, cs2, x] with weight taps w[c][0..3]; cs2 is the newest cached
 *    input; SiLU(y) = y * sigmoid(y); no bias.
 *  - Gated RMSNorm of the output ("gated-deltanet-qwen3.5" section 输出门控与
 *    RMSNorm: RMSNormGated(core_attn_out, z), an RMSNorm and then the output
 *    gate, SwiGLU-like): per token and value head, over the d_v channels,
 *    y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z).
 *
 * Parity: pinned (see tests/test_oracle_pins.py): linear-attention brute force,
 * delta-rule overwrite on orthonormal keys, per-step overwrite identity, pure
 * decay closed form, matrix-form recurrence, GDN-2 -> GDN reduction, KDA ->
 * GDN-2 (tied gates) and -> GDN (scalar decay), gate and norm closed forms, the
 * conv step and the prefill conv against a library convolution, the gated
 * RMSNorm against a library rms_norm and its closed forms, the GDN and GDN-2
 * backward against central finite differences.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL -1
#define ORACLE_ENOMEM -2

static inline double ld(const void* p, int f64, size_t i) {
  return f64 ? ((const double*)p)[i] : (double)((const float*)p)[i];
}

/* softplus(x) = log(1 + e^x) ("从 Full Attention 到 Gated DeltaNet", section 9) */
static double softplus(double x) {
  if (x > 0.0) return x + log1p(exp(-x));
  return log1p(exp(x));
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Scalar gates of one (token, value head), "Qwen3.5" module skeleton. */
static void gdn_gates(double a, double b, double A_log, double dt_bias,
                      double* g, double* beta) {
  *g = -exp(A_log) * softplus(a + dt_bias);
  *beta = sigmoid(b);
}

/* Copies x[0..n) (strided source) into out, L2-normalising and scaling. */
static void load_vec(const void* src, int f64, size_t off, int n, int l2norm,
                     double scale, double* out) {
  for (int i = 0; i < n; ++i) out[i] = ld(src, f64, off + (size_t)i);
  if (l2norm) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += out[i] * out[i];
    double inv = 1.0 / sqrt(ss + 1e-6);
    for (int i = 0; i < n; ++i) out[i] *= inv;
  }
  if (scale != 1.0)
    for (int i = 0; i < n; ++i) out[i] *= scale;
}

/* One gated-delta-rule token step on S[dk][dv] ("Qwen3.5", 五步递推):
 *   S' = alpha S ; kv_j = sum_i S'_ij k_i ; delta_j = beta (v_j - kv_j) ;
 *   S_ij = S'_ij + k_i delta_j ; o_j = sum_i S_ij q_i                       */
static void gdn_token_step(double* S, int dk, int dv, const double* q,
                           const double* k, const double* v, double alpha,
                           double beta, double* kv, double* o) {
  for (size_t x = 0; x < (size_t)dk * dv; ++x) S[x] *= alpha;
  for (int j = 0; j < dv; ++j) kv[j] = 0.0;
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) kv[j] += S[(size_t)i * dv + j] * k[i];
  for (int j = 0; j < dv; ++j) kv[j] = beta * (v[j] - kv[j]);
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += k[i] * kv[j];
  for (int j = 0; j < dv; ++j) o[j] = 0.0;
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < dv; ++j) o[j] += S[(size_t)i * dv + j] * q[i];
}

/*
 * GDN forward over whole sequences.
 *   q,k [B,T,Hk,dk]; v [B,T,Hv,dv]; a,b [B,T,Hv]; A_log,dt_bias [Hv];
 *   h0 [B,Hv,dk,dv] or NULL (zeros).
 *   gates_given = 1: a holds g (log-decay) and b holds beta directly, A_log and
 *   dt_bias unused (used by the pins to drive the core with exact gates).
 *   Outputs are compact over the selected heads: o [n_sel,T,dv], ht [n_sel,dk,dv]
 *   (either may be NULL).  sel lists b*Hv+hv; n_sel <= 0 means all heads in order.
 */
int oracle_gdn_fwd(const void* q, const void* k, const void* v, const void* a,
                   const void* b, const void* A_log, const void* dt_bias,
                   const void* h0, int in_f64, int B, int T, int Hk, int Hv,
                   int dk, int dv, double scale, int l2norm, int gates_given,
                   int n_sel, const int* sel, double* o, double* ht,
                   int n_threads) {
  if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return ORACLE_EINVAL;
  if (Hv % Hk != 0) return ORACLE_EINVAL;
  const int group = Hv / Hk;
  const int n_heads = n_sel > 0 ? n_sel : B * Hv;
  int err = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
  for (int s = 0; s < n_heads; ++s) {
    const int bh = n_sel > 0 ? sel[s] : s;
    const int bi = bh / Hv, hv = bh % Hv, hk = hv / group;
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* buf = (double*)malloc(sizeof(double) * (size_t)(2 * dk + 3 * dv));
    if (!S || !buf) {
      free(S); free(buf);
#pragma omp atomic write
      err = ORACLE_ENOMEM;
      continue;
    }
    double *qt = buf, *kt = buf + dk, *vt = buf + 2 * dk, *kv = vt + dv, *ot = kv + dv;
    if (h0)
      for (size_t x = 0; x < (size_t)dk * dv; ++x)
        S[x] = ld(h0, in_f64, (size_t)bh * dk * dv + x);
    for (int t = 0; t < T; ++t) {
      const size_t row = (size_t)bi * T + t;
      load_vec(q, in_f64, (row * Hk + hk) * dk, dk, l2norm, scale, qt);
      load_vec(k, in_f64, (row * Hk + hk) * dk, dk, l2norm, 1.0, kt);
      load_vec(v, in_f64, (row * Hv + hv) * dv, dv, 0, 1.0, vt);
      double g, beta;
      if (gates_given) {
        g = ld(a, in_f64, row * Hv + hv);
        beta = ld(b, in_f64, row * Hv + hv);
      } else {
        gdn_gates(ld(a, in_f64, row * Hv + hv), ld(b, in_f64, row * Hv + hv),
                  ld(A_log, in_f64, hv), ld(dt_bias, in_f64, hv), &g, &beta);
      }
      gdn_token_step(S, dk, dv, qt, kt, vt, exp(g), beta, kv, ot);
      if (o) memcpy(o + ((size_t)s * T + t) * dv, ot, sizeof(double) * dv);
    }
    if (ht) memcpy(ht + (size_t)s * dk * dv, S, sizeof(double) * dk * dv);
    free(S);
    free(buf);
  }
  return err;
}

/*
 * Gate and norm prologue alone: g, beta [B*T*Hv]; q_hat, k_hat [B*T*Hk*dk].
 */
int oracle_gate_prep(const void* q, const void* k, const void* a, const void* b,
                     const void* A_log, const void* dt_bias, int in_f64, int B,
                     int T, int Hk, int Hv, int d, double scale, double* q_hat,
                     double* k_hat, double* g, double* beta) {
  if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || d <= 0) return ORACLE_EINVAL;
  const size_t rows = (size_t)B * T;
  for (size_t r = 0; r < rows; ++r) {
    for (int h = 0; h < Hk; ++h) {
      const size_t off = (r * Hk + h) * d;
      if (q_hat) load_vec(q, in_f64, off, d, 1, scale, q_hat + off);
      if (k_hat) load_vec(k, in_f64, off, d, 1, 1.0, k_hat + off);
    }
    for (int h = 0; h < Hv; ++h) {
      double gg, bb;
      gdn_gates(ld(a, in_f64, r * Hv + h), ld(b, in_f64, r * Hv + h),
                ld(A_log, in_f64, h), ld(dt_bias, in_f64, h), &gg, &bb);
      if (g) g[r * Hv + h] = gg;
      if (beta) beta[r * Hv + h] = bb;
    }
  }
  return ORACLE_OK;
}

/*
 * Causal depthwise conv1d (kernel 4) + SiLU for one new input per channel,
 * with the cached window updated in place ("从 Full Attention 到 Gated DeltaNet"
 * section 10: x -> CausalConv1D -> SiLU; "gated-deltanet-qwen3.5": decode
 * updates conv_states).  Window [cs0, cs1, cs2, x]; tap 3 multiplies the newest
 * input; cs2 is the newest cached input; no bias.
 *   x [Cc] (strided source at offset x_off), conv_w [Cc,4], cs [Cc,3] in/out,
 *   y [Cc] out.
 */
static void conv_silu_step(const void* x, size_t x_off, const void* conv_w,
                           int in_f64, int Cc, double* cs, double* y) {
  for (int c = 0; c < Cc; ++c) {
    const double xn = ld(x, in_f64, x_off + (size_t)c);
    double acc = ld(conv_w, in_f64, (size_t)c * 4 + 0) * cs[c * 3 + 0] +
                 ld(conv_w, in_f64, (size_t)c * 4 + 1) * cs[c * 3 + 1] +
                 ld(conv_w, in_f64, (size_t)c * 4 + 2) * cs[c * 3 + 2] +
                 ld(conv_w, in_f64, (size_t)c * 4 + 3) * xn;
    y[c] = acc * sigmoid(acc);
    cs[c * 3 + 0] = cs[c * 3 + 1];
    cs[c * 3 + 1] = cs[c * 3 + 2];
    cs[c * 3 + 2] = xn;
  }
}

/* The conv step alone for N sequences: x [N,Cc], conv_state [N,Cc,3] in/out,
 * y [N,Cc] out. */
int oracle_conv_step(const void* x, const void* conv_w, int in_f64, int N,
                     int Cc, double* conv_state, double* y) {
  if (N < 0 || Cc <= 0) return ORACLE_EINVAL;
  for (int n = 0; n < N; ++n)
    conv_silu_step(x, (size_t)n * Cc, conv_w, in_f64, Cc,
                   conv_state + (size_t)n * Cc * 3, y + (size_t)n * Cc);
  return ORACLE_OK;
}

/* The conv step over a whole prefill, token after token (the window carried
 * from one token to the next exactly as between decode steps):
 * x [B, T, Cc], conv_state [B, Cc, 3] (float64) in/out, y [B, T, Cc] out. */
int oracle_conv_prefill(const void* x, const void* conv_w, int in_f64, int B, int T,
                        int Cc, double* conv_state, double* y) {
  if (B < 0 || T < 0 || Cc <= 0) return ORACLE_EINVAL;
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t)
      conv_silu_step(x, ((size_t)b * T + t) * Cc, conv_w, in_f64, Cc,
                     conv_state + (size_t)b * Cc * 3, y + ((size_t)b * T + t) * Cc);
  return ORACLE_OK;
}

/*
 * One decode step for the selected sequences: the conv step above over the
 * mixed [q | k | v] channel stream, then per value head the L2 norm, gates and
 * one gated-delta-rule token step.
 *   x [N, Cc] with Cc = 2*Hk*dk + Hv*dv (pre-conv when conv_w != NULL, else
 *   already post-conv); conv_w [Cc,4]; a,b [N,Hv]; A_log,dt_bias [Hv].
 *   In/out, compact over the selection: conv_state [n_sel,Cc,3] (float64),
 *   state [n_sel,Hv,dk,dv]; out: o [n_sel,Hv,dv].
 *   sel lists sequence indices; n_sel <= 0 means all N in order.
 */
int oracle_gdn_decode_step(const void* x, const void* conv_w, const void* a,
                           const void* b, const void* A_log, const void* dt_bias,
                           int in_f64, int N, int Hk, int Hv, int dk, int dv,
                           double scale, int n_sel, const int* sel,
                           double* conv_state, double* state, double* o,
                           int n_threads) {
  if (N < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk) return ORACLE_EINVAL;
  const int group = Hv / Hk;
  const int Cc = 2 * Hk * dk + Hv * dv;
  const int n_seq = n_sel > 0 ? n_sel : N;
  int err = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
  for (int s = 0; s < n_seq; ++s) {
    const int n = n_sel > 0 ? sel[s] : s;
    double* y = (double*)malloc(sizeof(double) * ((size_t)Cc + 2 * dk + 3 * dv));
    if (!y) {
#pragma omp atomic write
      err = ORACLE_ENOMEM;
      continue;
    }
    double *qt = y + Cc, *kt = qt + dk, *vt = kt + dk, *kv = vt + dv, *ot = kv + dv;
    if (conv_w) {
      conv_silu_step(x, (size_t)n * Cc, conv_w, in_f64, Cc,
                     conv_state + (size_t)s * Cc * 3, y);
    } else {
      for (int c = 0; c < Cc; ++c) y[c] = ld(x, in_f64, (size_t)n * Cc + c);
    }
    for (int hv = 0; hv < Hv; ++hv) {
      const int hk = hv / group;
      load_vec(y, 1, (size_t)hk * dk, dk, 1, scale, qt);
      load_vec(y, 1, (size_t)Hk * dk + (size_t)hk * dk, dk, 1, 1.0, kt);
      load_vec(y, 1, (size_t)2 * Hk * dk + (size_t)hv * dv, dv, 0, 1.0, vt);
      double g, beta;
      gdn_gates(ld(a, in_f64, (size_t)n * Hv + hv), ld(b, in_f64, (size_t)n * Hv + hv),
                ld(A_log, in_f64, hv), ld(dt_bias, in_f64, hv), &g, &beta);
      double* S = state + ((size_t)s * Hv + hv) * dk * dv;
      gdn_token_step(S, dk, dv, qt, kt, vt, exp(g), beta, kv, ot);
      memcpy(o + ((size_t)s * Hv + hv) * dv, ot, sizeof(double) * dv);
    }
    free(y);
  }
  return err;
}

/*
 * Gated DeltaNet-2 forward ("Gated DeltaNet-2", 新更新公式):
 *   d = exp(-exp(A_log[h,:]) * softplus(a_t + dt_bias[h,:]))   (channel decay)
 *   e = sigmoid(b_t) (.) k_hat ; z = sigmoid(w_t) (.) v
 *   S_bar = diag(d) S ; r = S_bar^T e ; S = S_bar + k_hat (z - r)^T ; o = S^T q_hat
 *   q,k [B,T,H,dk]; v [B,T,H,dv]; a,b_logit [B,T,H,dk]; w_logit [B,T,H,dv];
 *   A_log,dt_bias [H,dk]; h0 [B,H,dk,dv] or NULL.
 *   gates_given = 1: a holds the log-decay per channel, b_logit holds b and
 *   w_logit holds w directly.
 *   Outputs compact over the selection, as in oracle_gdn_fwd.
 */
int oracle_gdn2_fwd(const void* q, const void* k, const void* v, const void* a,
                    const void* b_logit, const void* w_logit, const void* A_log,
                    const void* dt_bias, const void* h0, int in_f64, int B, int T,
                    int H, int dk, int dv, double scale, int l2norm,
                    int gates_given, int n_sel, const int* sel, double* o,
                    double* ht, int n_threads) {
  if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_EINVAL;
  const int n_heads = n_sel > 0 ? n_sel : B * H;
  int err = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
  for (int s = 0; s < n_heads; ++s) {
    const int bh = n_sel > 0 ? sel[s] : s;
    const int bi = bh / H, h = bh % H;
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* buf = (double*)malloc(sizeof(double) * (size_t)(4 * dk + 4 * dv));
    if (!S || !buf) {
      free(S); free(buf);
#pragma omp atomic write
      err = ORACLE_ENOMEM;
      continue;
    }
    double *qt = buf, *kt = qt + dk, *et = kt + dk, *dec = et + dk;
    double *vt = dec + dk, *zt = vt + dv, *rt = zt + dv, *ot = rt + dv;
    if (h0)
      for (size_t x = 0; x < (size_t)dk * dv; ++x)
        S[x] = ld(h0, in_f64, (size_t)bh * dk * dv + x);
    for (int t = 0; t < T; ++t) {
      const size_t row = ((size_t)bi * T + t) * H + h;
      load_vec(q, in_f64, row * dk, dk, l2norm, scale, qt);
      load_vec(k, in_f64, row * dk, dk, l2norm, 1.0, kt);
      load_vec(v, in_f64, row * dv, dv, 0, 1.0, vt);
      for (int i = 0; i < dk; ++i) {
        double gi, bi_;
        if (gates_given) {
          gi = ld(a, in_f64, row * dk + i);
          bi_ = ld(b_logit, in_f64, row * dk + i);
        } else {
          gi = -exp(ld(A_log, in_f64, (size_t)h * dk + i)) *
               softplus(ld(a, in_f64, row * dk + i) + ld(dt_bias, in_f64, (size_t)h * dk + i));
          bi_ = sigmoid(ld(b_logit, in_f64, row * dk + i));
        }
        dec[i] = exp(gi);
        et[i] = bi_ * kt[i];
      }
      for (int j = 0; j < dv; ++j) {
        double wj = gates_given ? ld(w_logit, in_f64, row * dv + j)
                                : sigmoid(ld(w_logit, in_f64, row * dv + j));
        zt[j] = wj * vt[j];
      }
      /* S_bar = D S */
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= dec[i];
      /* r = S_bar^T e */
      for (int j = 0; j < dv; ++j) rt[j] = 0.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) rt[j] += S[(size_t)i * dv + j] * et[i];
      /* S = S_bar + k (z - r)^T */
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += kt[i] * (zt[j] - rt[j]);
      /* o = S^T q */
      for (int j = 0; j < dv; ++j) ot[j] = 0.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) ot[j] += S[(size_t)i * dv + j] * qt[i];
      if (o) memcpy(o + ((size_t)s * T + t) * dv, ot, sizeof(double) * dv);
    }
    if (ht) memcpy(ht + (size_t)s * dk * dv, S, sizeof(double) * dk * dv);
    free(S);
    free(buf);
  }
  return err;
}

/* Gradient of the L2 norm and scale of load_vec: x -> scale * x / sqrt(sum x^2 + eps)
 * (or scale * x without the norm); gy is the gradient at the output, gx += the
 * gradient at the input. */
static void load_vec_bwd(const double* x, int n, int l2norm, double scale, const double* gy,
                         double* gx) {
  if (!l2norm) {
    for (int i = 0; i < n; ++i) gx[i] += scale * gy[i];
    return;
  }
  double ss = 0.0, xg = 0.0;
  for (int i = 0; i < n; ++i) {
    ss += x[i] * x[i];
    xg += x[i] * gy[i];
  }
  const double nrm = sqrt(ss + 1e-6);
  for (int i = 0; i < n; ++i) gx[i] += scale * (gy[i] / nrm - x[i] * xg / (nrm * nrm * nrm));
}

/*
 * Backward of oracle_gdn_fwd (the next step after the forward pass): reverse-mode
 * differentiation of the five-step token recurrence, token by token from the
 * last, with the states of the forward pass stored.  For a cotangent do on o and
 * dht on the final state, it returns the gradients of sum(o * do) + sum(ht * dht):
 *   dq, dk [B,T,Hk,dk] (summed over the value heads of a key head), dv [B,T,Hv,dv],
 *   da, db [B,T,Hv] (with gates_given: the gradients with respect to g and beta),
 *   dA_log, ddt_bias [Hv] (summed over batch and tokens; untouched with
 *   gates_given), dh0 [B,Hv,dk,dv].  dht may be NULL (zero).  Single-threaded:
 *   it is meant for the small cases of the tests.
 * Per token, with S the state before it:
 *   S' = a S ; kv = S'^T k ; d = b (v - kv) ; S_t = S' + k d^T ; o = S_t^T q
 * reversed: dS += q do^T, dq = S_t do ; dk = dS d, dd = dS^T k ; db = dd.(v - kv),
 * dv = b dd, dkv = -b dd ; dS' = dS + k dkv^T, dk += S' dkv ; dS <- a dS',
 * da = <dS', S>.
 */
int oracle_gdn_bwd(const double* q, const double* k, const double* v, const double* a,
                   const double* b, const double* A_log, const double* dt_bias,
                   const double* h0, const double* dout, const double* dht, int B, int T,
                   int Hk, int Hv, int dk, int dv, double scale, int l2norm, int gates_given,
                   double* dq, double* dkk, double* dvv, double* da, double* db,
                   double* dA_log, double* ddt_bias, double* dh0) {
  if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk) return ORACLE_EINVAL;
  const int group = Hv / Hk;
  const size_t SZ = (size_t)dk * dv;
  memset(dq, 0, sizeof(double) * (size_t)B * T * Hk * dk);
  memset(dkk, 0, sizeof(double) * (size_t)B * T * Hk * dk);
  if (!gates_given) {
    memset(dA_log, 0, sizeof(double) * Hv);
    memset(ddt_bias, 0, sizeof(double) * Hv);
  }
  double* Sp = (double*)malloc(sizeof(double) * SZ * ((size_t)T + 1));  /* states S_0 .. S_T */
  double* St = (double*)malloc(sizeof(double) * SZ);                    /* S' of a token */
  double* dS = (double*)malloc(sizeof(double) * SZ);
  double* dSp = (double*)malloc(sizeof(double) * SZ);
  double* w = (double*)malloc(sizeof(double) * (size_t)(4 * dk + 6 * dv + 4));
  if (!Sp || !St || !dS || !dSp || !w) {
    free(Sp); free(St); free(dS); free(dSp); free(w);
    return ORACLE_ENOMEM;
  }
  double *qt = w, *kt = qt + dk, *gq = kt + dk, *gk = gq + dk;
  double *vt = gk + dk, *kv = vt + dv, *dd = kv + dv, *dl = dd + dv, *ot = dl + dv, *dkv = ot + dv;
  for (int bi = 0; bi < B; ++bi)
    for (int hv = 0; hv < Hv; ++hv) {
      const int hk = hv / group;
      const size_t bh = (size_t)bi * Hv + hv;
      for (size_t x = 0; x < SZ; ++x) Sp[x] = h0 ? h0[bh * SZ + x] : 0.0;
      /* forward, keeping S_0 .. S_T */
      for (int t = 0; t < T; ++t) {
        const size_t row = (size_t)bi * T + t;
        load_vec(q, 1, (row * Hk + hk) * dk, dk, l2norm, scale, qt);
        load_vec(k, 1, (row * Hk + hk) * dk, dk, l2norm, 1.0, kt);
        load_vec(v, 1, (row * Hv + hv) * dv, dv, 0, 1.0, vt);
        double g, beta;
        if (gates_given) {
          g = a[row * Hv + hv];
          beta = b[row * Hv + hv];
        } else {
          gdn_gates(a[row * Hv + hv], b[row * Hv + hv], A_log[hv], dt_bias[hv], &g, &beta);
        }
        memcpy(Sp + (size_t)(t + 1) * SZ, Sp + (size_t)t * SZ, sizeof(double) * SZ);
        gdn_token_step(Sp + (size_t)(t + 1) * SZ, dk, dv, qt, kt, vt, exp(g), beta, kv, ot);
      }
      /* backward */
      for (size_t x = 0; x < SZ; ++x) dS[x] = dht ? dht[bh * SZ + x] : 0.0;
      for (int t = T - 1; t >= 0; --t) {
        const size_t row = (size_t)bi * T + t;
        const double* S0 = Sp + (size_t)t * SZ;   /* state before the token */
        const double* S1 = Sp + (size_t)(t + 1) * SZ;
        load_vec(q, 1, (row * Hk + hk) * dk, dk, l2norm, scale, qt);
        load_vec(k, 1, (row * Hk + hk) * dk, dk, l2norm, 1.0, kt);
        load_vec(v, 1, (row * Hv + hv) * dv, dv, 0, 1.0, vt);
        double g, beta;
        if (gates_given) {
          g = a[row * Hv + hv];
          beta = b[row * Hv + hv];
        } else {
          gdn_gates(a[row * Hv + hv], b[row * Hv + hv], A_log[hv], dt_bias[hv], &g, &beta);
        }
        const double alpha = exp(g);
        const double* dO = dout + (row * Hv + hv) * dv;
        /* recompute S', kv and delta of the token */
        for (size_t x = 0; x < SZ; ++x) St[x] = alpha * S0[x];
        for (int j = 0; j < dv; ++j) kv[j] = 0.0;
        for (int i = 0; i < dk; ++i)
          for (int j = 0; j < dv; ++j) kv[j] += St[(size_t)i * dv + j] * kt[i];
        for (int j = 0; j < dv; ++j) dl[j] = beta * (vt[j] - kv[j]);
        /* o = S_t^T q */
        for (int i = 0; i < dk; ++i) {
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) {
            acc += S1[(size_t)i * dv + j] * dO[j];
            dS[(size_t)i * dv + j] += qt[i] * dO[j];
          }
          gq[i] = acc;
        }
        /* S_t = S' + k delta^T */
        for (int i = 0; i < dk; ++i) {
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) acc += dS[(size_t)i * dv + j] * dl[j];
          gk[i] = acc;
        }
        for (int j = 0; j < dv; ++j) {
          double acc = 0.0;
          for (int i = 0; i < dk; ++i) acc += dS[(size_t)i * dv + j] * kt[i];
          dd[j] = acc;
        }
        /* delta = beta (v - kv) */
        double dbeta = 0.0;
        for (int j = 0; j < dv; ++j) {
          dbeta += dd[j] * (vt[j] - kv[j]);
          dvv[(row * Hv + hv) * dv + j] = beta * dd[j];
          dkv[j] = -beta * dd[j];
        }
        /* kv = S'^T k */
        for (int i = 0; i < dk; ++i) {
          double acc = 0.0;
          for (int j = 0; j < dv; ++j) {
            dSp[(size_t)i * dv + j] = dS[(size_t)i * dv + j] + kt[i] * dkv[j];
            acc += St[(size_t)i * dv + j] * dkv[j];
          }
          gk[i] += acc;
        }
        /* S' = alpha S */
        double dalpha = 0.0;
        for (size_t x = 0; x < SZ; ++x) {
          dalpha += dSp[x] * S0[x];
          dS[x] = alpha * dSp[x];
        }
        const double dg = dalpha * alpha;
        if (gates_given) {
          da[row * Hv + hv] = dg;
          db[row * Hv + hv] = dbeta;
        } else {
          const double xg = a[row * Hv + hv] + dt_bias[hv];
          const double dx = dg * (-exp(A_log[hv])) * sigmoid(xg);
          da[row * Hv + hv] = dx;
          ddt_bias[hv] += dx;
          dA_log[hv] += dg * g;
          db[row * Hv + hv] = dbeta * beta * (1.0 - beta);
        }
        /* the norms of q and k */
        load_vec_bwd(q + (row * Hk + hk) * dk, dk, l2norm, scale, gq, dq + (row * Hk + hk) * dk);
        load_vec_bwd(k + (row * Hk + hk) * dk, dk, l2norm, 1.0, gk, dkk + (row * Hk + hk) * dk);
      }
      if (dh0) memcpy(dh0 + bh * SZ, dS, sizeof(double) * SZ);
    }
  free(Sp); free(St); free(dS); free(dSp); free(w);
  return ORACLE_OK;
}

/*
 * Backward of oracle_gdn2_fwd ("Gated DeltaNet-2", section Gate-aware 反向传播:
 * the per-channel gates stay inside the accumulations), reverse-mode token by
 * token from the last, the forward states stored.  Per token, with S the state
 * before it, d = exp(g) per key channel, e = b (.) k, z = w (.) v:
 *   S_bar = diag(d) S ; r = S_bar^T e ; S_t = S_bar + k (z - r)^T ; o = S_t^T q
 * reversed: dS += q do^T, dq = S_t do ; m = dS^T k, dk = dS (z - r), dz = m,
 * dr = -m ; dS_bar = dS + e dr^T, de = S_bar dr ; db = de (.) k, dk += de (.) b ;
 * dw = dz (.) v, dv = dz (.) w ; dS <- diag(d) dS_bar, dd_i = <dS_bar_i, S_i>.
 * Gradients of sum(o * do) + sum(ht * dht): dq, dk [B,T,H,dk], dv [B,T,H,dv],
 * da, db [B,T,H,dk], dw [B,T,H,dv] (with gates_given: with respect to g, b, w),
 * dA_log, ddt_bias [H,dk] (summed over batch and tokens), dh0 [B,H,dk,dv].
 */
int oracle_gdn2_bwd(const double* q, const double* k, const double* v, const double* a,
                    const double* b_logit, const double* w_logit, const double* A_log,
                    const double* dt_bias, const double* h0, const double* dout,
                    const double* dht, int B, int T, int H, int dk, int dv, double scale,
                    int l2norm, int gates_given, double* dq, double* dkk, double* dvv,
                    double* da, double* db, double* dw, double* dA_log, double* ddt_bias,
                    double* dh0) {
  if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_EINVAL;
  const size_t SZ = (size_t)dk * dv;
  memset(dq, 0, sizeof(double) * (size_t)B * T * H * dk);
  memset(dkk, 0, sizeof(double) * (size_t)B * T * H * dk);
  if (!gates_given) {
    memset(dA_log, 0, sizeof(double) * (size_t)H * dk);
    memset(ddt_bias, 0, sizeof(double) * (size_t)H * dk);
  }
  double* Sp = (double*)malloc(sizeof(double) * SZ * ((size_t)T + 1));
  double* Sb = (double*)malloc(sizeof(double) * SZ);
  double* dS = (double*)malloc(sizeof(double) * SZ);
  double* wk = (double*)malloc(sizeof(double) * (size_t)(9 * dk + 7 * dv));
  if (!Sp || !Sb || !dS || !wk) {
    free(Sp); free(Sb); free(dS); free(wk);
    return ORACLE_ENOMEM;
  }
  double *qt = wk, *kt = qt + dk, *gq = kt + dk, *gk = gq + dk, *dec = gk + dk, *gd = dec + dk;
  double *bg = gd + dk, *et = bg + dk, *de = et + dk;
  double *vt = de + dk, *wg = vt + dv, *zt = wg + dv, *rt = zt + dv, *ot = rt + dv, *m = ot + dv;
  double* drr = m + dv;
  for (int bi = 0; bi < B; ++bi)
    for (int h = 0; h < H; ++h) {
      const size_t bh = (size_t)bi * H + h;
      for (size_t x = 0; x < SZ; ++x) Sp[x] = h0 ? h0[bh * SZ + x] : 0.0;
      /* forward with the states kept: the same arithmetic as oracle_gdn2_fwd */
      for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1)
          for (size_t x = 0; x < SZ; ++x) dS[x] = dht ? dht[bh * SZ + x] : 0.0;
        for (int tt = 0; tt < T; ++tt) {
          const int t = pass == 0 ? tt : T - 1 - tt;
          const size_t row = ((size_t)bi * T + t) * H + h;
          load_vec(q, 1, row * dk, dk, l2norm, scale, qt);
          load_vec(k, 1, row * dk, dk, l2norm, 1.0, kt);
          load_vec(v, 1, row * dv, dv, 0, 1.0, vt);
          for (int i = 0; i < dk; ++i) {
            double gi;
            if (gates_given) {
              gi = a[row * dk + i];
              bg[i] = b_logit[row * dk + i];
            } else {
              gi = -exp(A_log[(size_t)h * dk + i]) *
                   softplus(a[row * dk + i] + dt_bias[(size_t)h * dk + i]);
              bg[i] = sigmoid(b_logit[row * dk + i]);
            }
            gd[i] = gi;
            dec[i] = exp(gi);
            et[i] = bg[i] * kt[i];
          }
          for (int j = 0; j < dv; ++j) {
            wg[j] = gates_given ? w_logit[row * dv + j] : sigmoid(w_logit[row * dv + j]);
            zt[j] = wg[j] * vt[j];
          }
          const double* S0 = Sp + (size_t)t * SZ;
          double* S1 = Sp + (size_t)(t + 1) * SZ;
          for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) Sb[(size_t)i * dv + j] = dec[i] * S0[(size_t)i * dv + j];
          for (int j = 0; j < dv; ++j) rt[j] = 0.0;
          for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) rt[j] += Sb[(size_t)i * dv + j] * et[i];
          if (pass == 0) {
            for (int i = 0; i < dk; ++i)
              for (int j = 0; j < dv; ++j)
                S1[(size_t)i * dv + j] = Sb[(size_t)i * dv + j] + kt[i] * (zt[j] - rt[j]);
            continue;
          }
          /* backward of the token */
          const double* dO = dout + row * dv;
          for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) {
              acc += S1[(size_t)i * dv + j] * dO[j];
              dS[(size_t)i * dv + j] += qt[i] * dO[j];
            }
            gq[i] = acc;
          }
          for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += dS[(size_t)i * dv + j] * kt[i];
            m[j] = acc;
            drr[j] = -acc;
          }
          for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) acc += dS[(size_t)i * dv + j] * (zt[j] - rt[j]);
            gk[i] = acc;
          }
          for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) {
              dS[(size_t)i * dv + j] += et[i] * drr[j];      /* dS_bar */
              acc += Sb[(size_t)i * dv + j] * drr[j];
            }
            de[i] = acc;
          }
          for (int j = 0; j < dv; ++j) {
            dvv[row * dv + j] = m[j] * wg[j];
            const double dwj = m[j] * vt[j];
            dw[row * dv + j] = gates_given ? dwj : dwj * wg[j] * (1.0 - wg[j]);
          }
          for (int i = 0; i < dk; ++i) {
            const double dbi = de[i] * kt[i];
            gk[i] += de[i] * bg[i];
            db[row * dk + i] = gates_given ? dbi : dbi * bg[i] * (1.0 - bg[i]);
            double ddi = 0.0;
            for (int j = 0; j < dv; ++j) {
              ddi += dS[(size_t)i * dv + j] * S0[(size_t)i * dv + j];
              dS[(size_t)i * dv + j] *= dec[i];
            }
            const double dgi = ddi * dec[i];
            if (gates_given) {
              da[row * dk + i] = dgi;
            } else {
              const double xg = a[row * dk + i] + dt_bias[(size_t)h * dk + i];
              const double dx = dgi * (-exp(A_log[(size_t)h * dk + i])) * sigmoid(xg);
              da[row * dk + i] = dx;
              ddt_bias[(size_t)h * dk + i] += dx;
              dA_log[(size_t)h * dk + i] += dgi * gd[i];
            }
          }
          load_vec_bwd(q + row * dk, dk, l2norm, scale, gq, dq + row * dk);
          load_vec_bwd(k + row * dk, dk, l2norm, 1.0, gk, dkk + row * dk);
        }
      }
      if (dh0) memcpy(dh0 + bh * SZ, dS, sizeof(double) * SZ);
    }
  free(Sp); free(Sb); free(dS); free(wk);
  return ORACLE_OK;
}

/*
 * KDA (Kimi Delta Attention) as the "Gated DeltaNet-2" page states its update
 * (section 标量绑定的数学表达), computed literally:
 *   S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T ;  o_t = S_t^T q_t
 * with D_t = diag(exp(g_t)), g_t = -exp(A_log) * softplus(a_t + dt_bias) per key
 * channel, and one scalar beta_t = sigmoid(b_t) per (token, head); the d_k x d_k
 * erase projection P = I - beta k k^T is formed and applied to D S.
 *   q,k [B,T,H,dk]; v [B,T,H,dv]; a [B,T,H,dk]; b [B,T,H]; A_log,dt_bias [H,dk];
 *   h0 [B,H,dk,dv] or NULL.  Out: o [B*H][T][dv], ht [B*H][dk][dv] (either NULL).
 */
int oracle_kda_fwd(const void* q, const void* k, const void* v, const void* a,
                   const void* b, const void* A_log, const void* dt_bias, const void* h0,
                   int in_f64, int B, int T, int H, int dk, int dv, double scale, int l2norm,
                   double* o, double* ht, int n_threads) {
  if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return ORACLE_EINVAL;
  int err = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
  for (int bh = 0; bh < B * H; ++bh) {
    const int bi = bh / H, h = bh % H;
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* DS = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* P = (double*)malloc(sizeof(double) * (size_t)dk * dk);
    double* buf = (double*)malloc(sizeof(double) * (size_t)(3 * dk + 2 * dv));
    if (!S || !DS || !P || !buf) {
      free(S); free(DS); free(P); free(buf);
#pragma omp atomic write
      err = ORACLE_ENOMEM;
      continue;
    }
    double *qt = buf, *kt = qt + dk, *dec = kt + dk, *vt = dec + dk, *ot = vt + dv;
    if (h0)
      for (size_t x = 0; x < (size_t)dk * dv; ++x)
        S[x] = ld(h0, in_f64, (size_t)bh * dk * dv + x);
    for (int t = 0; t < T; ++t) {
      const size_t row = ((size_t)bi * T + t) * H + h;
      load_vec(q, in_f64, row * dk, dk, l2norm, scale, qt);
      load_vec(k, in_f64, row * dk, dk, l2norm, 1.0, kt);
      load_vec(v, in_f64, row * dv, dv, 0, 1.0, vt);
      for (int i = 0; i < dk; ++i)
        dec[i] = exp(-exp(ld(A_log, in_f64, (size_t)h * dk + i)) *
                     softplus(ld(a, in_f64, row * dk + i) + ld(dt_bias, in_f64, (size_t)h * dk + i)));
      const double beta = sigmoid(ld(b, in_f64, row));
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) DS[(size_t)i * dv + j] = dec[i] * S[(size_t)i * dv + j];
      for (int i = 0; i < dk; ++i)
        for (int l = 0; l < dk; ++l) P[(size_t)i * dk + l] = (i == l ? 1.0 : 0.0) - beta * kt[i] * kt[l];
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) {
          double acc = beta * kt[i] * vt[j];
          for (int l = 0; l < dk; ++l) acc += P[(size_t)i * dk + l] * DS[(size_t)l * dv + j];
          S[(size_t)i * dv + j] = acc;
        }
      for (int j = 0; j < dv; ++j) ot[j] = 0.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) ot[j] += S[(size_t)i * dv + j] * qt[i];
      if (o) memcpy(o + ((size_t)bh * T + t) * dv, ot, sizeof(double) * dv);
    }
    if (ht) memcpy(ht + (size_t)bh * dk * dv, S, sizeof(double) * dk * dv);
    free(S); free(DS); free(P); free(buf);
  }
  return err;
}

/* Gated RMSNorm of N rows of d_v channels: o, z [N, dv], weight [dv] (shared by
 * every row), y [N, dv] out. */
int oracle_rmsnorm_gated(const void* o, const void* z, const void* weight, int in_f64,
                         int N, int dv, double eps, double* y) {
  if (N < 0 || dv <= 0 || !(eps >= 0.0)) return ORACLE_EINVAL;
  for (int n = 0; n < N; ++n) {
    double ss = 0.0;
    for (int j = 0; j < dv; ++j) {
      const double v = ld(o, in_f64, (size_t)n * dv + j);
      ss += v * v;
    }
    const double inv = 1.0 / sqrt(ss / dv + eps);
    for (int j = 0; j < dv; ++j) {
      const double zj = ld(z, in_f64, (size_t)n * dv + j);
      y[(size_t)n * dv + j] =
          ld(o, in_f64, (size_t)n * dv + j) * inv * ld(weight, in_f64, (size_t)j) * (zj * sigmoid(zj));
    }
  }
  return ORACLE_OK;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
