/*
 * FusedBitLinear oracle: a plain, slow, scalar CPU statement of what the projection computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark may load this library.  The product path (the CUDA library and its Python binding)
 * never calls it and shares no code with it.
 *
 * Sources (page title, section):
 *  [P1] "matmulfreellm 評価: 行列積を消した HGRNBit を Transformers 互換で読む" (hysenlabs, ja),
 *       section "HGRNBit という層構成を読む": every i/f/g/o projection is a FusedBitLinear that
 *       holds an RMSNorm(eps=1e-08) inside it; the MLP is gate_proj 2048->11264, then SiLU, then
 *       down_proj 5632->2048.
 *  [P3] "MatMul-Free LM: Ternary-Gewichte statt Matrixmultiplikation im Transformer" (hysenlabs,
 *       de), section "HGRNBit: was in einem Block tatsächlich passiert": bias=False, the norm is
 *       fused with the ternary projection.
 *  [P4] "MatMul-freie LLMs: Zentrale Konzepte erklärt" (datacamp, de):
 *       section "MatMul durch ternäre Operationen ersetzen" (absmean quantisation of the weight
 *       matrix to {-1,0,1}; multiplications become additions and subtractions);
 *       section "Kernkomponenten: MLGRU und GLU", figure items 4 (scaled ternary accumulation)
 *       and 5 (RMSNorm normalises activations before quantisation), and the GLU paragraph
 *       (one branch through SiLU, multiplied element-wise by the other).
 *  [P5] "量子化とは何か？MatMulというAIの計算やモデルサイズの最大のネック" (bluegarage, ja),
 *       section "MatMulとは具体的にどんな計算か" and its worked example "具体例".
 *  [P4] again, section "Kernkomponenten: MLGRU und GLU", the MLGRU paragraph: the recurrence
 *       runs token by token; each step takes the current token and the previous hidden state
 *       and updates the state element-wise through gates, vectors of values between 0 and 1,
 *       that weigh which parts of the previous state and of the current token carry on.
 *  [P1] again: the gating of the attention side is FusedRMSNormSwishGate, and its output goes
 *       through o_proj.
 *
 * Readings where the pages are silent (each is also listed with its reason in the design notes):
 *  - activations: per-token absmax to int8, s = 127/gamma, round half to even, clamp [-128,127];
 *  - RMSNorm: r = sqrt(mean(x^2) + eps) with the mean of squares accumulated in double and
 *    rounded once to float; then xhat = (x * (1/r)) * g in float;
 *  - gamma and beta are floored at 1e-5 so that an all-zero row or matrix divides safely;
 *  - beta = float( double(exact sum |W|) / (N*K) ): the exact sum removes any dependence on
 *    summation order, so the value is unique;
 *  - dequantisation y = acc * (gamma/127) * beta and the GLU are evaluated in double;
 *  - GLU: the first half [0,I) of gate_proj's 2I outputs goes through SiLU, the second half is
 *    the multiplier.
 *  - MLGRU (the pages give no formula): forget gate f = sigmoid(f_proj output), candidate
 *    c = silu(i_proj output), h_t = f * h_{t-1} + (1 - f) * c, the state before the first token
 *    given (zero by default); all in double.
 *  - FusedRMSNormSwishGate: o = (h / sqrt(mean_j h_j^2 + eps)) * w * silu(g_proj output), the
 *    mean over the H channels of one token, in double.
 *  - backward (the pages give none): straight-through through both quantisers, i.e. the
 *    gradient of the bilinear map of the dequantised operands, then of the RMSNorm; the latent
 *    weight takes the quantised weight's gradient; in double.
 *
 * Every decision that turns a float into an integer (an activation code, a weight code) is made
 * in IEEE single precision, the precision the GPU path uses for the same decision.
 *
 * Pins: tests/test_oracle_pins.py checks this file against the worked integer example of [P5],
 * brute force over all ternary rows of short length, exact rational arithmetic, closed forms and
 * rounding bounds.  Parity status: every exported function is pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

#define ORC_FLOOR 1e-5f

/* ------------------------------------------------------------------------------------------ */
/* Generic integer matrix product, the definition worked through in [P5] "具体例":              */
/* C[i][j] = sum_p A[i][p] * B[p][j], A is m x k, B is k x n, all row-major.                     */
ORC_API void orc_dense_matmul_i64(const int64_t* A, const int64_t* B, int64_t m, int64_t k,
                                  int64_t n, int64_t* C) {
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) {
      int64_t s = 0;
      for (int64_t p = 0; p < k; ++p) s += A[i * k + p] * B[p * n + j];
      C[i * n + j] = s;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* RMSNorm inside the projection ([P1], [P3]; [P4] figure item 5: the norm comes before the     */
/* quantisation), then per-token absmax int8 quantisation of the normalised activations.        */
/* x: T x K floats; g: K floats or NULL (NULL means 1); outputs q (T x K int8), gamma (T),       */
/* rowsum (T, the plain sum of the row's codes; may be NULL).                                   */
ORC_API void orc_rmsnorm_actquant(const float* x, int64_t T, int64_t K, const float* g, float eps,
                                  int8_t* q, float* gamma, int32_t* rowsum) {
  float* xh = (float*)malloc(sizeof(float) * (size_t)K);
  for (int64_t t = 0; t < T; ++t) {
    const float* xr = x + t * K;
    double ss = 0.0;
    for (int64_t k = 0; k < K; ++k) ss += (double)xr[k] * (double)xr[k];
    float ms = (float)(ss / (double)K);
    float r = sqrtf(ms + eps);
    float inv_r = 1.0f / r;
    float gmax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float gk = g ? g[k] : 1.0f;
      xh[k] = (xr[k] * inv_r) * gk;
      float a = fabsf(xh[k]);
      if (a > gmax) gmax = a;
    }
    if (gmax < ORC_FLOOR) gmax = ORC_FLOOR;
    gamma[t] = gmax;
    float s = 127.0f / gmax;
    int32_t sum = 0;
    for (int64_t k = 0; k < K; ++k) {
      float v = rintf(xh[k] * s);
      if (v > 127.0f) v = 127.0f;
      if (v < -128.0f) v = -128.0f;
      q[t * K + k] = (int8_t)v;
      sum += (int32_t)v;
    }
    if (rowsum) rowsum[t] = sum;
  }
  free(xh);
}

/* ------------------------------------------------------------------------------------------ */
/* Absmean scale of a weight matrix ([P4] "MatMul durch ternäre Operationen ersetzen": the      */
/* matrix is scaled by its mean absolute value).  The sum of |W| is formed exactly: every       */
/* finite float is an integer multiple of 2^-149 below 2^128, so the sum is an integer that     */
/* fits a 384-bit accumulator for any count below 2^100.  It is rounded once to double (round   */
/* half to even), divided by the element count in double and rounded to float.                 */
typedef struct { uint64_t w[6]; } orc_big;

static void big_add(orc_big* a, uint64_t m, int shift) {
  int li = shift / 64, off = shift % 64;
  uint64_t lo = m << off;
  uint64_t hi = off ? (m >> (64 - off)) : 0;
  uint64_t c = 0;
  for (int i = li; i < 6; ++i) {
    uint64_t add = (i == li) ? lo : (i == li + 1 ? hi : 0);
    uint64_t s = a->w[i] + add;
    uint64_t c1 = s < add;
    uint64_t s2 = s + c;
    uint64_t c2 = s2 < c;
    a->w[i] = s2;
    c = c1 | c2;
    if (i > li + 1 && c == 0) break;
  }
}

static int big_bit(const orc_big* a, int b) { return (int)((a->w[b / 64] >> (b % 64)) & 1u); }

/* Round the accumulator (units of 2^-149) to the nearest double, ties to even. */
static double big_to_double(const orc_big* a) {
  int top = -1;
  for (int b = 6 * 64 - 1; b >= 0; --b)
    if (big_bit(a, b)) { top = b; break; }
  if (top < 0) return 0.0;
  if (top < 53) {
    uint64_t v = a->w[0];
    return ldexp((double)v, -149);
  }
  uint64_t mant = 0;
  for (int b = top; b > top - 53; --b) mant = (mant << 1) | (uint64_t)big_bit(a, b);
  int round = big_bit(a, top - 53);
  int sticky = 0;
  for (int b = top - 54; b >= 0; --b)
    if (big_bit(a, b)) { sticky = 1; break; }
  int exp2 = top - 52;
  if (round && (sticky || (mant & 1u))) {
    mant += 1;
    if (mant == (1ull << 53)) { mant >>= 1; exp2 += 1; }
  }
  return ldexp((double)mant, exp2 - 149);
}

/* Exact sum of |W| rounded once to double.  Returns NaN if any element is not finite. */
ORC_API double orc_abs_sum_exact(const float* W, int64_t n) {
  orc_big acc;
  memset(&acc, 0, sizeof(acc));
  for (int64_t i = 0; i < n; ++i) {
    uint32_t bits;
    memcpy(&bits, &W[i], 4);
    bits &= 0x7fffffffu;
    uint32_t e = bits >> 23, f = bits & 0x7fffffu;
    if (e == 255u) return NAN;
    if (e == 0u) {
      if (f) big_add(&acc, f, 0);             /* subnormal: f * 2^-149 */
    } else {
      big_add(&acc, f | 0x800000u, (int)e - 1); /* (1.f) * 2^(e-127) = (f|2^23) * 2^(e-150) */
    }
  }
  return big_to_double(&acc);
}

ORC_API float orc_absmean_beta(const float* W, int64_t n) {
  double s = orc_abs_sum_exact(W, n);
  float beta = (float)(s / (double)n);
  if (!(beta >= ORC_FLOOR)) beta = (beta != beta) ? beta : ORC_FLOOR;
  return beta;
}

/* Ternary codes c = clamp(round(W / beta), -1, 1) ([P4] "MatMul durch ternäre Operationen     */
/* ersetzen": each element is rounded to the nearest of -1, 0, 1).  Division and rounding in    */
/* float, ties to even.                                                                         */
ORC_API void orc_ternary_codes(const float* W, int64_t n, float beta, int8_t* c) {
  for (int64_t i = 0; i < n; ++i) {
    float v = rintf(W[i] / beta);
    if (v > 1.0f) v = 1.0f;
    if (v < -1.0f) v = -1.0f;
    c[i] = (int8_t)v;
  }
}

/* ------------------------------------------------------------------------------------------ */
/* 2-bit packing (the pages fix none; this is the library's layout).  A row of K codes is      */
/* stored in K/4 bytes.  The 16 codes k = 16G + 4i + j (i, j in 0..3) of group G live in the    */
/* little-endian 32-bit word at bytes 4G..4G+3 of the row, at bits 8j + 2i and 8j + 2i + 1,     */
/* holding e = c + 1 (0, 1 or 2; 3 never occurs).                                               */
ORC_API void orc_pack_codes(const int8_t* c, int64_t N, int64_t K, uint8_t* Wp) {
  memset(Wp, 0, (size_t)(N * (K / 4)));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      int64_t grp = k / 16, i = (k % 16) / 4, j = k % 4;
      uint32_t e = (uint32_t)(c[n * K + k] + 1);
      int bit = 8 * (int)j + 2 * (int)i;
      uint8_t* word = Wp + n * (K / 4) + 4 * grp;
      word[bit / 8] |= (uint8_t)(e << (bit % 8));
    }
}

ORC_API void orc_unpack_codes(const uint8_t* Wp, int64_t N, int64_t K, int8_t* c) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      int64_t grp = k / 16, i = (k % 16) / 4, j = k % 4;
      int bit = 8 * (int)j + 2 * (int)i;
      const uint8_t* word = Wp + n * (K / 4) + 4 * grp;
      int e = (word[bit / 8] >> (bit % 8)) & 3;
      c[n * K + k] = (int8_t)(e - 1);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Ternary accumulation ([P4]: multiplying by -1 negates, by 0 gives 0, by 1 keeps the value;  */
/* figure item 4, scaled ternary accumulation).  acc[t][n] = sum over k of q[t][k] where        */
/* c[n][k] = +1, minus the sum of q[t][k] where c[n][k] = -1.  Written as literal branches.     */
ORC_API void orc_ternary_accumulate(const int8_t* q, int64_t T, int64_t K, const int8_t* c,
                                    int64_t N, int32_t* acc) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t n = 0; n < N; ++n) {
      int32_t s = 0;
      const int8_t* qr = q + t * K;
      const int8_t* cr = c + n * K;
      for (int64_t k = 0; k < K; ++k) {
        if (cr[k] == 1)
          s += qr[k];
        else if (cr[k] == -1)
          s -= qr[k];
      }
      acc[t * N + n] = s;
    }
}

/* Dequantisation ([P4] figure item 4, "scaled"): y = acc * (gamma_t / 127) * beta, double.    */
ORC_API void orc_dequant(const int32_t* acc, int64_t T, int64_t N, const float* gamma, float beta,
                         double* y) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t n = 0; n < N; ++n)
      y[t * N + n] = (double)acc[t * N + n] * ((double)gamma[t] / 127.0) * (double)beta;
}

/* SiLU-GLU ([P4] GLU paragraph; [P1] gate_proj 2I wide, down_proj I wide, SiLU):              */
/* h[t][i] = silu(y[t][i]) * y[t][I + i], silu(z) = z / (1 + exp(-z)), double.                  */
ORC_API void orc_silu_glu(const double* y, int64_t T, int64_t I, double* h) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t i = 0; i < I; ++i) {
      double z = y[t * 2 * I + i];
      double u = y[t * 2 * I + I + i];
      h[t * I + i] = z / (1.0 + exp(-z)) * u;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* The whole projection, step by step: RMSNorm -> int8 activations -> absmean ternary weights   */
/* -> ternary accumulation -> dequantisation (-> SiLU-GLU when glu != 0, N = 2I, out is T x I). */
/* Returns beta.  out is T x N (or T x N/2) doubles.                                            */
ORC_API float orc_bitlinear_forward(const float* x, int64_t T, int64_t K, const float* g,
                                    float eps, const float* W, int64_t N, int glu, double* out) {
  int8_t* q = (int8_t*)malloc((size_t)(T * K));
  float* gamma = (float*)malloc(sizeof(float) * (size_t)T);
  int8_t* c = (int8_t*)malloc((size_t)(N * K));
  int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * N));
  double* y = glu ? (double*)malloc(sizeof(double) * (size_t)(T * N)) : out;
  orc_rmsnorm_actquant(x, T, K, g, eps, q, gamma, NULL);
  float beta = orc_absmean_beta(W, N * K);
  orc_ternary_codes(W, N * K, beta, c);
  orc_ternary_accumulate(q, T, K, c, N, acc);
  orc_dequant(acc, T, N, gamma, beta, y);
  if (glu) {
    orc_silu_glu(y, T, N / 2, out);
    free(y);
  }
  free(q);
  free(gamma);
  free(c);
  free(acc);
  return beta;
}

/* ------------------------------------------------------------------------------------------ */
/* MLGRU recurrence ([P4] "Kernkomponenten: MLGRU und GLU", the MLGRU paragraph).  The pages    */
/* describe it in words only: token by token, gates with values in (0, 1) weigh the previous    */
/* hidden state against the current token, element-wise.  Reading taken: the forget gate       */
/* f = sigmoid(F) keeps that share of the previous state and the rest, 1 - f, comes from the    */
/* token's candidate c = silu(I):                                                                */
/*     h_t = f_t * h_{t-1} + (1 - f_t) * c_t,    h_{-1} = h0 (zero when h0 is NULL).            */
/* I, F: [T x H] row-major (the i_proj and f_proj outputs of T tokens).  h: [T x H], the state   */
/* after each token.  hT: [H], the state after the last token (may be NULL).  Double throughout. */
ORC_API void orc_mlgru_scan(const double* I, const double* F, int64_t T, int64_t H,
                            const double* h0, double* h, double* hT) {
  for (int64_t j = 0; j < H; ++j) {
    double s = h0 ? h0[j] : 0.0;
    for (int64_t t = 0; t < T; ++t) {
      double f = 1.0 / (1.0 + exp(-F[t * H + j]));
      double z = I[t * H + j];
      double c = z / (1.0 + exp(-z));
      s = f * s + (1.0 - f) * c;
      h[t * H + j] = s;
    }
    if (hT) hT[j] = s;
  }
}

/* FusedRMSNormSwishGate ([P1] "HGRNBit という層構成を読む": the gate of the attention side, ahead */
/* of o_proj).  Reading taken: an RMSNorm of the state over its H channels, scaled by the norm   */
/* weight w (1 when NULL), times the swish (SiLU) of the g_proj output:                          */
/*     o_tj = h_tj / sqrt(mean_j h_tj^2 + eps) * w_j * silu(G_tj).                              */
/* h, G, o: [T x H] row-major.  Double throughout.                                               */
ORC_API void orc_swish_gate_norm(const double* h, const double* G, int64_t T, int64_t H,
                                 const double* w, double eps, double* o) {
  for (int64_t t = 0; t < T; ++t) {
    const double* hr = h + t * H;
    double ss = 0.0;
    for (int64_t j = 0; j < H; ++j) ss += hr[j] * hr[j];
    double r = sqrt(ss / (double)H + eps);
    for (int64_t j = 0; j < H; ++j) {
      double g = G[t * H + j];
      double sg = g / (1.0 + exp(-g));
      o[t * H + j] = hr[j] / r * (w ? w[j] : 1.0) * sg;
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* FusedBitLinear backward.  The pages print no backward pass.  [P4] "MatMul durch ternäre      */
/* Operationen ersetzen" says the weights are trained in full precision and mapped to ternary   */
/* values by absmean quantisation during training: the quantisers sit inside the training       */
/* forward pass.  Reading taken (straight-through): rounding and clamping in both quantisers    */
/* pass the gradient unchanged, so the layer is differentiated as the bilinear map of its       */
/* dequantised operands after the RMSNorm,                                                      */
/*     y_tn  = sum_k xq_tk * wq_nk,   xq_tk = q_tk * gamma_t / 127,   wq_nk = c_nk * beta,      */
/*     xhat_tk = x_tk / r_t * g_k,    r_t = sqrt(mean_k x_tk^2 + eps),                          */
/* where the latent full-precision weight receives the gradient of wq and the quantiser's input */
/* xhat receives the gradient of xq.  In reverse order of the forward pass:                     */
/*     dW_nk  = sum_t dy_tn * xq_tk                                                              */
/*     dxh_tk = sum_n dy_tn * wq_nk                                                              */
/*     dx_tk  = g_k * dxh_tk / r_t - x_tk / (K r_t^3) * sum_j g_j * dxh_tj * x_tj               */
/*     dg_k   = sum_t dxh_tk * x_tk / r_t                                                        */
/* x: [T x K]; g: [K] or NULL (all ones); q [T x K] and gamma [T]: the forward pass's codes and */
/* scales; c: [N x K] weight codes, beta their scale; dy: [T x N], the gradient of y.  Outputs: */
/* dx [T x K], dW [N x K], dg [K] (skipped when NULL).  Double throughout.                      */
ORC_API void orc_bitlinear_backward(const double* x, int64_t T, int64_t K, const double* g,
                                    double eps, const int8_t* q, const float* gamma,
                                    const int8_t* c, float beta, int64_t N, const double* dy,
                                    double* dx, double* dW, double* dg) {
  double* dxh = (double*)malloc(sizeof(double) * (size_t)K);
  for (int64_t i = 0; i < N * K; ++i) dW[i] = 0.0;
  if (dg)
    for (int64_t k = 0; k < K; ++k) dg[k] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    const double a = (double)gamma[t] / 127.0;
    /* weights: every output n of this token adds dy_tn times the token's dequantised codes */
    for (int64_t n = 0; n < N; ++n) {
      const double d = dy[t * N + n];
      for (int64_t k = 0; k < K; ++k) dW[n * K + k] += d * ((double)q[t * K + k] * a);
    }
    /* through the activation quantiser: the gradient of the dequantised codes (each dxh[k]
       sums its terms in ascending n; the loops run n-outer only to read c row by row) */
    for (int64_t k = 0; k < K; ++k) dxh[k] = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const double d = dy[t * N + n];
      for (int64_t k = 0; k < K; ++k) dxh[k] += d * ((double)c[n * K + k] * (double)beta);
    }
    /* through the RMSNorm */
    double ss = 0.0, dot = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      const double xv = x[t * K + k];
      ss += xv * xv;
      dot += (g ? g[k] : 1.0) * dxh[k] * xv;
    }
    const double r = sqrt(ss / (double)K + eps);
    for (int64_t k = 0; k < K; ++k) {
      const double xv = x[t * K + k];
      dx[t * K + k] = (g ? g[k] : 1.0) * dxh[k] / r - xv * dot / ((double)K * r * r * r);
      if (dg) dg[k] += dxh[k] * xv / r;
    }
  }
  free(dxh);
}
