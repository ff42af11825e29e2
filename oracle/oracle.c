/*
 * Plain CPU oracle for the fused low-bit linear of SteerQuant's Rudder kernels.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the CPU
 * baseline of the benchmark; never by the product path.  Independent of the
 * CUDA library: no shared code, headers, helpers or tables.
 *
 * Every function follows the definition in the order the paper states it, with
 * plain nested loops and no blocking, fusion or reordering.  Compile with
 * -O2 -ffp-contract=off and without -ffast-math so every float operation is a
 * single IEEE-754 binary32 operation rounded to nearest-even (x86-64 SSE).
 *
 * Citations are to "SteerQuant: Steering Quantization Error with Action-Guided
 * Scaling in World-Action Models" (paperlayer.ai abstract page 2609.39056v1).
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EBADARG (-1)
#define ORACLE_ENONFINITE (-2)
#define ORACLE_EOVERFLOW (-3)
#define ORACLE_ENOMEM (-4)

/* bf16 is the upper half of a binary32 pattern, so widening is exact. */
float oracle_bf16_to_float(uint16_t b) {
  uint32_t bits = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return f;
}

/* Round a double once to bf16 (8 significant bits), ties to even.  Going
 * double -> float -> bf16 could round twice, so the rounding is done directly:
 * scale the magnitude so the kept bits sit left of the binary point, round to
 * an integer with nearbyint (current mode: nearest-even), scale back. */
uint16_t oracle_double_to_bf16(double v) {
  if (isnan(v)) return (uint16_t)0x7FC0;
  uint16_t sign = signbit(v) ? (uint16_t)0x8000 : (uint16_t)0;
  double a = fabs(v);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80);
  int e;
  (void)frexp(a, &e); /* a = f * 2^e with f in [0.5, 1) */
  if (e < -125) e = -125; /* below the smallest normal 2^-126: fixed quantum 2^-133 */
  double r = nearbyint(ldexp(a, 8 - e));
  double mag = ldexp(r, e - 8);
  if (mag > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80); /* past bf16 max */
  float f32 = (float)mag; /* exact: at most 9 significant bits */
  uint32_t bits;
  memcpy(&bits, &f32, sizeof bits);
  return (uint16_t)(sign | (uint16_t)(bits >> 16));
}

/* §3.1: symmetric k-bit code of one value, given its scale.  The quotient is a
 * binary32 IEEE division, rounded to an integer half-to-even (rintf under the
 * default rounding mode) and clamped to [-qmax, qmax].  A zero scale gives 0. */
static int quantize_value(float v, float s, float qmax) {
  if (s == 0.0f) return 0;
  float t = v / s;
  float r = rintf(t);
  if (r > qmax) r = qmax;
  if (r < -qmax) r = -qmax;
  return (int)r;
}

static uint8_t pack_pair(int lo, int hi) {
  return (uint8_t)(((unsigned)lo & 0xFu) | (((unsigned)hi & 0xFu) << 4));
}

static int unpack_nibble(uint8_t byte, int high) {
  int v = high ? (byte >> 4) & 0xF : byte & 0xF;
  return v >= 8 ? v - 16 : v;
}

/* §4.2, calibration side: the shared positive diagonal, in SmoothQuant's
 * equivalent-scaling form (the paper's §2 cites it): c[k] = sqrt(a_k / b_k) with
 * a_k = max_m |x_cal[m,k]| and b_k = max_n |W[n,k]|; c = 1 where either is 0. */
int oracle_channel_scale(const uint16_t* x_cal, int Mcal, const uint16_t* W, int N,
                         int K, float* c, float* cinv) {
  if (!x_cal || !W || !c || !cinv || Mcal < 1 || N < 1 || K < 1) return ORACLE_EBADARG;
  for (int k = 0; k < K; ++k) {
    float a = 0.0f, b = 0.0f;
    for (int m = 0; m < Mcal; ++m) {
      float v = fabsf(oracle_bf16_to_float(x_cal[(size_t)m * K + k]));
      if (!isfinite(v)) return ORACLE_ENONFINITE;
      if (v > a) a = v;
    }
    for (int n = 0; n < N; ++n) {
      float v = fabsf(oracle_bf16_to_float(W[(size_t)n * K + k]));
      if (!isfinite(v)) return ORACLE_ENONFINITE;
      if (v > b) b = v;
    }
    float ck = 1.0f;
    if (a > 0.0f && b > 0.0f) ck = sqrtf(a / b);
    if (!isfinite(ck) || ck <= 0.0f) return ORACLE_ENONFINITE;
    c[k] = ck;
    cinv[k] = 1.0f / ck;
  }
  return 0;
}

/* Figure 2 (offline weight preparation) with §4.2 and §3.1: one static int4
 * matrix per layer.  For each output channel n: w'_k = W[n,k]*c[k];
 * s_w[n] = max_k |w'_k| / 7; code = clamp(rint(w'_k / s_w[n]), -7, 7). */
int oracle_pack_int4(const uint16_t* W, const float* c, int N, int K, uint8_t* qw,
                     float* s_w) {
  if (!W || !qw || !s_w || N < 1 || K < 2 || (K % 2) != 0) return ORACLE_EBADARG;
  float* wp = (float*)malloc(sizeof(float) * (size_t)K);
  if (!wp) return ORACLE_ENOMEM;
  const float qmax = 7.0f;
  for (int n = 0; n < N; ++n) {
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      float ck = c ? c[k] : 1.0f;
      wp[k] = oracle_bf16_to_float(W[(size_t)n * K + k]) * ck;
      if (!isfinite(wp[k])) { free(wp); return ORACLE_ENONFINITE; }
      float a = fabsf(wp[k]);
      if (a > amax) amax = a;
    }
    float s = amax / qmax;
    s_w[n] = s;
    for (int k = 0; k < K; k += 2) {
      int lo = quantize_value(wp[k], s, qmax);
      int hi = quantize_value(wp[k + 1], s, qmax);
      qw[(size_t)n * (K / 2) + k / 2] = pack_pair(lo, hi);
    }
  }
  free(wp);
  return 0;
}

/* §4.4 first kernel, with §4.2 and §4.3 folded in.  For token row m with stream
 * sid = stream_id[m]:
 *   x'_k  = x[m,k] * cinv[k]                       (§4.2: activations scaled down)
 *   amax  = max_k |x'_k|
 *   clip  = alpha[step][sid] * amax                 (§4.3: table row (step, stream))
 *   s     = clip / qmax                             (qmax 127 or 7, App. D)
 *   q_k   = clamp(rint(x'_k / s), -qmax, qmax)      (§3.1: symmetric)
 * Codes for 4-bit activations are packed two per byte (low nibble = even k). */
int oracle_act_quant(const uint16_t* x, int M, int K, const float* cinv,
                     const uint8_t* stream_id, const float* alpha, int S, int T,
                     int step, int act_bits, void* qx, float* s_tok) {
  if (!x || !stream_id || !alpha || !qx || !s_tok) return ORACLE_EBADARG;
  if (M < 0 || K < 2 || (K % 2) != 0 || S < 1 || T < 1 || step < 0 || step >= T)
    return ORACLE_EBADARG;
  if (act_bits != 8 && act_bits != 4) return ORACLE_EBADARG;
  const float qmax = act_bits == 8 ? 127.0f : 7.0f;
  float* xp = (float*)malloc(sizeof(float) * (size_t)K);
  if (!xp) return ORACLE_ENOMEM;
  for (int m = 0; m < M; ++m) {
    int sid = stream_id[m];
    if (sid >= S) { free(xp); return ORACLE_EBADARG; }
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      float ck = cinv ? cinv[k] : 1.0f;
      xp[k] = oracle_bf16_to_float(x[(size_t)m * K + k]) * ck;
      if (!isfinite(xp[k])) { free(xp); return ORACLE_ENONFINITE; }
      float a = fabsf(xp[k]);
      if (a > amax) amax = a;
    }
    float clip = alpha[(size_t)step * S + sid] * amax;
    float s = clip / qmax;
    s_tok[m] = s;
    if (act_bits == 8) {
      int8_t* row = (int8_t*)qx + (size_t)m * K;
      for (int k = 0; k < K; ++k) row[k] = (int8_t)quantize_value(xp[k], s, qmax);
    } else {
      uint8_t* row = (uint8_t*)qx + (size_t)m * (K / 2);
      for (int k = 0; k < K; k += 2)
        row[k / 2] = pack_pair(quantize_value(xp[k], s, qmax),
                               quantize_value(xp[k + 1], s, qmax));
    }
  }
  free(xp);
  return 0;
}

/* §4.3 read as static clipping (the layer-step table holds one shared clip
 * threshold per step and a bounded gain per stream): the token's stream gain g
 * narrows the threshold thr to clip = thr / g, the scale is clip / qmax, and the
 * code is the nearest integer to x'/s clamped to +-qmax; the inverse gain stays
 * inside the scale that the epilogue multiplies back (§4.4).  No row maximum is
 * involved.  thr [T]; gain [T][S]. */
int oracle_act_quant_static(const uint16_t* x, int M, int K, const float* cinv,
                            const uint8_t* stream_id, const float* thr, const float* gain,
                            int S, int T, int step, int act_bits, void* qx, float* s_tok) {
  if (!x || !stream_id || !thr || !gain || !qx || !s_tok) return ORACLE_EBADARG;
  if (M < 0 || K < 2 || (K % 2) != 0 || S < 1 || T < 1 || step < 0 || step >= T)
    return ORACLE_EBADARG;
  if (act_bits != 8 && act_bits != 4) return ORACLE_EBADARG;
  const float qmax = act_bits == 8 ? 127.0f : 7.0f;
  float* xp = (float*)malloc(sizeof(float) * (size_t)K);
  if (!xp) return ORACLE_ENOMEM;
  for (int m = 0; m < M; ++m) {
    int sid = stream_id[m];
    if (sid >= S) { free(xp); return ORACLE_EBADARG; }
    for (int k = 0; k < K; ++k) {
      float ck = cinv ? cinv[k] : 1.0f;
      xp[k] = ck * oracle_bf16_to_float(x[(size_t)m * K + k]);
      if (!isfinite(xp[k])) { free(xp); return ORACLE_ENONFINITE; }
    }
    float g = gain[(size_t)step * S + sid];
    float clip = g > 0.0f ? thr[step] / g : 0.0f;
    float s = clip / qmax;
    s_tok[m] = s;
    if (act_bits == 8) {
      int8_t* row = (int8_t*)qx + (size_t)m * K;
      for (int k = 0; k < K; ++k) row[k] = (int8_t)quantize_value(xp[k], s, qmax);
    } else {
      uint8_t* row = (uint8_t*)qx + (size_t)m * (K / 2);
      for (int k = 0; k < K; k += 2)
        row[k / 2] = pack_pair(quantize_value(xp[k], s, qmax),
                               quantize_value(xp[k + 1], s, qmax));
    }
  }
  free(xp);
  return 0;
}

static int act_code(const void* qx, int act_bits, int K, int m, int k) {
  if (act_bits == 8) return ((const int8_t*)qx)[(size_t)m * K + k];
  uint8_t b = ((const uint8_t*)qx)[(size_t)m * (K / 2) + k / 2];
  return unpack_nibble(b, k & 1);
}

/* §4.4 second kernel, integer part: acc[m,n] = sum_k q[m,k] * qw[n,k], summed in
 * 64-bit and required to fit int32. */
int oracle_gemm_s32(const void* qx, int act_bits, const uint8_t* qw, int M, int N,
                    int K, int32_t* acc) {
  if (!qx || !qw || !acc || M < 0 || N < 1 || K < 2 || (K % 2) != 0) return ORACLE_EBADARG;
  if (act_bits != 8 && act_bits != 4) return ORACLE_EBADARG;
  for (int m = 0; m < M; ++m) {
    for (int n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int k = 0; k < K; ++k) {
        int w = unpack_nibble(qw[(size_t)n * (K / 2) + k / 2], k & 1);
        sum += (int64_t)act_code(qx, act_bits, K, m, k) * (int64_t)w;
      }
      if (sum > INT32_MAX || sum < INT32_MIN) return ORACLE_EOVERFLOW;
      acc[(size_t)m * N + n] = (int32_t)sum;
    }
  }
  return 0;
}

/* §4.4 second kernel, epilogue: dequantization (s_tok * s_w), bias, and the
 * output compensation beta of table row (step, stream), then one bf16 rounding.
 * The inverse stream gain is already inside s_tok (the clip ratio is 1/gain). */
int oracle_epilogue(const int32_t* acc, const float* s_tok, const float* s_w,
                    const float* bias, const float* beta, const uint8_t* stream_id,
                    int M, int N, int S, int T, int step, uint16_t* y) {
  if (!acc || !s_tok || !s_w || !stream_id || !y || M < 0 || N < 1 || S < 1 || T < 1 ||
      step < 0 || step >= T)
    return ORACLE_EBADARG;
  for (int m = 0; m < M; ++m) {
    int sid = stream_id[m];
    if (sid >= S) return ORACLE_EBADARG;
    for (int n = 0; n < N; ++n) {
      double v = (double)s_tok[m] * (double)s_w[n] * (double)acc[(size_t)m * N + n];
      if (bias) v += (double)bias[n];
      if (beta) v += (double)beta[((size_t)step * S + sid) * N + n];
      y[(size_t)m * N + n] = oracle_double_to_bf16(v);
    }
  }
  return 0;
}

int oracle_linear(const uint16_t* x, int M, int K, int N, const float* cinv,
                  const uint8_t* stream_id, const float* alpha, const float* beta,
                  int S, int T, int step, int act_bits, const uint8_t* qw,
                  const float* s_w, const float* bias, uint16_t* y, void* qx_out,
                  float* s_tok_out, int32_t* acc_out) {
  if (!y || (act_bits != 8 && act_bits != 4) || M < 0 || N < 1 || K < 2) return ORACLE_EBADARG;
  size_t qbytes = act_bits == 8 ? (size_t)M * K : (size_t)M * (K / 2);
  void* qx = qx_out ? qx_out : malloc(qbytes ? qbytes : 1);
  float* s_tok = s_tok_out ? s_tok_out : (float*)malloc(sizeof(float) * (size_t)(M ? M : 1));
  int32_t* acc = acc_out ? acc_out : (int32_t*)malloc(sizeof(int32_t) * ((size_t)M * N + 1));
  int rc = ORACLE_ENOMEM;
  if (qx && s_tok && acc) {
    rc = oracle_act_quant(x, M, K, cinv, stream_id, alpha, S, T, step, act_bits, qx, s_tok);
    if (rc == 0) rc = oracle_gemm_s32(qx, act_bits, qw, M, N, K, acc);
    if (rc == 0)
      rc = oracle_epilogue(acc, s_tok, s_w, bias, beta, stream_id, M, N, S, T, step, y);
  }
  if (!qx_out) free(qx);
  if (!s_tok_out) free(s_tok);
  if (!acc_out) free(acc);
  return rc;
}

/* App. D (GELU in BF16): GELU(v) = v * Phi(v) with Phi(v) = 0.5 * erfc(-v / sqrt(2)),
 * in fp64; the bf16 result is rounded once from that value. */
double oracle_gelu(double v) { return v * 0.5 * erfc(-v / sqrt(2.0)); }

int oracle_gelu_bf16(const uint16_t* v, size_t n, uint16_t* h) {
  if (n > 0 && (!v || !h)) return ORACLE_EBADARG;
  for (size_t i = 0; i < n; ++i) {
    double a = (double)oracle_bf16_to_float(v[i]);
    if (!isfinite(a)) return ORACLE_ENONFINITE;
    h[i] = oracle_double_to_bf16(oracle_gelu(a));
  }
  return 0;
}
