/*
 * Plain CPU oracle for the fused low-bit linear of SteerQuant's Rudder kernels.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this code: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header or constant table with the
 * CUDA library.
 *
 * Source: "SteerQuant: Steering Quantization Error with Action-Guided Scaling
 * in World-Action Models" (paperlayer.ai abstract page 2609.39056v1):
 *   §3.1 WAM Quantization      symmetric k-bit quantization of weights and activations
 *   §4.2 Shared-Weight Error Routing   shared positive diagonal D_l: weights scaled up,
 *                                      activations scaled down by the same diagonal
 *   §4.3 Stream-Specific Activation Modulation  per-(layer, step) clip and stream
 *                                      gains kept in a layer-step lookup table
 *   §4.4 Rudder                scaling and gains applied during activation
 *                              quantization; low-bit GEMM with dequantization,
 *                              inverse-gain compensation and bias; only integer
 *                              activations and row scales pass between kernels
 *   Figure 2                   offline weight preparation; token-wise stream gains
 *   App. D "Quantization"      4-bit weights, 8- or 4-bit activations
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - quantization arithmetic is fp32 with round-half-to-even and clamp to +-qmax
 *     (qmax = 127 for 8-bit, 7 for 4-bit); the scale is s = (alpha*amax)/qmax and
 *     the code is rint(x'/s) computed with an IEEE division;
 *   - the stream gain enters as a clip ratio alpha = 1/gain read from the table
 *     row (step, stream); the inverse-gain compensation is then carried inside the
 *     per-token scale;
 *   - output compensation is an additive fp32 vector beta[step][stream][n];
 *   - the dequantize/bias/compensation epilogue is evaluated in fp64 here (the
 *     pages fix no precision for it) and rounded once to bf16 (round-half-even);
 *   - a row (or weight row) whose scale is 0 gets scale 0 and all-zero codes;
 *   - packed int4: two's-complement nibbles, the low nibble holds the even k;
 *   - channel scale c[k] = sqrt(max_m|x_cal[m,k]| / max_n|W[n,k]|) in fp32
 *     (SmoothQuant-style equivalent scaling, cited in the paper's §2), c = 1 when
 *     either maximum is 0; cinv = 1/c.
 *
 * bf16 values are passed as their raw 16-bit patterns (uint16_t).
 * All functions return 0 on success and a negative value on a bad argument.
 */
#ifndef WQ_ORACLE_H
#define WQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* §4.2 (calibration side): c[k], cinv[k] from a calibration batch x_cal [Mcal][K]
 * and the bf16 weight W [N][K]. */
int oracle_channel_scale(const uint16_t* x_cal, int Mcal, const uint16_t* W, int N,
                         int K, float* c, float* cinv);

/* Figure 2 / §4.2 / §3.1: offline weight preparation.  W' = W*c (c may be NULL,
 * meaning 1), per-output-channel symmetric int4 codes, packed [N][K/2]; s_w [N]. */
int oracle_pack_int4(const uint16_t* W, const float* c, int N, int K, uint8_t* qw,
                     float* s_w);

/* §4.3 read as static clipping: one shared clip threshold thr[step] per layer
 * step and a bounded gain per stream, gain [T][S]; clip = thr[step] / gain (0 when
 * the gain is not positive), s = clip / qmax, codes as in oracle_act_quant.
 * Same layouts as oracle_act_quant. */
int oracle_act_quant_static(const uint16_t* x, int M, int K, const float* cinv,
                            const uint8_t* stream_id, const float* thr, const float* gain,
                            int S, int T, int step, int act_bits, void* qx, float* s_tok);

/* §4.4 first kernel (with §4.3 and §4.2 folded in): per-token quantization.
 * x [M][K] bf16; cinv [K] or NULL (=1); stream_id [M]; alpha [T][S] clip ratios;
 * act_bits 8 -> qx int8 [M][K]; act_bits 4 -> qx packed uint8 [M][K/2].
 * s_tok [M] receives the per-token scale. */
int oracle_act_quant(const uint16_t* x, int M, int K, const float* cinv,
                     const uint8_t* stream_id, const float* alpha, int S, int T,
                     int step, int act_bits, void* qx, float* s_tok);

/* §4.4 second kernel, integer part: acc[m][n] = sum_k q[m][k]*qw[n][k] (int32). */
int oracle_gemm_s32(const void* qx, int act_bits, const uint8_t* qw, int M, int N,
                    int K, int32_t* acc);

/* §4.4 second kernel, epilogue: y = bf16(s_tok[m]*s_w[n]*acc + bias[n]
 * + beta[step][sid][n]) evaluated in fp64.  bias and beta may be NULL. */
int oracle_epilogue(const int32_t* acc, const float* s_tok, const float* s_w,
                    const float* bias, const float* beta, const uint8_t* stream_id,
                    int M, int N, int S, int T, int step, uint16_t* y);

/* The whole linear: act_quant -> gemm_s32 -> epilogue.  Optional outputs
 * (qx, s_tok, acc) may be NULL; scratch is allocated internally. */
int oracle_linear(const uint16_t* x, int M, int K, int N, const float* cinv,
                  const uint8_t* stream_id, const float* alpha, const float* beta,
                  int S, int T, int step, int act_bits, const uint8_t* qw,
                  const float* s_w, const float* bias, uint16_t* y, void* qx_out,
                  float* s_tok_out, int32_t* acc_out);

/* App. D keeps GELU in BF16 between the FFN up- and down-projections; fusing the
 * down-projection's activation quantization into the up-projection's epilogue is
 * an extension of the pages' two-kernel split.  GELU is read as the exact form
 * GELU(v) = v * Phi(v), Phi the standard normal distribution function, evaluated
 * in fp64 as v * 0.5 * erfc(-v / sqrt(2)) (erfc keeps Phi accurate for negative v).
 * oracle_gelu_bf16: h[i] = bf16(GELU(v[i])) for bf16 inputs v [n], one rounding
 * (half to even).  Non-finite inputs are rejected. */
double oracle_gelu(double v);
int oracle_gelu_bf16(const uint16_t* v, size_t n, uint16_t* h);

/* Helpers exposed for the pin tests. */
float oracle_bf16_to_float(uint16_t b);
uint16_t oracle_double_to_bf16(double v);

#ifdef __cplusplus
}
#endif

#endif /* WQ_ORACLE_H */
