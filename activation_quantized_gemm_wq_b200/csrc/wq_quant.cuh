// Quantization kernels of the fused low-bit linear (SteerQuant / Rudder):
//   act_quant     the first Rudder kernel (SteerQuant §4.4): per-token quantization
//                 with the shared channel scale (§4.2) and the per-(step, stream)
//                 clip ratio from the layer-step table (§4.3) folded in
//   pack_int4     offline weight preparation (Figure 2): W' = W * c, one symmetric
//                 int4 code matrix with per-output-channel scales
//   channel_scale the shared diagonal c[k] = sqrt(max|x_cal[:,k]| / max|W[:,k]|)
//                 (SmoothQuant-style equivalent scaling, cited in §2)
//
// All arithmetic that decides a code is IEEE binary32 with round-to-nearest-even:
// explicit __fmul_rn / __fdiv_rn / __fsqrt_rn intrinsics, no contraction, no
// fast-math, so codes and scales are reproducible bit for bit.
#pragma once
#include <cuda_bf16.h>

#include "wq_internal.h"
#include "wq_ptx.cuh"

namespace wq {
namespace {

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int QMAX>
__device__ __forceinline__ int quantize(float v, float s) {
  if (s == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(v, s));  // saturating convert, ties to even
  q = q > QMAX ? QMAX : q;
  q = q < -QMAX ? -QMAX : q;
  return q;
}

// Exact code through the IEEE quotient; kept out of line so the rare near-tie
// path below stays a real branch instead of being computed for every element.
template <int QMAX>
__device__ __noinline__ int quantize_exact(float v, float s) {
  return quantize<QMAX>(v, s);
}

// Adding 1.5 * 2^23 to a float of magnitude below 2^22 rounds it to an integer
// (the addition's own round-half-to-even), and that integer sits in the low
// bits of the sum's bit pattern, two's complement for negative values.
constexpr float kRoundMagic = 12582912.0f;

// Eight codes from the correctly rounded reciprocal r = 1/s (s > 0, r finite),
// identical to quantize<QMAX>(v[e], s) for every input.  t = v*r lies within
// |t|*2^-22 of the IEEE quotient fl(v/s) (three roundings of at most 2^-24
// each), i.e. within 2^-12 while |t| <= 2^10.  Two values that close round to
// different integers only if a half-integer lies between them, so whenever t is
// farther than 2^-12 from every half-integer, the rounding of t is the rounding
// of fl(v/s); beyond |t| = 2^10 both clamp to the same end of the range.  The few
// other elements take the exact quotient.  Each result's low byte is the code.
template <int QMAX>
__device__ __forceinline__ void quantize8_recip(const float (&v)[8], float s, float r,
                                                uint32_t (&c)[8]) {
  constexpr float lo = kRoundMagic - static_cast<float>(QMAX);
  constexpr float hi = kRoundMagic + static_cast<float>(QMAX);
  bool near_tie = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float t = __fmul_rn(v[e], r);
    const float u = __fadd_rn(t, kRoundMagic);                 // kRoundMagic + rint(t)
    const float d = __fsub_rn(t, __fsub_rn(u, kRoundMagic));   // t - rint(t), exact
    near_tie = near_tie || fabsf(d) >= 0.5f - 0x1p-12f;
    c[e] = __float_as_uint(fminf(fmaxf(u, lo), hi));           // clamp to +-QMAX
  }
  if (near_tie) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float t = __fmul_rn(v[e], r);
      const float u = __fadd_rn(t, kRoundMagic);
      const float d = __fsub_rn(t, __fsub_rn(u, kRoundMagic));
      if (fabsf(d) >= 0.5f - 0x1p-12f) c[e] = static_cast<uint32_t>(quantize_exact<QMAX>(v[e], s));
    }
  }
}

// One code from the reciprocal, as quantize8_recip does for eight: identical to
// quantize<QMAX>(v, s) for every input (s > 0, r = 1/s finite).  The result's low
// byte is the code.
template <int QMAX>
__device__ __forceinline__ uint32_t quantize1_recip(float v, float s, float r) {
  const float t = __fmul_rn(v, r);
  const float u = __fadd_rn(t, kRoundMagic);
  const float d = __fsub_rn(t, __fsub_rn(u, kRoundMagic));
  if (fabsf(d) >= 0.5f - 0x1p-12f) return static_cast<uint32_t>(quantize_exact<QMAX>(v, s));
  return __float_as_uint(fminf(fmaxf(u, kRoundMagic - static_cast<float>(QMAX)),
                               kRoundMagic + static_cast<float>(QMAX)));
}

// GELU(v) = v * Phi(v), Phi the standard normal distribution function, written
// as Phi(v) = erfc(-v / sqrt(2)) / 2 so that it stays accurate for negative v;
// fp32 with CUDA's erfcf.
__device__ __forceinline__ float gelu_f32(float v) {
  return __fmul_rn(__fmul_rn(v, 0.5f), erfcf(__fmul_rn(v, -0.70710678118654752f)));
}

// Low bytes of four words -> one word.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c,
                                                   uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Low nibbles of eight words -> one word, code 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t pack_low_nibbles(const uint32_t (&c)[8]) {
  uint32_t n = pack_low_bytes(c[0], c[1], c[2], c[3]) & 0x0F0F0F0Fu;
  uint32_t m = pack_low_bytes(c[4], c[5], c[6], c[7]) & 0x0F0F0F0Fu;
  n |= n >> 4;  // bytes 0 and 2 now hold (c0 | c1 << 4) and (c2 | c3 << 4)
  m |= m >> 4;
  return __byte_perm(n, m, 0x6420);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// cinv chunk c from the CTA's shared-memory copy (8 floats).
__device__ __forceinline__ void load_cinv8(const float* cinv_s, int c, float (&ci)[8]) {
  const float4 a = reinterpret_cast<const float4*>(cinv_s)[2 * c];
  const float4 b = reinterpret_cast<const float4*>(cinv_s)[2 * c + 1];
  ci[0] = a.x; ci[1] = a.y; ci[2] = a.z; ci[3] = a.w;
  ci[4] = b.x; ci[5] = b.y; ci[6] = b.z; ci[7] = b.w;
}

// cinv chunk c through L1, or all ones when there is no channel scale.
__device__ __forceinline__ void load_cinv8_global(const float* cinv, int c, float (&ci)[8]) {
  if (cinv == nullptr) {
#pragma unroll
    for (int e = 0; e < 8; ++e) ci[e] = 1.0f;
    return;
  }
  const float4 a = __ldg(reinterpret_cast<const float4*>(cinv) + 2 * c);
  const float4 b = __ldg(reinterpret_cast<const float4*>(cinv) + 2 * c + 1);
  ci[0] = a.x; ci[1] = a.y; ci[2] = a.z; ci[3] = a.w;
  ci[4] = b.x; ci[5] = b.y; ci[6] = b.z; ci[7] = b.w;
}

// x' = x * cinv for one chunk of 8 channels (bf16 widening is exact).
__device__ __forceinline__ void scale8(const uint4 raw, const float (&ci)[8], float (&v)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = __fmul_rn(bf16lo(w[e]), ci[2 * e]);
    v[2 * e + 1] = __fmul_rn(bf16hi(w[e]), ci[2 * e + 1]);
  }
}

// x' = x * cinv for one chunk of 8 channels as four value pairs (packed fp32x2
// multiplies: the same IEEE products as scale8).
__device__ __forceinline__ void scale8_pairs(const uint4 raw, const float* cinv_s, int c,
                                             float2 (&v)[4]) {
  const float4 a = reinterpret_cast<const float4*>(cinv_s)[2 * c];
  const float4 b = reinterpret_cast<const float4*>(cinv_s)[2 * c + 1];
  const float2 ci[4] = {make_float2(a.x, a.y), make_float2(a.z, a.w), make_float2(b.x, b.y),
                        make_float2(b.z, b.w)};
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] = __fmul2_rn(make_float2(bf16lo(w[e]), bf16hi(w[e])), ci[e]);
}

template <int QMAX, int GW>
__device__ __forceinline__ uint2 codes_packed(const float2 (&v)[GW / 2], float s, float r,
                                              bool narrow);

// Persistent CTAs; each pass handles RPC token rows, one row per TPR threads.
// cinv is copied to shared memory once per CTA.  Each thread loads its CPT
// chunks of 8 channels (128-bit loads, all issued before any use, so x is read
// from HBM once with CPT loads in flight per thread), then forms x * cinv twice:
// once for the row maximum and once for the codes, which keeps register use low;
// both in packed fp32x2 arithmetic, the codes two at a time (codes_packed).
// STORE_BITS: 8 writes one code per int8 byte (the int4 codes too, for the fused
// linear's workspace), 4 packs two int4 codes per byte (low nibble = even k).
// STATIC: the clip comes from the layer-step table alone (§4.3 read as a shared
// threshold thr[step] narrowed by the stream gain, clip = thr / gain, with `alpha`
// holding the gains [T][S]); no row maximum, so x is scaled and quantized once.
template <int ACT_BITS, int STORE_BITS, int TPR, int CPT, bool STATIC>
__global__ void __launch_bounds__(256) act_quant_kernel(
    const uint16_t* __restrict__ x, int M, int K, const float* __restrict__ cinv,
    const uint8_t* __restrict__ stream_id, const float* __restrict__ alpha,
    const float* __restrict__ thr, int S, int step, void* __restrict__ qx,
    float* __restrict__ s_tok, uint4* __restrict__ zero, size_t zero_n16) {
  constexpr int RPC = 256 / TPR;  // rows per CTA pass
  constexpr int WPR = TPR / 32;   // warps per row
  constexpr int QMAX = ACT_BITS == 8 ? 127 : 7;
  extern __shared__ float4 cinv_s4[];
  float* cinv_s = reinterpret_cast<float*>(cinv_s4);
  __shared__ float red[8];

  // Everything this kernel reads or writes may belong to the previous kernel in
  // the stream; once that has finished, the GEMM that follows may start its
  // prologue (and its weight loads) while this one runs.
  griddep_wait();
  griddep_launch_dependents();
  // Clear the next GEMM's split-K accumulators and counters (16-byte words) here
  // rather than in a separate launch.
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < zero_n16; i += (size_t)gridDim.x * 256)
    zero[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int k = threadIdx.x * 4; k < K; k += 256 * 4)
    *reinterpret_cast<float4*>(cinv_s + k) =
        cinv ? __ldg(reinterpret_cast<const float4*>(cinv + k)) : make_float4(1.f, 1.f, 1.f, 1.f);
  __syncthreads();

  const int local_row = threadIdx.x / TPR;
  const int t = threadIdx.x % TPR;
  const int nchunk = K >> 3;
  const int groups = (M + RPC - 1) / RPC;

  for (int grp = blockIdx.x; grp < groups; grp += gridDim.x) {  // CTA-uniform loop
    const int row = grp * RPC + local_row;
    const bool row_ok = row < M;
    uint4 raw[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = t + i * TPR;
      raw[i] = (row_ok && c < nchunk)
                   ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)row * K) + c)
                   : make_uint4(0u, 0u, 0u, 0u);
    }
    float amax = 0.0f;
    if constexpr (!STATIC) {
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = t + i * TPR;
        if (c < nchunk) {
          float2 v[4];
          scale8_pairs(raw[i], cinv_s, c, v);
#pragma unroll
          for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(v[e].x), fabsf(v[e].y)));
        }
      }
      amax = warp_max(amax);
      if constexpr (WPR > 1) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < WPR; ++j) amax = fmaxf(amax, red[local_row * WPR + j]);
        __syncthreads();  // red is rewritten by the next pass
      }
    }
    if (!row_ok) continue;

    float s = 0.0f;
    const int sid = stream_id[row];
    if (sid < S) {
      float clip;
      if constexpr (STATIC) {
        const float g = __ldg(alpha + step * S + sid);
        clip = g > 0.0f ? __fdiv_rn(__ldg(thr + step), g) : 0.0f;
      } else {
        clip = __fmul_rn(__ldg(alpha + step * S + sid), amax);
      }
      s = __fdiv_rn(clip, static_cast<float>(QMAX));
    } else if (t == 0) {
      raise_error(kErrBadStreamId);
    }
    if (t == 0) s_tok[row] = s;
    const float r = s > 0.0f ? __frcp_rn(s) : 0.0f;
    const bool fast = s > 0.0f && isfinite(r);  // else: zero row, or a tiny scale

#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = t + i * TPR;
      if (c >= nchunk) continue;
      float2 v[4];
      scale8_pairs(raw[i], cinv_s, c, v);
      uint2 cw;  // the 8 codes, one per byte
      if (fast) {
        // codes_packed's 16-bit clamp needs |x'| / s < 2^15: the row maximum bounds
        // it (dynamic clipping), else this chunk's own maximum
        float cmax = amax;
        if constexpr (STATIC) {
#pragma unroll
          for (int e = 0; e < 4; ++e) cmax = fmaxf(cmax, fmaxf(fabsf(v[e].x), fabsf(v[e].y)));
        }
        cw = codes_packed<QMAX, 8>(v, s, r, cmax <= 16384.0f * s);
      } else {
        uint32_t q[8];  // low byte of each: the code
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          q[2 * e] = static_cast<uint32_t>(quantize<QMAX>(v[e].x, s));
          q[2 * e + 1] = static_cast<uint32_t>(quantize<QMAX>(v[e].y, s));
        }
        cw = make_uint2(pack_low_bytes(q[0], q[1], q[2], q[3]),
                        pack_low_bytes(q[4], q[5], q[6], q[7]));
      }
      if constexpr (STORE_BITS == 8) {
        reinterpret_cast<uint2*>(static_cast<int8_t*>(qx) + (size_t)row * K)[c] = cw;
      } else {
        // nibbles: bytes 0 and 2 of n hold (c0 | c1 << 4) and (c2 | c3 << 4)
        uint32_t n0 = cw.x & 0x0F0F0F0Fu, n1 = cw.y & 0x0F0F0F0Fu;
        n0 |= n0 >> 4;
        n1 |= n1 >> 4;
        reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(qx) + (size_t)row * (K / 2))[c] =
            __byte_perm(n0, n1, 0x6420);
      }
    }
  }
}

template <int ACT_BITS, int STORE_BITS, int TPR, int CPT, bool STATIC>
cudaError_t run_act_quant(const uint16_t* x, int M, int K, const float* cinv,
                          const uint8_t* sid, const float* alpha, const float* thr, int S,
                          int step, void* qx, float* s_tok, uint4* zero, size_t zero_n16,
                          cudaStream_t st) {
  constexpr int RPC = 256 / TPR;
  const size_t smem = static_cast<size_t>(K) * sizeof(float);  // cinv copy
  static std::atomic<bool> attr_set[kAttrDevices] = {};  // per template instance and device
  // resident CTAs per SM for the last K seen, packed with that K into one word so
  // concurrent callers never pair one K with another K's count: (K << 32) | CTAs
  static std::atomic<uint64_t> occupancy{0};
  // cinv's shared-memory copy: up to kMaxK floats
  const cudaError_t ea = set_smem_once(act_quant_kernel<ACT_BITS, STORE_BITS, TPR, CPT, STATIC>,
                                       kMaxK * 4, attr_set);
  if (ea != cudaSuccess) return ea;
  const uint64_t occ = occupancy.load(std::memory_order_relaxed);
  int per_sm = static_cast<int>(occ & 0xFFFFFFFFu);
  if (static_cast<int>(occ >> 32) != K) {
    per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, act_quant_kernel<ACT_BITS, STORE_BITS, TPR, CPT, STATIC>, 256, smem);
    if (per_sm < 1) per_sm = 1;
    occupancy.store((static_cast<uint64_t>(K) << 32) | static_cast<uint32_t>(per_sm),
                    std::memory_order_relaxed);
  }
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int groups = (M + RPC - 1) / RPC;
  const int grid = groups < per_sm * sms ? groups : per_sm * sms;
  return launch_pdl(act_quant_kernel<ACT_BITS, STORE_BITS, TPR, CPT, STATIC>, grid, 256, smem, st, 1, x, M, K, cinv, sid,
                    alpha, thr, S, step, qx, s_tok, zero, zero_n16);
}

// One warp per token row, no block-level synchronisation: pass 1 streams the row
// for its maximum (absent with static clipping), pass 2 reads it again (from L2)
// and writes the codes.  Warps progress independently, so one warp's loads
// overlap other warps' arithmetic.
template <int ACT_BITS, int STORE_BITS, bool STATIC>
__global__ void __launch_bounds__(256) act_quant_row_kernel(
    const uint16_t* __restrict__ x, int M, int K, const float* __restrict__ cinv,
    const uint8_t* __restrict__ stream_id, const float* __restrict__ alpha,
    const float* __restrict__ thr, int S, int step, void* __restrict__ qx,
    float* __restrict__ s_tok, uint4* __restrict__ zero, size_t zero_n16) {
  constexpr int QMAX = ACT_BITS == 8 ? 127 : 7;
  constexpr int U = 4;  // chunks in flight per lane
  griddep_wait();
  griddep_launch_dependents();
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < zero_n16; i += (size_t)gridDim.x * 256)
    zero[i] = make_uint4(0u, 0u, 0u, 0u);
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * 8;
  const int nchunk = K >> 3;
  for (int row = blockIdx.x * 8 + (threadIdx.x >> 5); row < M; row += nwarps) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * K);
    float amax = 0.0f;
    if constexpr (!STATIC) {
      for (int c0 = lane; c0 < nchunk; c0 += 32 * U) {
        uint4 raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + 32 * u;
          raw[u] = c < nchunk ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + 32 * u;
          if (c < nchunk) {
            float ci[8], v[8];
            load_cinv8_global(cinv, c, ci);
            scale8(raw[u], ci, v);
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
          }
        }
      }
      amax = warp_max(amax);
    }
    float s = 0.0f;
    const int sid = stream_id[row];
    if (sid < S) {
      float clip;
      if constexpr (STATIC) {
        const float g = __ldg(alpha + step * S + sid);
        clip = g > 0.0f ? __fdiv_rn(__ldg(thr + step), g) : 0.0f;
      } else {
        clip = __fmul_rn(__ldg(alpha + step * S + sid), amax);
      }
      s = __fdiv_rn(clip, static_cast<float>(QMAX));
    } else if (lane == 0) {
      raise_error(kErrBadStreamId);
    }
    if (lane == 0) s_tok[row] = s;
    const float r = s > 0.0f ? __frcp_rn(s) : 0.0f;
    const bool fast = s > 0.0f && isfinite(r);
    for (int c0 = lane; c0 < nchunk; c0 += 32 * U) {
      uint4 raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        raw[u] = c < nchunk ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + 32 * u;
        if (c >= nchunk) continue;
        float ci[8], v[8];
        load_cinv8_global(cinv, c, ci);
        scale8(raw[u], ci, v);
        uint32_t q[8];
        if (fast) {
          quantize8_recip<QMAX>(v, s, r, q);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) q[e] = static_cast<uint32_t>(quantize<QMAX>(v[e], s));
        }
        if constexpr (STORE_BITS == 8) {
          reinterpret_cast<uint2*>(static_cast<int8_t*>(qx) + (size_t)row * K)[c] =
              make_uint2(pack_low_bytes(q[0], q[1], q[2], q[3]),
                         pack_low_bytes(q[4], q[5], q[6], q[7]));
        } else {
          reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(qx) + (size_t)row * (K / 2))[c] =
              pack_low_nibbles(q);
        }
      }
    }
  }
}

template <int ACT_BITS, int STORE_BITS, bool STATIC>
cudaError_t run_act_quant_rows(const uint16_t* x, int M, int K, const float* cinv,
                               const uint8_t* sid, const float* alpha, const float* thr, int S,
                               int step, void* qx, float* s_tok, uint4* zero, size_t zero_n16,
                               cudaStream_t st) {
  static const int per_sm = [] {  // per template instance; thread-safe initialisation
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &n, act_quant_row_kernel<ACT_BITS, STORE_BITS, STATIC>, 256, 0);
    return n < 1 ? 1 : n;
  }();
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int want = (M + 7) / 8;  // one warp per row
  const int grid = want < per_sm * sms ? want : per_sm * sms;
  return launch_pdl(act_quant_row_kernel<ACT_BITS, STORE_BITS, STATIC>, grid, 256, 0, st, 1, x, M,
                    K, cinv, sid, alpha, thr, S, step, qx, s_tok, zero, zero_n16);
}

// ---------------------------------------------------------------- staged rows
// Many rows of K = 512*C channels: rows are staged in shared memory by bulk copies
// (a ring of kRingSlots rounds of R = kRingRoundElems / K rows, copies of later
// rounds in flight while a round is computed), and every one of the 512 threads
// owns C fixed channels of every row, so its C channel scales stay in registers
// for the whole launch and each staged element is read from shared memory once:
// x' = x * cinv is formed once into registers, the row maxima are combined
// across the CTA (warp shuffles, then one shared-memory atomic max per warp and
// row), R threads turn them into the rows' scales, and every thread writes the
// codes of its channels.  One CTA per SM, persistent over rounds.
constexpr int kRingElemsPerThread = 64;  // of every round

constexpr int kRingSlots = 3;
#ifndef WQ_RING_MIN_ROWS
#define WQ_RING_MIN_ROWS 512
#endif
constexpr int kRingMinRows = WQ_RING_MIN_ROWS;

// NT threads per CTA (512: one CTA per SM; 256: two, so that one computes while
// the other waits at a barrier), C channels per thread.
template <int C, int NT>
struct Ring {
  static constexpr int K = NT * C;
  static constexpr int R = kRingElemsPerThread / C;       // rows per round
  static constexpr int ROUND_BYTES = R * K * 2;
  static constexpr int OFF_AMAX = kRingSlots * ROUND_BYTES;  // uint32 [3][R], rounds mod 3
  static constexpr int OFF_BAR = (OFF_AMAX + 3 * R * 4 + 7) / 8 * 8;
  static constexpr int SMEM = OFF_BAR + kRingSlots * 8;
  static_assert(R >= 1 && C >= 4 && C % 4 == 0, "C = K / 512 channels per thread");
};

// N codes from the reciprocal (see quantize8_recip); each result's low byte is the code.
template <int QMAX, int N>
__device__ __forceinline__ void quantize_recip_n(const float* v, float s, float r,
                                                 uint32_t* c) {
  constexpr float lo = kRoundMagic - static_cast<float>(QMAX);
  constexpr float hi = kRoundMagic + static_cast<float>(QMAX);
  bool near_tie = false;
#pragma unroll
  for (int e = 0; e < N; ++e) {
    const float t = __fmul_rn(v[e], r);
    const float u = __fadd_rn(t, kRoundMagic);
    const float d = __fsub_rn(t, __fsub_rn(u, kRoundMagic));
    near_tie = near_tie || fabsf(d) >= 0.5f - 0x1p-12f;
    c[e] = __float_as_uint(fminf(fmaxf(u, lo), hi));
  }
  if (near_tie) {
#pragma unroll
    for (int e = 0; e < N; ++e) {
      const float t = __fmul_rn(v[e], r);
      const float u = __fadd_rn(t, kRoundMagic);
      const float d = __fsub_rn(t, __fsub_rn(u, kRoundMagic));
      if (fabsf(d) >= 0.5f - 0x1p-12f) c[e] = static_cast<uint32_t>(quantize_exact<QMAX>(v[e], s));
    }
  }
}

// Maxima over the warp of R values per lane (R a power of two, at most 32), with
// R - 1 + 5 - log2(R) shuffles instead of 5 R: each step halves the values a lane
// keeps and the lanes exchanging them.  Returns, in lane l, the maximum of value
// index (l >> (5 - log2 R)) over all 32 lanes.
template <int R>
__device__ __forceinline__ float warp_max_multi(float (&v)[R], int lane) {
  int o = 16;
#pragma unroll
  for (int n = R; n > 1; n >>= 1, o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = upper ? v[j] : v[j + n / 2];
      const float keep = upper ? v[j + n / 2] : v[j];
      v[j] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, o));
    }
  }
#pragma unroll
  for (; o > 0; o >>= 1) v[0] = fmaxf(v[0], __shfl_xor_sync(0xFFFFFFFFu, v[0], o));
  return v[0];
}

template <int R>
constexpr int log2_of() { return R <= 1 ? 0 : 1 + log2_of<R / 2>(); }

// Codes of one group of GW = 4 or 8 values (x' as GW/2 pairs), scale s > 0 with
// r = 1/s finite, as bytes (GW/4 words): the general path, one value at a time
// (float clamp, exact quotient at near ties).  Kept out of line: the packed path
// below serves almost every group.
template <int QMAX, int GW>
__device__ __noinline__ uint2 codes_general(float4 a, float4 b, float s, float r) {
  const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t c[8];
  quantize_recip_n<QMAX, GW>(v, s, r, c);
  return make_uint2(pack_low_bytes(c[0], c[1], c[2], c[3]),
                    GW == 8 ? pack_low_bytes(c[4], c[5], c[6], c[7]) : 0u);
}

// The same codes two values at a time: t = x' * r, u = t + 1.5*2^23 (u's low 16 bits
// are rint(t) as a two's-complement int16 while |t| < 2^15), clamped as 16-bit
// pairs.  `narrow` says |t| < 2^15 holds for the row (its maximum |x'| <= 16384 s).
// Falls back to codes_general when a value lies near a half-integer or the row is
// not narrow; the result equals quantize<QMAX>(v, s) for every value.
template <int QMAX, int GW>
__device__ __forceinline__ uint2 codes_packed(const float2 (&v)[GW / 2], float s, float r,
                                              bool narrow) {
  const float2 r2 = make_float2(r, r);
  const float2 m2 = make_float2(kRoundMagic, kRoundMagic);
  const float2 nm2 = make_float2(-kRoundMagic, -kRoundMagic);
  const float2 neg1 = make_float2(-1.0f, -1.0f);
  bool near_tie = false;
  uint32_t h[GW / 2];
#pragma unroll
  for (int p = 0; p < GW / 2; ++p) {
    const float2 t = __fmul2_rn(v[p], r2);
    const float2 u = __fadd2_rn(t, m2);
    const float2 d = __ffma2_rn(__fadd2_rn(u, nm2), neg1, t);  // t - rint(t), exact
    near_tie = near_tie || fabsf(d.x) >= 0.5f - 0x1p-12f || fabsf(d.y) >= 0.5f - 0x1p-12f;
    h[p] = __byte_perm(__float_as_uint(u.x), __float_as_uint(u.y), 0x5410);
  }
  if (near_tie || !narrow) {
    const float4 a = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
    const float4 b = GW == 8 ? make_float4(v[GW / 2 - 2].x, v[GW / 2 - 2].y, v[GW / 2 - 1].x,
                                           v[GW / 2 - 1].y)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    return codes_general<QMAX, GW>(a, b, s, r);
  }
  constexpr uint32_t lo = static_cast<uint32_t>(static_cast<uint16_t>(-QMAX)) * 0x00010001u;
  constexpr uint32_t hi = static_cast<uint32_t>(QMAX) * 0x00010001u;
#pragma unroll
  for (int p = 0; p < GW / 2; ++p) h[p] = __vmins2(__vmaxs2(h[p], lo), hi);
  return make_uint2(__byte_perm(h[0], h[1], 0x6420),
                    GW == 8 ? __byte_perm(h[GW / 2 - 2], h[GW / 2 - 1], 0x6420) : 0u);
}

template <int ACT_BITS, int STORE_BITS, int C, int NT, bool STATIC>
__global__ void __launch_bounds__(NT, 512 / NT) act_quant_ring_kernel(
    const uint16_t* __restrict__ x, int M, const float* __restrict__ cinv,
    const uint8_t* __restrict__ stream_id, const float* __restrict__ alpha,
    const float* __restrict__ thr, int S, int step, void* __restrict__ qx,
    float* __restrict__ s_tok, uint4* __restrict__ zero, size_t zero_n16) {
  using G = Ring<C, NT>;
  constexpr int K = G::K, R = G::R;
  constexpr int QMAX = ACT_BITS == 8 ? 127 : 7;
  // thread t owns channel groups g = t + NT * j of GW channels each
  constexpr int GW = C % 8 == 0 ? 8 : 4;
  constexpr int NG = C / GW;
  constexpr int P = C / 2;  // value pairs per row and thread
  extern __shared__ __align__(128) uint8_t ring_smem[];
  uint32_t* amax_s = reinterpret_cast<uint32_t*>(ring_smem + G::OFF_AMAX);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring_smem + G::OFF_BAR);
  const int t = threadIdx.x;
  const int lane = t & 31;

  if (t == 0) {
    for (int i = 0; i < kRingSlots; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  if (t < 3 * R) amax_s[t] = 0u;
  float2 ci[P];
#pragma unroll
  for (int j = 0; j < NG; ++j) {
#pragma unroll
    for (int q4 = 0; q4 < GW / 4; ++q4) {
      const int k0 = GW * (t + NT * j) + 4 * q4;
      const float4 a = cinv ? __ldg(reinterpret_cast<const float4*>(cinv + k0))
                            : make_float4(1.f, 1.f, 1.f, 1.f);
      ci[j * (GW / 2) + 2 * q4] = make_float2(a.x, a.y);
      ci[j * (GW / 2) + 2 * q4 + 1] = make_float2(a.z, a.w);
    }
  }
  __syncthreads();
  // x, the ids and the split-K scratch may belong to the previous kernel
  griddep_wait();
  griddep_launch_dependents();
  for (size_t i = (size_t)blockIdx.x * NT + t; i < zero_n16; i += (size_t)gridDim.x * NT)
    zero[i] = make_uint4(0u, 0u, 0u, 0u);

  const int rounds = (M + R - 1) / R;
  auto issue = [&](int local) {  // copy this CTA's round `local` into its slot
    const int q = blockIdx.x + local * gridDim.x;
    if (q >= rounds) return;
    const int rows = min(R, M - q * R);
    uint64_t* bar = &full[local % kRingSlots];
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * K * 2);
    bulk_load_1d(ring_smem + (local % kRingSlots) * G::ROUND_BYTES, x + (size_t)q * R * K,
                 static_cast<uint32_t>(rows) * K * 2, bar);
  };
  if (t == 0)
    for (int i = 0; i < kRingSlots; ++i) issue(i);

  int issued = kRingSlots;
  bool ok = true;
  int local = 0;
  for (int q = blockIdx.x; q < rounds; q += gridDim.x, ++local) {
    const int slot = local % kRingSlots;
    const int row0 = q * R;
    const int rows = min(R, M - row0);
    const bool landed = mbar_wait(&full[slot], (local / kRingSlots) & 1u);
    // x' of this thread's channels of every row of the round, and the row maxima
    float2 xv[R][P];
    float pmax[R];  // this thread's maximum of |x'| per row
    const uint8_t* base = ring_smem + slot * G::ROUND_BYTES;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        uint32_t w[GW / 2];
        const uint8_t* src = base + (size_t)i * K * 2 + 2 * GW * (t + NT * j);
        if (landed && i < rows) {
          if constexpr (GW == 8) {
            const uint4 q4 = *reinterpret_cast<const uint4*>(src);
            w[0] = q4.x; w[1] = q4.y; w[2 % (GW / 2)] = q4.z; w[3 % (GW / 2)] = q4.w;
          } else {
            const uint2 q2 = *reinterpret_cast<const uint2*>(src);
            w[0] = q2.x; w[1] = q2.y;
          }
        } else {
#pragma unroll
          for (int e = 0; e < GW / 2; ++e) w[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < GW / 2; ++e) {
          const float2 f = make_float2(bf16lo(w[e]), bf16hi(w[e]));
          const float2 v = __fmul2_rn(f, ci[j * (GW / 2) + e]);
          xv[i][j * (GW / 2) + e] = v;
          amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
        }
      }
      pmax[i] = amax;
    }
    {
      // row (lane >> SH) of the round, reduced over the warp, then over the warps
      // (non-negative floats order as their bit patterns)
      constexpr int SH = 5 - log2_of<R>();
      const float wmax = warp_max_multi<R>(pmax, lane);
      if ((lane & ((1 << SH) - 1)) == 0 && wmax > 0.0f)
        atomicMax(&amax_s[(local % 3) * R + (lane >> SH)], __float_as_uint(wmax));
    }
    // the next round's maxima (the round before last, whose readers all passed the
    // previous barrier, used this third of the buffer)
    if (t < R) amax_s[((local + 1) % 3) * R + t] = 0u;
    // every thread has read its channels of the slot, and every row maximum is in
    if (__syncthreads_or(!landed)) { ok = false; break; }
    if (t == 0 && issued < kRingSlots + local + 1) {  // refill the slot just read
      issue(local + kRingSlots);
      issued = kRingSlots + local + 1;
    }
    // Every warp derives the round's scales itself (lane i takes row i) and passes
    // them along by shuffles: one CTA barrier per round.  Warp 0 alone writes s_tok
    // and reports a bad stream id.
    float sc_l = 0.0f, rs_l = 0.0f;
    if (lane < rows) {
      const int row = row0 + lane;
      const float amax = __uint_as_float(amax_s[(local % 3) * R + lane]);
      const int sid = stream_id[row];
      if (sid < S) {
        float clip;
        if constexpr (STATIC) {
          const float g = __ldg(alpha + step * S + sid);
          clip = g > 0.0f ? __fdiv_rn(__ldg(thr + step), g) : 0.0f;
        } else {
          clip = __fmul_rn(__ldg(alpha + step * S + sid), amax);
        }
        sc_l = __fdiv_rn(clip, static_cast<float>(QMAX));
      } else if (t < 32) {
        raise_error(kErrBadStreamId);
      }
      if (t < 32) s_tok[row] = sc_l;
      const float rc = sc_l > 0.0f ? __frcp_rn(sc_l) : 0.0f;
      // negative reciprocal: this row takes the general path (a zero or tiny scale)
      const bool fast = sc_l > 0.0f && isfinite(rc);
      rs_l = fast ? (amax <= 16384.0f * sc_l ? rc : -rc) : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const float sc = __shfl_sync(0xFFFFFFFFu, sc_l, i);
      const float rs = __shfl_sync(0xFFFFFFFFu, rs_l, i);
      if (i >= rows) break;
      const float rc = fabsf(rs);
      const bool fast = rs != 0.0f;
      const bool narrow = rs > 0.0f;
      const size_t row = static_cast<size_t>(row0 + i);
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        uint2 cw;
        if (fast) {
          float2 vv[GW / 2];
#pragma unroll
          for (int e = 0; e < GW / 2; ++e) vv[e] = xv[i][j * (GW / 2) + e];
          cw = codes_packed<QMAX, GW>(vv, sc, rc, narrow);
        } else {
          uint32_t cq[GW];
#pragma unroll
          for (int e = 0; e < GW / 2; ++e) {
            cq[2 * e] = static_cast<uint32_t>(quantize<QMAX>(xv[i][j * (GW / 2) + e].x, sc));
            cq[2 * e + 1] = static_cast<uint32_t>(quantize<QMAX>(xv[i][j * (GW / 2) + e].y, sc));
          }
          cw = make_uint2(pack_low_bytes(cq[0], cq[1], cq[2], cq[3]),
                          GW == 8 ? pack_low_bytes(cq[4 % GW], cq[5 % GW], cq[6 % GW], cq[7 % GW])
                                  : 0u);
        }
        const int g = t + NT * j;  // channel group: channels GW*g .. GW*g + GW-1
        if constexpr (STORE_BITS == 8) {
          if constexpr (GW == 8)
            reinterpret_cast<uint2*>(static_cast<int8_t*>(qx) + row * K)[g] = cw;
          else
            reinterpret_cast<uint32_t*>(static_cast<int8_t*>(qx) + row * K)[g] = cw.x;
        } else {
          // nibbles: bytes 0 and 2 of n hold (c0 | c1 << 4) and (c2 | c3 << 4)
          uint32_t n0 = cw.x & 0x0F0F0F0Fu;
          n0 |= n0 >> 4;
          if constexpr (GW == 8) {
            uint32_t n1 = cw.y & 0x0F0F0F0Fu;
            n1 |= n1 >> 4;
            reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(qx) + row * (K / 2))[g] =
                __byte_perm(n0, n1, 0x6420);
          } else {
            reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(qx) + row * (K / 2))[g] =
                static_cast<uint16_t>(__byte_perm(n0, 0u, 0x0020) & 0xFFFFu);
          }
        }
      }
    }
  }
  // copies still in flight (after an error, or none): wait for them before exiting
  if (t == 0) {
    const int my_rounds = blockIdx.x < rounds ? (rounds - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int last = min(issued, my_rounds);
    for (int i = ok ? last : local; i < last; ++i)
      mbar_wait_drain(&full[i % kRingSlots], (i / kRingSlots) & 1u);
  }
}

template <int ACT_BITS, int STORE_BITS, int C, int NT, bool STATIC>
cudaError_t run_act_quant_ring(const uint16_t* x, int M, const float* cinv, const uint8_t* sid,
                               const float* alpha, const float* thr, int S, int step, void* qx,
                               float* s_tok, uint4* zero, size_t zero_n16, cudaStream_t st) {
  using G = Ring<C, NT>;
  static std::atomic<bool> attr_set[kAttrDevices] = {};  // per template instance and device
  const cudaError_t ea = set_smem_once(act_quant_ring_kernel<ACT_BITS, STORE_BITS, C, NT, STATIC>,
                                       G::SMEM, attr_set);
  if (ea != cudaSuccess) return ea;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rounds = (M + G::R - 1) / G::R;
  const int slots = sms * (512 / NT);  // resident CTAs
  const int grid = rounds < slots ? rounds : slots;
  return launch_pdl(act_quant_ring_kernel<ACT_BITS, STORE_BITS, C, NT, STATIC>, grid, NT, G::SMEM,
                    st, 1, x, M, cinv, sid, alpha, thr, S, step, qx, s_tok, zero, zero_n16);
}

template <int ACT_BITS, int STORE_BITS, bool STATIC>
cudaError_t dispatch_act_quant(const uint16_t* x, int M, int K, const float* cinv,
                               const uint8_t* sid, const float* alpha, const float* thr, int S,
                               int step, void* qx, float* s_tok, uint4* zero, size_t zero_n16,
                               cudaStream_t st) {
#define WQ_RING(C_, NT_)                                                                      \
  return run_act_quant_ring<ACT_BITS, STORE_BITS, C_, NT_, STATIC>(x, M, cinv, sid, alpha, thr, \
                                                                   S, step, qx, s_tok, zero,    \
                                                                   zero_n16, st)
  // Many rows of K = 4096: rows staged in shared memory, channels owned by threads,
  // two CTAs of 256 threads per SM (measured 16 % faster than one warp per row at
  // M = 8512; at K = 2048, 8192 and 16384 the kernels below were as fast or faster).
  if (M >= kRingMinRows && K == 4096) WQ_RING(16, 256);
#undef WQ_RING
  // Many rows of moderate length: independent warps, one per row (measured faster
  // for M = 4288 and 8512 at K = 2048 and 4096).  Few rows, or long rows, keep a
  // CTA's threads on each row (measured faster for M <= 256, and for K >= 8192).
  if (M >= 1024 && K <= 4096)
    return run_act_quant_rows<ACT_BITS, STORE_BITS, STATIC>(x, M, K, cinv, sid, alpha, thr, S,
                                                            step, qx, s_tok, zero, zero_n16, st);
  const int nchunk = K / 8;
#define WQ_AQ(TPR, CPT) \
  return run_act_quant<ACT_BITS, STORE_BITS, TPR, CPT, STATIC>(x, M, K, cinv, sid, alpha, thr, S, \
                                                               step, qx, s_tok, zero, zero_n16, st)
  // Few rows (the launch is one pass): a whole CTA per row, so each thread's
  // share, and the pass's latency, stays small.
  if (M <= 64) {
    if (nchunk <= 256) WQ_AQ(256, 1);
    if (nchunk <= 512) WQ_AQ(256, 2);
    if (nchunk <= 1024) WQ_AQ(256, 4);
  }
  // one warp per row up to K = 2048 (no block-level reduction), 8 chunks of 8
  // channels per thread beyond that
  if (nchunk <= 32) WQ_AQ(32, 1);
  if (nchunk <= 64) WQ_AQ(32, 2);
  if (nchunk <= 128) WQ_AQ(32, 4);
  if (nchunk <= 256) WQ_AQ(32, 8);
  if (nchunk <= 512) WQ_AQ(64, 8);
  if (nchunk <= 1024) WQ_AQ(128, 8);
  if (nchunk <= 2048) WQ_AQ(256, 8);
  WQ_AQ(256, 16);
#undef WQ_AQ
}

// ------------------------------------------------------------ offline weights

__device__ __forceinline__ float block_max_256(float v, float* red) {
  v = warp_max(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int j = 1; j < 8; ++j) r = fmaxf(r, red[j]);
  __syncthreads();
  return r;
}

// One CTA per output channel n: s_w[n] = max_k |W[n,k]*c[k]| / 7, codes packed
// two per byte (low nibble = even k).
__global__ void __launch_bounds__(256) pack_int4_kernel(const uint16_t* __restrict__ W,
                                                        const float* __restrict__ c, int K,
                                                        uint8_t* __restrict__ qw,
                                                        float* __restrict__ s_w) {
  __shared__ float red[8];
  const int n = blockIdx.x;
  const uint16_t* row = W + (size_t)n * K;
  float amax = 0.0f;
  for (int k = threadIdx.x; k < K; k += 256) {
    const float w = __fmul_rn(__uint_as_float((uint32_t)row[k] << 16), c ? c[k] : 1.0f);
    amax = fmaxf(amax, fabsf(w));
  }
  amax = block_max_256(amax, red);
  const float s = __fdiv_rn(amax, 7.0f);
  if (threadIdx.x == 0) s_w[n] = s;
  for (int j = threadIdx.x; j < K / 2; j += 256) {
    const int k = 2 * j;
    const float w0 = __fmul_rn(__uint_as_float((uint32_t)row[k] << 16), c ? c[k] : 1.0f);
    const float w1 = __fmul_rn(__uint_as_float((uint32_t)row[k + 1] << 16), c ? c[k + 1] : 1.0f);
    const int q0 = quantize<7>(w0, s), q1 = quantize<7>(w1, s);
    qw[(size_t)n * (K / 2) + j] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
  }
}

// One thread per input channel k: column maxima over the calibration batch and
// over the weight rows, then c = sqrt(a / b) (1 when either maximum is 0).
__global__ void channel_scale_kernel(const uint16_t* __restrict__ x_cal, int Mcal,
                                     const uint16_t* __restrict__ W, int N, int K,
                                     float* __restrict__ c, float* __restrict__ cinv) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float a = 0.0f, b = 0.0f;
  for (int m = 0; m < Mcal; ++m)
    a = fmaxf(a, fabsf(__uint_as_float((uint32_t)x_cal[(size_t)m * K + k] << 16)));
  for (int n = 0; n < N; ++n)
    b = fmaxf(b, fabsf(__uint_as_float((uint32_t)W[(size_t)n * K + k] << 16)));
  float ck = 1.0f;
  if (a > 0.0f && b > 0.0f) ck = __fsqrt_rn(__fdiv_rn(a, b));
  c[k] = ck;
  cinv[k] = __fdiv_rn(1.0f, ck);
}

}  // namespace

template <bool STATIC>
cudaError_t launch_act_quant_mode(const uint16_t* x, int M, int K, const float* cinv,
                                  const uint8_t* sid, const float* table, const float* thr,
                                  int S, int step, int act_bits, void* qx, float* s_tok,
                                  cudaStream_t st, void* zero, size_t zero_bytes,
                                  bool bytes_per_code) {
  if (M == 0) return cudaSuccess;
  uint4* z = static_cast<uint4*>(zero);
  const size_t n16 = zero ? zero_bytes / 16 : 0;
  if (act_bits == 8)
    return dispatch_act_quant<8, 8, STATIC>(x, M, K, cinv, sid, table, thr, S, step, qx, s_tok, z,
                                            n16, st);
  if (bytes_per_code)
    return dispatch_act_quant<4, 8, STATIC>(x, M, K, cinv, sid, table, thr, S, step, qx, s_tok, z,
                                            n16, st);
  return dispatch_act_quant<4, 4, STATIC>(x, M, K, cinv, sid, table, thr, S, step, qx, s_tok, z,
                                          n16, st);
}

cudaError_t launch_act_quant(const uint16_t* x, int M, int K, const float* cinv,
                             const uint8_t* stream_id, const float* alpha, int S, int step,
                             int act_bits, void* qx, float* s_tok, cudaStream_t st,
                             void* zero, size_t zero_bytes, bool bytes_per_code) {
  return launch_act_quant_mode<false>(x, M, K, cinv, stream_id, alpha, nullptr, S, step, act_bits,
                                      qx, s_tok, st, zero, zero_bytes, bytes_per_code);
}

cudaError_t launch_act_quant_static(const uint16_t* x, int M, int K, const float* cinv,
                                    const uint8_t* stream_id, const float* thr,
                                    const float* gain, int S, int step, int act_bits, void* qx,
                                    float* s_tok, cudaStream_t st, void* zero, size_t zero_bytes,
                                    bool bytes_per_code) {
  return launch_act_quant_mode<true>(x, M, K, cinv, stream_id, gain, thr, S, step, act_bits, qx,
                                     s_tok, st, zero, zero_bytes, bytes_per_code);
}

cudaError_t launch_pack_int4(const uint16_t* W, const float* c, int N, int K, uint8_t* qw,
                             float* s_w, cudaStream_t st) {
  pack_int4_kernel<<<N, 256, 0, st>>>(W, c, K, qw, s_w);
  return cudaGetLastError();
}

cudaError_t launch_channel_scale(const uint16_t* x_cal, int Mcal, const uint16_t* W, int N,
                                 int K, float* c, float* cinv, cudaStream_t st) {
  channel_scale_kernel<<<(K + 127) / 128, 128, 0, st>>>(x_cal, Mcal, W, N, K, c, cinv);
  return cudaGetLastError();
}

}  // namespace wq
