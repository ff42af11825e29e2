// Internal launch interface between the C-ABI layer (wq_api.cu) and the
// kernels.  Arguments are assumed validated by the caller.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace wq {

// Largest K the quantizer keeps in registers (K/8 chunks spread over 256 threads,
// at most 16 chunks each).
constexpr int kMaxK = 32768;

cudaError_t launch_channel_scale(const uint16_t* x_cal, int Mcal, const uint16_t* W, int N,
                                 int K, float* c, float* cinv, cudaStream_t st);

cudaError_t launch_pack_int4(const uint16_t* W, const float* c, int N, int K, uint8_t* qw,
                             float* s_w, cudaStream_t st);

cudaError_t launch_act_quant(const uint16_t* x, int M, int K, const float* cinv,
                             const uint8_t* stream_id, const float* alpha, int S, int step,
                             int act_bits, void* qx, float* s_tok, cudaStream_t st);

// Epilogue inputs of the fused GEMM.
struct EpilogueArgs {
  const float* s_tok;        // [M]
  const uint8_t* stream_id;  // [M]
  const float* s_w;          // [N]
  const float* bias;         // [N] or null
  const float* beta;         // [T][S][N] or null
  int S;
  int step;
};

// y[M][N] (bf16) = epilogue(qx x qw^T) when out_s32 == false; acc[M][N] (int32)
// when out_s32 == true (the epilogue arguments are then ignored).
cudaError_t launch_gemm(const void* qx, int act_bits, const uint8_t* qw, int M, int N, int K,
                        const EpilogueArgs& ep, void* out, bool out_s32, cudaStream_t st);

}  // namespace wq
