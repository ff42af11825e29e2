// Internal launch interface between the C-ABI layer (wq_api.cu) and the
// kernels.  Arguments are assumed validated by the caller.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace wq {

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream is still running, and must call griddep_wait()
// before it touches anything that kernel (or an earlier one) writes.
// cluster > 1: clusters of that many CTAs along x (the grid a multiple of it).
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                       cudaStream_t st, int cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster > 1 ? cluster : 1);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Set a kernel's shared-memory limit once per device: function attributes belong
// to each device's context, so a process that drives several GPUs sets them on
// each.  `done` is the caller's per-kernel flag array.
constexpr int kAttrDevices = 64;
// (The flags are atomic: host threads may launch concurrently; two threads that
// both find a flag clear just set the same attribute twice.)
template <class Kernel>
cudaError_t set_smem_once(Kernel kernel, int bytes, std::atomic<bool> (&done)[kAttrDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
  const bool cached = dev >= 0 && dev < kAttrDevices;
  if (cached && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cached) done[dev].store(true, std::memory_order_release);
  return e;
}

// Largest K the quantizer keeps in registers (K/8 chunks spread over 256 threads,
// at most 16 chunks each).
constexpr int kMaxK = 32768;

cudaError_t launch_channel_scale(const uint16_t* x_cal, int Mcal, const uint16_t* W, int N,
                                 int K, float* c, float* cinv, cudaStream_t st);

cudaError_t launch_pack_int4(const uint16_t* W, const float* c, int N, int K, uint8_t* qw,
                             float* s_w, cudaStream_t st);

// `zero` (16-byte aligned, zero_bytes a multiple of 16) is cleared by the same
// launch: the fused linear uses it for the GEMM's split-K scratch.
// bytes_per_code: int4 codes are written one per int8 byte ([M][K]) instead of
// packed two per byte ([M][K/2]); int8 codes are always one per byte.
cudaError_t launch_act_quant(const uint16_t* x, int M, int K, const float* cinv,
                             const uint8_t* stream_id, const float* alpha, int S, int step,
                             int act_bits, void* qx, float* s_tok, cudaStream_t st,
                             void* zero = nullptr, size_t zero_bytes = 0,
                             bool bytes_per_code = false);

// The same quantizer with static clipping: clip = thr[step] / gain[step][stream]
// (0 when the gain is not positive) instead of alpha * (row maximum).
cudaError_t launch_act_quant_static(const uint16_t* x, int M, int K, const float* cinv,
                                    const uint8_t* stream_id, const float* thr,
                                    const float* gain, int S, int step, int act_bits, void* qx,
                                    float* s_tok, cudaStream_t st, void* zero = nullptr,
                                    size_t zero_bytes = 0, bool bytes_per_code = false);

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

// The single-kernel linear (token counts up to kSingleKernelMaxM, one token tile):
// the GEMM quantizes the bf16 activations itself (qmax 127 for act_bits 8, 7 for
// 4) into its shared-memory operand tiles.  Dynamic clipping with table = alpha
// [T][S] when thr is null; static clipping (clip = thr[step] / gain) with table =
// the gains [T][S] otherwise.  ep.s_tok is unused.
constexpr int kSingleKernelMaxM = 64;
cudaError_t launch_linear_single(const uint16_t* x, const float* cinv, const float* table,
                                 const float* thr, int act_bits, const uint8_t* qw, int M, int N,
                                 int K, const EpilogueArgs& ep, void* y, cudaStream_t st);

// Split-K (small token counts): the K blocks of each output tile are spread over
// `splits` CTAs so that about kSplitTargetCtas CTAs stream the weights, through
// scratch for the int32 partial tiles and one counter per epilogue-warp slice of
// each tile.
constexpr int kSplitTargetCtas = 148;
// epilogue warps of a GEMM CTA at most (the split-K counters hold one per warp and tile)
constexpr int kMaxEpiWarps = 12;
int gemm_splits(int M, int N, int K);
size_t gemm_split_scratch_bytes(int M, int N, int K);  // partials + counters, 0 if no split

struct SplitScratch {
  int32_t* partial;  // [tiles][BN][128] int32 sums of the splits, zero before the launch
  int* counters;     // [tiles][kMaxEpiWarps], zero before the launch
};

// The split-K scratch of a shape whose K is split, laid out from base (256-byte
// aligned): the partial tiles, then the counters, each part rounded up to 256 bytes;
// gemm_split_scratch_bytes(M, N, K) bytes in all.
SplitScratch split_scratch_at(void* base, int M, int N);

// How the GEMM runs one shape: the rules launch_gemm and launch_gemm_gelu_quant
// follow, for reporting (host arithmetic only; the SM count is the current
// device's, 148 when none is visible).
struct GemmPlan {
  int tile_tokens;      // token tile (the MMA's N): 16, 32, 64, 128, 224 or 256
  int tile_channels;    // output channels per tile: 128, or 256 on a CTA pair
  int ctas_per_tile;    // 1, or 2 for a CTA pair (tcgen05 cta_group::2)
  int k_splits;         // CTAs sharing one tile's K loop (1: K not split)
  int k_stage;          // K depth of one pipeline stage: 128 or 256
  int tiles;            // output tiles
  int weights_in_tmem;  // 1 when the unpacked int8 weight tile is the MMA's A in TMEM
};
// split_scratch: the call passes a split-K scratch (the fused linears,
// wq_gemm_w4ax_ws, the debug calls); gelu_quant: the GELU-and-quantize epilogue.
GemmPlan gemm_plan(int M, int N, int K, int act_bits, bool split_scratch, bool gelu_quant);

// Optional parts of a GEMM launch.
struct GemmExtras {
  int32_t* acc_out = nullptr;  // int32 [M][N]: a copy of the accumulators (debug view)
  // launch_gemm_gelu_quant: the next linear's static clipping, thresholds [T] and
  // stream gains [T][S]; its channel scale [N] (or null); its per-token scales
  // s_next [M] (written); h = bf16(GELU(y)) [M][N] (written when not null)
  const float* next_thr = nullptr;
  const float* next_gain = nullptr;
  const float* next_cinv = nullptr;
  float* next_s = nullptr;
  uint16_t* h = nullptr;
};

// y[M][N] (bf16) = epilogue(qx x qw^T).  y may be null when extras->acc_out is
// set: the launch then writes only the int32 accumulators (the epilogue
// arguments other than S and step are not read).  With scratch == nullptr K is
// never split; otherwise it is split as gemm_splits() says, through the scratch,
// which must be zero before the launch.  Every instance writes the same
// accumulators through the same pipeline whether or not acc_out is set.
// w_prefetch: the packed weights (and nothing else) may be read before the
// previous kernel in the stream has finished.  Only valid when that kernel is
// this library's quantizer, which starts its dependents only after everything
// launched before it has completed.
cudaError_t launch_gemm(const void* qx, int act_bits, const uint8_t* qw, int M, int N, int K,
                        const EpilogueArgs& ep, void* y, const SplitScratch* scratch,
                        cudaStream_t st, bool w_prefetch = false,
                        const GemmExtras* extras = nullptr);

// Builds, once per device, the GELU table launch_gemm_gelu_quant reads; call before
// anything of that call is launched (it may synchronize the stream once).
cudaError_t ensure_gelu_table(cudaStream_t st);

// The FFN up-projection whose epilogue quantizes for the down-projection: the
// same GEMM on int8 codes qx, y as launch_gemm computes it, then h = bf16(GELU(y))
// and codes[m][n] = clamp(rint(h * next_cinv[n] / s_next[m]), +-qmax_next) with
// s_next[m] = (next_thr[step] / next_gain[step][stream]) / qmax_next (qmax_next 127
// for next_bits 8, 7 for 4), one code per int8 byte [M][N].  y is not stored.
cudaError_t launch_gemm_gelu_quant(const void* qx, const uint8_t* qw, int M, int N, int K,
                                   const EpilogueArgs& ep, int next_bits, int8_t* codes,
                                   const SplitScratch* scratch, cudaStream_t st, bool w_prefetch,
                                   const GemmExtras& extras);

}  // namespace wq
