// C ABI of libwq (declared in include/wq.h): host-side validation, workspace
// layout and launches.  The whole library is this one translation unit; the
// kernels live in the included .cuh files.
#include "wq.h"

#include <cstdint>
#include <mutex>

#include "wq_gemm.cuh"
#include "wq_internal.h"
#include "wq_quant.cuh"

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

wq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA; }

wq_status check_mk(int M, int K) {
  if (M < 0 || K < 128 || (K % 128) != 0 || K > wq::kMaxK) return WQ_ERR_SHAPE;
  return WQ_OK;
}

wq_status check_n(int N) { return (N < 16 || (N % 16) != 0) ? WQ_ERR_SHAPE : WQ_OK; }

wq_status check_table(int S, int T, int step) {
  if (S < 1 || S > 255 || T < 1 || step < 0 || step >= T) return WQ_ERR_ARG;
  return WQ_OK;
}

size_t act_bytes(int M, int K, int act_bits) {
  return act_bits == 8 ? static_cast<size_t>(M) * K : static_cast<size_t>(M) * (K / 2);
}

#define WQ_TRY(expr)                 \
  do {                               \
    const wq_status _s = (expr);     \
    if (_s != WQ_OK) return _s;      \
  } while (0)

wq_status gemm_checks(const void* qx, const float* s_tok, int act_bits, int M, int K, int N,
                      const uint8_t* stream_id, const float* beta, int S, int T, int step,
                      const uint8_t* qw, const float* s_w, const float* bias, const void* y) {
  if (act_bits != 8 && act_bits != 4) return WQ_ERR_ARG;
  WQ_TRY(check_mk(M, K));
  WQ_TRY(check_n(N));
  WQ_TRY(check_table(S, T, step));
  if (M == 0) return WQ_OK;
  if (!qx || !s_tok || !stream_id || !qw || !s_w || !y) return WQ_ERR_NULL;
  if (!aligned16(qx) || !aligned16(qw) || !aligned16(y) || !aligned16(s_tok) ||
      !aligned16(stream_id) || !aligned16(s_w) || (bias && !aligned16(bias)) ||
      (beta && !aligned16(beta)))
    return WQ_ERR_ALIGN;
  return WQ_OK;
}

// The workspace of a fused linear: codes | token scales | split-K partial tiles |
// split-K counters.  The codes are stored one per int8 byte for both widths: the
// tensor cores take int8 operands, so int4 activation codes in bytes feed the int8
// mainloop directly instead of being unpacked again for every weight tile.
struct Workspace {
  void* qx;
  float* s_tok;
  wq::SplitScratch scratch;  // partial == nullptr: K is not split
  void* zero;                // the split-K scratch, cleared by the quantizer's launch
  size_t zero_bytes;
};

Workspace carve(void* workspace, int M, int K, int N) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  Workspace w{};
  w.qx = ws;
  const size_t off_stok = round_up(act_bytes(M, K, 8));
  w.s_tok = reinterpret_cast<float*>(ws + off_stok);
  const size_t off_part = off_stok + round_up(sizeof(float) * static_cast<size_t>(M));
  if (wq::gemm_splits(M, N, K) > 1) {
    w.scratch = wq::split_scratch_at(ws + off_part, M, N);
    w.zero = ws + off_part;
    w.zero_bytes = wq::gemm_split_scratch_bytes(M, N, K);
  }
  return w;
}

// Host-side checks shared by the fused linears.
wq_status linear_checks(const wq_bf16* x, int M, int K, int N, const float* cinv,
                        const uint8_t* stream_id, const float* alpha, const float* beta, int S,
                        int T, int step, const uint8_t* qw, const float* s_w, const float* bias,
                        const void* out, void* workspace, size_t ws_bytes, int act_bits,
                        const float* thr) {
  if (act_bits != 8 && act_bits != 4) return WQ_ERR_ARG;
  WQ_TRY(check_mk(M, K));
  WQ_TRY(check_n(N));
  WQ_TRY(check_table(S, T, step));
  if (M == 0) return WQ_OK;  // empty batch: token tensors may be NULL
  if (!x || !stream_id || !alpha || !qw || !s_w || !out || !workspace) return WQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qw) || !aligned16(out) || !aligned16(s_w) ||
      !aligned16(stream_id) || !aligned16(alpha) || (thr && !aligned16(thr)) ||
      (cinv && !aligned16(cinv)) || (bias && !aligned16(bias)) || (beta && !aligned16(beta)) ||
      (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return WQ_ERR_ALIGN;
  if (ws_bytes < wq_workspace_bytes(M, K, N, act_bits)) return WQ_ERR_ARG;
  return WQ_OK;
}

// The first kernel of a fused linear: codes and token scales into the workspace
// (and the split-K scratch cleared).  alpha: the clip ratios [T][S] (dynamic
// clipping), or, when thr is not NULL, the stream gains [T][S] of static clipping
// with thresholds thr [T].
wq_status quantize_into(const Workspace& w, const wq_bf16* x, int M, int K, const float* cinv,
                        const uint8_t* stream_id, const float* alpha, int S, int step,
                        int act_bits, const float* thr, cudaStream_t st) {
  if (thr)
    return from_cuda(wq::launch_act_quant_static(x, M, K, cinv, stream_id, thr, alpha, S, step,
                                                 act_bits, w.qx, w.s_tok, st, w.zero,
                                                 w.zero_bytes, /*bytes_per_code=*/true));
  return from_cuda(wq::launch_act_quant(x, M, K, cinv, stream_id, alpha, S, step, act_bits,
                                        w.qx, w.s_tok, st, w.zero, w.zero_bytes,
                                        /*bytes_per_code=*/true));
}

wq_status linear(const wq_bf16* x, int M, int K, int N, const float* cinv,
                 const uint8_t* stream_id, const float* alpha, const float* beta, int S, int T,
                 int step, const uint8_t* qw, const float* s_w, const float* bias, wq_bf16* y,
                 void* workspace, size_t ws_bytes, wq_stream_t stream, int act_bits,
                 const float* thr = nullptr, int32_t* acc_out = nullptr) {
  WQ_TRY(linear_checks(x, M, K, N, cinv, stream_id, alpha, beta, S, T, step, qw, s_w, bias, y,
                       workspace, ws_bytes, act_bits, thr));
  if (M == 0) return WQ_OK;
  if (acc_out && !aligned16(acc_out)) return WQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Workspace w = carve(workspace, M, K, N);
  WQ_TRY(quantize_into(w, x, M, K, cinv, stream_id, alpha, S, step, act_bits, thr, st));
  const wq::EpilogueArgs ep{w.s_tok, stream_id, s_w, bias, beta, S, step};
  wq::GemmExtras ex;
  ex.acc_out = acc_out;
  // weights may stream while the quantizer runs (it started the GEMM only after
  // everything before it in the stream had finished); int8-stored codes: the
  // int8-activation mainloop (the int32 sums are the same)
  return from_cuda(wq::launch_gemm(w.qx, 8, qw, M, N, K, ep, y,
                                   w.scratch.partial ? &w.scratch : nullptr, st,
                                   /*w_prefetch=*/true, acc_out ? &ex : nullptr));
}

// ------------------------------------------------------------ no-alloc variant
// Scratch of wq_linear_w4a8_noalloc: the int8 codes and token scales that pass
// between the two kernels.  One copy per GPU that loads the library, held until
// the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

}  // namespace

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per
// device with that device current.  (In host code the array's name is only a
// host-side stand-in, not a device address.)
wq_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return WQ_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return WQ_OK;
}

}  // namespace

extern "C" {

const char* wq_status_string(wq_status s) {
  switch (s) {
    case WQ_OK: return "WQ_OK";
    case WQ_ERR_NULL: return "WQ_ERR_NULL: a required pointer is NULL";
    case WQ_ERR_SHAPE: return "WQ_ERR_SHAPE: M, N or K outside the supported range";
    case WQ_ERR_ALIGN: return "WQ_ERR_ALIGN: a tensor pointer is not 16-byte aligned";
    case WQ_ERR_ARG: return "WQ_ERR_ARG: bad act_bits, S, T, step or workspace size";
    case WQ_ERR_CUDA: return "WQ_ERR_CUDA: the CUDA runtime rejected a launch";
    case WQ_ERR_TIMEOUT: return "WQ_ERR_TIMEOUT: a kernel's bounded wait gave up";
    case WQ_ERR_DEVICE: return "WQ_ERR_DEVICE: a device-side precondition failed";
    case WQ_ERR_SCRATCH:
      return "WQ_ERR_SCRATCH: codes and token scales exceed the 16 MiB fixed scratch of "
             "wq_linear_w4a8_noalloc";
  }
  return "unknown wq_status";
}

int wq_version(void) { return 101; }

size_t wq_workspace_bytes(int M, int K, int N, int act_bits) {
  if ((act_bits != 8 && act_bits != 4) || check_mk(M, K) != WQ_OK || check_n(N) != WQ_OK)
    return 0;
  // codes one per byte for both widths (see linear())
  return round_up(act_bytes(M, K, 8)) + round_up(sizeof(float) * static_cast<size_t>(M)) +
         wq::gemm_split_scratch_bytes(M, N, K);
}

wq_status wq_channel_scale(const wq_bf16* x_cal, int Mcal, const wq_bf16* W, int N, int K,
                           float* c, float* cinv, wq_stream_t stream) {
  if (Mcal < 1 || N < 1 || K < 1) return WQ_ERR_SHAPE;
  if (!x_cal || !W || !c || !cinv) return WQ_ERR_NULL;
  if (!aligned16(x_cal) || !aligned16(W) || !aligned16(c) || !aligned16(cinv)) return WQ_ERR_ALIGN;
  return from_cuda(wq::launch_channel_scale(x_cal, Mcal, W, N, K, c, cinv,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_pack_int4(const wq_bf16* W, const float* c, int N, int K, uint8_t* qw,
                       float* s_w, wq_stream_t stream) {
  WQ_TRY(check_mk(0, K));
  if (N < 1) return WQ_ERR_SHAPE;
  if (!W || !qw || !s_w) return WQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(qw) || (c && !aligned16(c))) return WQ_ERR_ALIGN;
  return from_cuda(
      wq::launch_pack_int4(W, c, N, K, qw, s_w, reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_act_quant(const wq_bf16* x, int M, int K, const float* cinv,
                       const uint8_t* stream_id, const float* alpha, int S, int T, int step,
                       int act_bits, void* qx, float* s_tok, wq_stream_t stream) {
  if (act_bits != 8 && act_bits != 4) return WQ_ERR_ARG;
  WQ_TRY(check_mk(M, K));
  WQ_TRY(check_table(S, T, step));
  if (M == 0) return WQ_OK;
  if (!x || !stream_id || !alpha || !qx || !s_tok) return WQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qx) || !aligned16(s_tok) || !aligned16(stream_id) ||
      !aligned16(alpha) || (cinv && !aligned16(cinv)))
    return WQ_ERR_ALIGN;
  return from_cuda(wq::launch_act_quant(x, M, K, cinv, stream_id, alpha, S, step, act_bits, qx,
                                        s_tok, reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_act_quant_static(const wq_bf16* x, int M, int K, const float* cinv,
                              const uint8_t* stream_id, const float* thr, const float* gain,
                              int S, int T, int step, int act_bits, void* qx, float* s_tok,
                              wq_stream_t stream) {
  if (act_bits != 8 && act_bits != 4) return WQ_ERR_ARG;
  WQ_TRY(check_mk(M, K));
  WQ_TRY(check_table(S, T, step));
  if (M == 0) return WQ_OK;
  if (!x || !stream_id || !thr || !gain || !qx || !s_tok) return WQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qx) || !aligned16(s_tok) || !aligned16(stream_id) ||
      !aligned16(thr) || !aligned16(gain) || (cinv && !aligned16(cinv)))
    return WQ_ERR_ALIGN;
  return from_cuda(wq::launch_act_quant_static(x, M, K, cinv, stream_id, thr, gain, S, step,
                                               act_bits, qx, s_tok,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_linear_w4ax_static(const wq_bf16* x, int M, int K, int N, const float* cinv,
                                const uint8_t* stream_id, const float* thr, const float* gain,
                                const float* beta, int S, int T, int step, int act_bits,
                                const uint8_t* qw, const float* s_w, const float* bias,
                                wq_bf16* y, void* workspace, size_t ws_bytes,
                                wq_stream_t stream) {
  if (M > 0 && !thr) return WQ_ERR_NULL;
  return linear(x, M, K, N, cinv, stream_id, gain, beta, S, T, step, qw, s_w, bias, y,
                workspace, ws_bytes, stream, act_bits, thr);
}

wq_status wq_linear_w4ax_single(const wq_bf16* x, int M, int K, int N, const float* cinv,
                                const uint8_t* stream_id, const float* table, const float* thr,
                                const float* beta, int S, int T, int step, int act_bits,
                                const uint8_t* qw, const float* s_w, const float* bias,
                                wq_bf16* y, wq_stream_t stream) {
  if (act_bits != 8 && act_bits != 4) return WQ_ERR_ARG;
  WQ_TRY(check_mk(M, K));
  WQ_TRY(check_n(N));
  WQ_TRY(check_table(S, T, step));
  if (M > wq::kSingleKernelMaxM) return WQ_ERR_SHAPE;
  if (M == 0) return WQ_OK;
  if (!x || !stream_id || !table || !qw || !s_w || !y) return WQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(qw) || !aligned16(y) || !aligned16(s_w) ||
      !aligned16(stream_id) || !aligned16(table) || (thr && !aligned16(thr)) ||
      (cinv && !aligned16(cinv)) || (bias && !aligned16(bias)) || (beta && !aligned16(beta)))
    return WQ_ERR_ALIGN;
  const wq::EpilogueArgs ep{nullptr, stream_id, s_w, bias, beta, S, step};
  return from_cuda(wq::launch_linear_single(x, cinv, table, thr, act_bits, qw, M, N, K, ep, y,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

wq_status wq_gemm_w4ax(const void* qx, const float* s_tok, int act_bits, int M, int K, int N,
                       const uint8_t* stream_id, const float* beta, int S, int T, int step,
                       const uint8_t* qw, const float* s_w, const float* bias, wq_bf16* y,
                       wq_stream_t stream) {
  WQ_TRY(gemm_checks(qx, s_tok, act_bits, M, K, N, stream_id, beta, S, T, step, qw, s_w, bias,
                     y));
  const wq::EpilogueArgs ep{s_tok, stream_id, s_w, bias, beta, S, step};
  return from_cuda(wq::launch_gemm(qx, act_bits, qw, M, N, K, ep, y, nullptr,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

size_t wq_gemm_scratch_bytes(int M, int K, int N) {
  if (check_mk(M, K) != WQ_OK || check_n(N) != WQ_OK || M == 0) return 0;
  return wq::gemm_split_scratch_bytes(M, N, K);
}

wq_status wq_gemm_plan_query(int M, int K, int N, int act_bits, int call, wq_gemm_plan* plan) {
  if (!plan) return WQ_ERR_NULL;
  *plan = wq_gemm_plan{};
  if (call < WQ_PLAN_GEMM || call > WQ_PLAN_GELU_QUANT) return WQ_ERR_ARG;
  const bool gemm_only = call == WQ_PLAN_GEMM || call == WQ_PLAN_GEMM_WS;
  if (gemm_only && act_bits != 8 && act_bits != 4) return WQ_ERR_ARG;
  WQ_TRY(check_mk(M, K));
  WQ_TRY(check_n(N));
  // the fused linears keep one code per int8 byte for both widths
  const wq::GemmPlan g = wq::gemm_plan(M, N, K, gemm_only ? act_bits : 8, call != WQ_PLAN_GEMM,
                                       call == WQ_PLAN_GELU_QUANT);
  plan->tile_tokens = g.tile_tokens;
  plan->tile_channels = g.tile_channels;
  plan->ctas_per_tile = g.ctas_per_tile;
  plan->k_splits = g.k_splits;
  plan->k_stage = g.k_stage;
  plan->tiles = g.tiles;
  plan->weights_in_tmem = g.weights_in_tmem;
  return WQ_OK;
}

wq_status wq_gemm_w4ax_ws(const void* qx, const float* s_tok, int act_bits, int M, int K, int N,
                          const uint8_t* stream_id, const float* beta, int S, int T, int step,
                          const uint8_t* qw, const float* s_w, const float* bias, wq_bf16* y,
                          void* workspace, size_t ws_bytes, wq_stream_t stream) {
  WQ_TRY(gemm_checks(qx, s_tok, act_bits, M, K, N, stream_id, beta, S, T, step, qw, s_w, bias,
                     y));
  const wq::EpilogueArgs ep{s_tok, stream_id, s_w, bias, beta, S, step};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t split_bytes = M > 0 ? wq::gemm_split_scratch_bytes(M, N, K) : 0;
  wq::SplitScratch sc{nullptr, nullptr};
  if (split_bytes > 0) {
    if (!workspace) return WQ_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return WQ_ERR_ALIGN;
    if (ws_bytes < split_bytes) return WQ_ERR_ARG;
    sc = wq::split_scratch_at(workspace, M, N);
    WQ_TRY(from_cuda(cudaMemsetAsync(workspace, 0, split_bytes, st)));
  }
  return from_cuda(wq::launch_gemm(qx, act_bits, qw, M, N, K, ep, y,
                                   split_bytes > 0 ? &sc : nullptr, st));
}

wq_status wq_linear_w4a8(const wq_bf16* x, int M, int K, int N, const float* cinv,
                         const uint8_t* stream_id, const float* alpha, const float* beta,
                         int S, int T, int step, const uint8_t* qw, const float* s_w,
                         const float* bias, wq_bf16* y, void* workspace, size_t ws_bytes,
                         wq_stream_t stream) {
  return linear(x, M, K, N, cinv, stream_id, alpha, beta, S, T, step, qw, s_w, bias, y,
                workspace, ws_bytes, stream, 8);
}

wq_status wq_linear_w4a4(const wq_bf16* x, int M, int K, int N, const float* cinv,
                         const uint8_t* stream_id, const float* alpha, const float* beta,
                         int S, int T, int step, const uint8_t* qw, const float* s_w,
                         const float* bias, wq_bf16* y, void* workspace, size_t ws_bytes,
                         wq_stream_t stream) {
  return linear(x, M, K, N, cinv, stream_id, alpha, beta, S, T, step, qw, s_w, bias, y,
                workspace, ws_bytes, stream, 4);
}

wq_status wq_debug_gemm_s32(const void* qx, int act_bits, const uint8_t* qw, int M, int N,
                            int K, int32_t* acc, void* workspace, size_t ws_bytes,
                            wq_stream_t stream) {
  if (act_bits != 8 && act_bits != 4) return WQ_ERR_ARG;
  WQ_TRY(check_mk(M, K));
  WQ_TRY(check_n(N));
  if (M == 0) return WQ_OK;
  if (!qx || !qw || !acc) return WQ_ERR_NULL;
  if (!aligned16(qx) || !aligned16(qw) || !aligned16(acc)) return WQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const wq::EpilogueArgs ep{nullptr, nullptr, nullptr, nullptr, nullptr, 1, 0};
  wq::GemmExtras ex;
  ex.acc_out = acc;
  const size_t split_bytes = wq::gemm_split_scratch_bytes(M, N, K);
  wq::SplitScratch sc{nullptr, nullptr};
  if (split_bytes > 0) {  // the fused linear's split of K, through the caller's scratch
    if (!workspace) return WQ_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return WQ_ERR_ALIGN;
    if (ws_bytes < split_bytes) return WQ_ERR_ARG;
    sc = wq::split_scratch_at(workspace, M, N);
    WQ_TRY(from_cuda(cudaMemsetAsync(workspace, 0, split_bytes, st)));
  }
  return from_cuda(wq::launch_gemm(qx, act_bits, qw, M, N, K, ep, nullptr,
                                   split_bytes > 0 ? &sc : nullptr, st, false, &ex));
}

wq_status wq_debug_linear_s32(const wq_bf16* x, int M, int K, int N, const float* cinv,
                              const uint8_t* stream_id, const float* alpha, const float* beta,
                              int S, int T, int step, int act_bits, const uint8_t* qw,
                              const float* s_w, const float* bias, wq_bf16* y, int32_t* acc,
                              void* workspace, size_t ws_bytes, wq_stream_t stream) {
  if (M > 0 && !acc) return WQ_ERR_NULL;
  return linear(x, M, K, N, cinv, stream_id, alpha, beta, S, T, step, qw, s_w, bias, y,
                workspace, ws_bytes, stream, act_bits, nullptr, acc);
}

wq_status wq_linear_gelu_quant(const wq_bf16* x, int M, int K, int N, const float* cinv,
                               const uint8_t* stream_id, const float* alpha, const float* beta,
                               int S, int T, int step, int act_bits, const uint8_t* qw,
                               const float* s_w, const float* bias, const float* cinv_next,
                               const float* thr_next, const float* gain_next, int act_bits_next,
                               int8_t* codes_next, float* s_next, wq_bf16* h, void* workspace,
                               size_t ws_bytes, wq_stream_t stream) {
  if (act_bits_next != 8 && act_bits_next != 4) return WQ_ERR_ARG;
  WQ_TRY(linear_checks(x, M, K, N, cinv, stream_id, alpha, beta, S, T, step, qw, s_w, bias,
                       codes_next, workspace, ws_bytes, act_bits, nullptr));
  if (M == 0) return WQ_OK;
  if (!thr_next || !gain_next || !s_next) return WQ_ERR_NULL;
  if (!aligned16(thr_next) || !aligned16(gain_next) || !aligned16(s_next) ||
      (cinv_next && !aligned16(cinv_next)) || (h && !aligned16(h)))
    return WQ_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WQ_TRY(from_cuda(wq::ensure_gelu_table(st)));
  const Workspace w = carve(workspace, M, K, N);
  WQ_TRY(quantize_into(w, x, M, K, cinv, stream_id, alpha, S, step, act_bits, nullptr, st));
  const wq::EpilogueArgs ep{w.s_tok, stream_id, s_w, bias, beta, S, step};
  wq::GemmExtras ex;
  ex.next_thr = thr_next;
  ex.next_gain = gain_next;
  ex.next_cinv = cinv_next;
  ex.next_s = s_next;
  ex.h = h;
  return from_cuda(wq::launch_gemm_gelu_quant(w.qx, qw, M, N, K, ep, act_bits_next, codes_next,
                                              w.scratch.partial ? &w.scratch : nullptr, st,
                                              /*w_prefetch=*/true, ex));
}

wq_status wq_debug_inject_stall(int enable, unsigned limit_us) {
  const int kblock = enable ? 0 : -1;
  const unsigned long long limit =
      enable ? static_cast<unsigned long long>(limit_us) * 1000ull : wq::kWaitLimitNs;
  if (enable && limit_us == 0) return WQ_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return WQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(wq::g_wait_limit_ns, &limit, sizeof limit) != cudaSuccess ||
      cudaMemcpyToSymbol(wq::g_stall_kblock, &kblock, sizeof kblock) != cudaSuccess)
    return WQ_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_linear_w4a8_noalloc(const wq_bf16* x, int M, int K, int N, const float* cinv,
                                 const uint8_t* stream_id, const float* alpha,
                                 const float* beta, int S, int T, int step, const uint8_t* qw,
                                 const float* s_w, const float* bias, wq_bf16* y,
                                 wq_stream_t stream) {
  const size_t need = wq_workspace_bytes(M, K, N, 8);  // 0: invalid sizes, or M == 0
  if (need > kNoAllocScratchBytes) return WQ_ERR_SCRATCH;
  void* scratch = nullptr;
  if (need > 0) WQ_TRY(noalloc_scratch(&scratch));
  return linear(x, M, K, N, cinv, stream_id, alpha, beta, S, T, step, qw, s_w, bias, y, scratch,
                need > 0 ? kNoAllocScratchBytes : 0, stream, 8);
}

wq_status wq_device_status(unsigned* flags) {
  unsigned word = 0;
  const unsigned zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return WQ_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&word, wq::g_error_word, sizeof word) != cudaSuccess) return WQ_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(wq::g_error_word, &zero, sizeof zero) != cudaSuccess)
    return WQ_ERR_CUDA;
  if (flags) *flags = word;
  if (word & WQ_DEVICE_ERR_TIMEOUT) return WQ_ERR_TIMEOUT;
  if (word) return WQ_ERR_DEVICE;
  return WQ_OK;
}

}  // extern "C"
