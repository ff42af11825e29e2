/*
 * wq.h -- C ABI of the fused low-bit (W4A8 / W4A4) linear layer of SteerQuant's
 * Rudder kernels, for NVIDIA B200 (sm_100a).
 *
 * Source: "SteerQuant: Steering Quantization Error with Action-Guided Scaling in
 * World-Action Models" (paperlayer.ai abstract page 2609.39056v1), cited below by
 * section.  The method keeps ONE static int4 weight matrix per layer (§1, §4.2,
 * Figure 2) and, per layer and denoising step, a lookup table of activation clip
 * settings per token stream (video / proprio / action; §4.3).  Rudder runs two
 * fused kernels (§4.4): (1) activation quantization with the channel scaling and
 * stream gains folded in, (2) a low-bit GEMM whose epilogue applies
 * dequantization, inverse-gain compensation, bias and output compensation (§1).
 * Only integer activations and per-row scales pass between the two kernels.
 *
 * Arithmetic contract (readings where the pages are silent):
 *   x'[m,k]  = fp32(x[m,k]) * cinv[k]                        (fp32, no rounding to bf16)
 *   amax[m]  = max_k |x'[m,k]|
 *   s_tok[m] = (alpha[step][sid] * amax[m]) / qmax            qmax = 127 (A8) or 7 (A4)
 *   q[m,k]   = clamp(rint_half_even(x'[m,k] / s_tok[m]), -qmax, qmax)   (IEEE fp32 divide)
 *   acc[m,n] = sum_k q[m,k] * qw[n,k]                          (int32)
 *   y[m,n]   = bf16( s_tok[m]*s_w[n]*acc[m,n] + bias[n] + beta[step][sid][n] )
 * with sid = stream_id[m].  The stream gain is carried as the clip ratio
 * alpha = 1/gain, so the inverse-gain compensation lives inside s_tok.  A row
 * whose scale is 0 gets all-zero codes.  Codes, scales and accumulators are
 * exactly reproducible; y is computed in fp32 (one rounding to bf16 at the end).
 *
 * Packed int4 layout (weights and 4-bit activations): two's-complement nibbles,
 * two per byte, the LOW nibble holds the even k.  Row-major, K/2 bytes per row.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never frees or retains them.  Row-major, densely packed.
 *   - bf16 tensors are passed as raw 16-bit patterns (wq_bf16).
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *     Argument errors are returned synchronously before anything is launched.
 *   - Kernels are launched with programmatic stream serialization: one may start
 *     while the previous kernel in the stream finishes, but it waits for that
 *     kernel before touching memory, so stream order is preserved (and the calls
 *     can be captured in CUDA graphs).
 *   - Nothing throws or aborts across this boundary.
 *   - Preconditions checked on the host: M >= 0 (M == 0 returns WQ_OK at once
 *     after the size and table checks; token tensors may then be NULL), K a
 *     multiple of 128 with 128 <= K <= 32768, N a multiple of 16 and >= 16,
 *     1 <= S <= 255, T >= 1, 0 <= step < T, act_bits in {4, 8}, every tensor
 *     pointer 16-byte aligned, the workspace at least wq_workspace_bytes().
 *   - Precondition checked on the device: stream_id[m] < S.  A violation gives
 *     that row scale 0 and sets WQ_DEVICE_ERR_STREAM_ID (see wq_device_status).
 *   - Inputs must be finite; alpha entries must be positive.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* wq_stream_t; /* identical to cudaStream_t */
typedef uint16_t wq_bf16;                /* raw bfloat16 bit pattern */

typedef enum {
  WQ_OK = 0,
  WQ_ERR_NULL = 1,    /* a required pointer is NULL */
  WQ_ERR_SHAPE = 2,   /* M, N or K outside the supported range */
  WQ_ERR_ALIGN = 3,   /* a tensor pointer is not 16-byte aligned */
  WQ_ERR_ARG = 4,     /* bad act_bits, S, T, step, or workspace too small */
  WQ_ERR_CUDA = 5,    /* the CUDA runtime rejected a launch */
  WQ_ERR_TIMEOUT = 6, /* wq_device_status: a kernel's bounded wait gave up */
  WQ_ERR_DEVICE = 7,  /* wq_device_status: a device-side precondition failed */
  WQ_ERR_SCRATCH = 8  /* wq_linear_w4a8_noalloc: the sizes exceed its fixed scratch */
} wq_status;

/* Device error bits reported by wq_device_status(). */
#define WQ_DEVICE_ERR_TIMEOUT 1u
#define WQ_DEVICE_ERR_STREAM_ID 2u

/* Human-readable name of a status code (static string, never NULL). */
const char* wq_status_string(wq_status s);

/* ABI version of this library (major * 100 + minor; the minor number grows when
 * entry points are added, the major one when an existing signature or contract
 * changes).  101: adds wq_gemm_plan_query. */
int wq_version(void);

/* Bytes of device workspace wq_linear_w4a8 / wq_linear_w4a4 need for M token
 * rows, K input channels, N output channels: the integer activation codes
 * (M*K bytes: one code per byte for both widths, since the tensor cores take
 * int8 operands), the per-token scales (4*M bytes) and, for token counts too
 * small to fill the GPU with output tiles, the split-K scratch, each rounded
 * up to 256 bytes.  Returns 0 for invalid sizes (act_bits not 8 or 4 included). */
size_t wq_workspace_bytes(int M, int K, int N, int act_bits);

/* §4.2 (calibration side of the shared diagonal D): for each input channel k,
 * c[k] = sqrt(max_m |x_cal[m,k]| / max_n |W[n,k]|), 1 when either maximum is 0,
 * and cinv[k] = 1 / c[k], both IEEE fp32 correctly rounded.
 *   x_cal [Mcal][K] bf16 calibration activations; W [N][K] bf16 weights;
 *   c, cinv [K] fp32 outputs.  Offline (run once per layer). */
wq_status wq_channel_scale(const wq_bf16* x_cal, int Mcal, const wq_bf16* W, int N, int K,
                           float* c, float* cinv, wq_stream_t stream);

/* Figure 2 / §4.2 / §3.1: offline weight preparation.  W' = W * c (c may be
 * NULL, meaning 1), s_w[n] = max_k |W'[n,k]| / 7, qw = clamp(rint(W'/s_w), -7, 7)
 * packed two per byte.
 *   W [N][K] bf16 in; qw [N][K/2] uint8 out; s_w [N] fp32 out. */
wq_status wq_pack_int4(const wq_bf16* W, const float* c, int N, int K, uint8_t* qw,
                       float* s_w, wq_stream_t stream);

/* §4.4 first kernel: per-token activation quantization with the channel scale
 * (§4.2) and the (step, stream) clip ratio (§4.3) folded in.
 *   x [M][K] bf16; cinv [K] fp32 or NULL (= 1); stream_id [M] uint8;
 *   alpha [T][S] fp32 clip ratios; step in [0, T).
 *   act_bits 8: qx is int8 [M][K]; act_bits 4: qx is packed uint8 [M][K/2].
 *   s_tok [M] fp32 out. */
wq_status wq_act_quant(const wq_bf16* x, int M, int K, const float* cinv,
                       const uint8_t* stream_id, const float* alpha, int S, int T, int step,
                       int act_bits, void* qx, float* s_tok, wq_stream_t stream);

/* §4.4 second kernel on already-quantized activations: GEMM with int32
 * accumulation on tcgen05 tensor cores and the fused epilogue.
 *   qx: int8 [M][K] (act_bits 8) or packed [M][K/2] (act_bits 4); s_tok [M];
 *   stream_id [M]; beta [T][S][N] fp32 or NULL; qw [N][K/2]; s_w [N];
 *   bias [N] fp32 or NULL; y [M][N] bf16 out. */
wq_status wq_gemm_w4ax(const void* qx, const float* s_tok, int act_bits, int M, int K, int N,
                       const uint8_t* stream_id, const float* beta, int S, int T, int step,
                       const uint8_t* qw, const float* s_w, const float* bias, wq_bf16* y,
                       wq_stream_t stream);

/* Bytes of scratch wq_gemm_w4ax_ws uses to split K across SMs for (M, K, N): the
 * int32 partial tiles and their arrival counters, 0 when the shape does not split
 * (enough output tiles to fill the GPU).  0 for invalid sizes too. */
size_t wq_gemm_scratch_bytes(int M, int K, int N);

/* wq_gemm_w4ax with a caller workspace (device memory, 256-byte aligned, at least
 * wq_gemm_scratch_bytes(M, K, N) bytes; may be NULL when that is 0) through which
 * few-token shapes split K over every SM, as the fused linear does.  The call
 * clears the scratch on `stream` (one memset) before the GEMM; the int32 sums of
 * the splits are exact, so y is bit-identical to wq_gemm_w4ax's.  Returns
 * WQ_ERR_NULL / WQ_ERR_ALIGN / WQ_ERR_ARG for a missing, misaligned or short
 * workspace; other arguments as in wq_gemm_w4ax. */
wq_status wq_gemm_w4ax_ws(const void* qx, const float* s_tok, int act_bits, int M, int K, int N,
                          const uint8_t* stream_id, const float* beta, int S, int T, int step,
                          const uint8_t* qw, const float* s_w, const float* bias, wq_bf16* y,
                          void* workspace, size_t ws_bytes, wq_stream_t stream);

/* Which instance of the §4.4 GEMM a call runs for one shape (introspection: host
 * arithmetic only, no device work; the SM count is the current device's, 148 when
 * none is visible).  `call` names the entry point:
 *   WQ_PLAN_GEMM        wq_gemm_w4ax (K is never split);
 *   WQ_PLAN_GEMM_WS     wq_gemm_w4ax_ws and wq_debug_gemm_s32;
 *   WQ_PLAN_LINEAR      wq_linear_w4a8 / _w4a4 / _w4ax_static / _w4a8_noalloc and
 *                       wq_debug_linear_s32 (both widths keep one code per byte, so
 *                       both run the int8-activation GEMM);
 *   WQ_PLAN_GELU_QUANT  wq_linear_gelu_quant.
 * act_bits (8 or 4) is the codes' format for WQ_PLAN_GEMM and WQ_PLAN_GEMM_WS and is
 * ignored otherwise.  *plan is zeroed first, and stays zero for M == 0.  Returns
 * WQ_ERR_NULL (plan NULL), WQ_ERR_ARG (call or act_bits), WQ_ERR_SHAPE (M, K, N as
 * in wq_gemm_w4ax). */
typedef struct wq_gemm_plan {
  int tile_tokens;     /* token tile, the MMA's N: 16, 32, 64, 128, 224 or 256 */
  int tile_channels;   /* output channels per tile: 128, or 256 on a CTA pair */
  int ctas_per_tile;   /* 1, or 2 for a CTA pair (tcgen05 cta_group::2) */
  int k_splits;        /* CTAs sharing one tile's K loop (1: K not split) */
  int k_stage;         /* K depth of one pipeline stage: 128 or 256 */
  int tiles;           /* output tiles of the launch */
  int weights_in_tmem; /* 1: the unpacked int8 weight tile is the MMA's A operand in TMEM */
} wq_gemm_plan;

enum {
  WQ_PLAN_GEMM = 0,
  WQ_PLAN_GEMM_WS = 1,
  WQ_PLAN_LINEAR = 2,
  WQ_PLAN_GELU_QUANT = 3
};

wq_status wq_gemm_plan_query(int M, int K, int N, int act_bits, int call, wq_gemm_plan* plan);

/* The fused W4A8 linear: wq_act_quant (8-bit) then wq_gemm_w4ax, with the codes
 * and token scales kept in the caller's workspace (device memory of at least
 * wq_workspace_bytes(M, K, N, 8) bytes, 256-byte aligned; its contents are
 * overwritten).  Arguments as in the two calls above. */
wq_status wq_linear_w4a8(const wq_bf16* x, int M, int K, int N, const float* cinv,
                         const uint8_t* stream_id, const float* alpha, const float* beta,
                         int S, int T, int step, const uint8_t* qw, const float* s_w,
                         const float* bias, wq_bf16* y, void* workspace, size_t ws_bytes,
                         wq_stream_t stream);

/* The fused W4A4 linear: as wq_linear_w4a8 with 4-bit activation codes
 * (qmax 7; workspace of wq_workspace_bytes(M, K, N, 4) bytes, in which the
 * codes are kept one per byte, not packed as wq_act_quant writes them). */
wq_status wq_linear_w4a4(const wq_bf16* x, int M, int K, int N, const float* cinv,
                         const uint8_t* stream_id, const float* alpha, const float* beta,
                         int S, int T, int step, const uint8_t* qw, const float* s_w,
                         const float* bias, wq_bf16* y, void* workspace, size_t ws_bytes,
                         wq_stream_t stream);

/* §4.3, static reading of the layer-step table: one shared clip threshold per
 * step, thr [T] fp32, narrowed per stream by a bounded gain, gain [T][S] fp32:
 * clip = thr[step] / gain[step][stream_id[m]] (IEEE division; 0 when the gain is
 * not positive), s_tok[m] = clip / qmax, and the codes as in wq_act_quant (round
 * half to even, clamp to +-qmax).  The inverse gain stays inside s_tok, which the
 * GEMM's epilogue multiplies back (§4.4).  No row maximum is taken, so x is read
 * and quantized in one pass.  Layouts, preconditions and errors as wq_act_quant;
 * thr and gain must not be NULL. */
wq_status wq_act_quant_static(const wq_bf16* x, int M, int K, const float* cinv,
                              const uint8_t* stream_id, const float* thr, const float* gain,
                              int S, int T, int step, int act_bits, void* qx, float* s_tok,
                              wq_stream_t stream);

/* The fused W4A8 (act_bits 8) or W4A4 (act_bits 4) linear with static clipping:
 * wq_act_quant_static then the GEMM and epilogue, with the workspace of
 * wq_workspace_bytes(M, K, N, act_bits) bytes (codes one per byte, as in
 * wq_linear_w4a8 / wq_linear_w4a4).  Other arguments as wq_linear_w4a8. */
wq_status wq_linear_w4ax_static(const wq_bf16* x, int M, int K, int N, const float* cinv,
                                const uint8_t* stream_id, const float* thr, const float* gain,
                                const float* beta, int S, int T, int step, int act_bits,
                                const uint8_t* qw, const float* s_w, const float* bias,
                                wq_bf16* y, void* workspace, size_t ws_bytes,
                                wq_stream_t stream);

/* The fused linear as ONE kernel, for token counts that fit one token tile
 * (1 <= M <= 64; larger M returns WQ_ERR_SHAPE): the quantization (qmax 127 for
 * act_bits 8, 7 for act_bits 4) runs inside the GEMM, which stages the bf16
 * activations next to the weights and quantizes each K block into its
 * shared-memory operand tile, so no codes pass through device memory and no
 * workspace is needed.
 *   thr == NULL: dynamic clipping as wq_linear_w4a8 / w4a4, table = alpha [T][S].
 *     Every CTA first reads the tile's rows in full for their maxima.
 *   thr != NULL: static clipping as wq_linear_w4ax_static, table = gain [T][S]
 *     and thresholds thr [T]; no row maximum is needed.
 * The pages split the linear into two kernels (§4.4); this single-kernel form is
 * an option for tiny batches (action tokens).  Results equal the two-kernel
 * calls bit for bit.  Other arguments as wq_linear_w4a8. */
wq_status wq_linear_w4ax_single(const wq_bf16* x, int M, int K, int N, const float* cinv,
                                const uint8_t* stream_id, const float* table, const float* thr,
                                const float* beta, int S, int T, int step, int act_bits,
                                const uint8_t* qw, const float* s_w, const float* bias,
                                wq_bf16* y, wq_stream_t stream);

/* Debug view of the GEMM's integer core (§4.4): the product GEMM -- the same
 * kernel instance, pipeline and split of K as the fused linears use for these
 * sizes -- on codes qx (as in wq_gemm_w4ax), writing the int32 accumulators
 * acc [M][N] (every element) instead of y.  workspace: device memory of at least
 * wq_workspace_bytes(M, K, N, act_bits) bytes, 256-byte aligned (only its split-K
 * part is used, and only for token counts small enough to split K; it may be
 * NULL when no split is needed); its contents are overwritten. */
wq_status wq_debug_gemm_s32(const void* qx, int act_bits, const uint8_t* qw, int M, int N,
                            int K, int32_t* acc, void* workspace, size_t ws_bytes,
                            wq_stream_t stream);

/* Debug view of the fused linear: exactly wq_linear_w4a8 (act_bits 8) or
 * wq_linear_w4a4 (act_bits 4) -- the same two launches -- with the GEMM's int32
 * accumulators acc [M][N] (sum_k q[m,k] * qw[n,k]) also written.  y, the
 * workspace's codes and token scales are those of the plain call. */
wq_status wq_debug_linear_s32(const wq_bf16* x, int M, int K, int N, const float* cinv,
                              const uint8_t* stream_id, const float* alpha, const float* beta,
                              int S, int T, int step, int act_bits, const uint8_t* qw,
                              const float* s_w, const float* bias, wq_bf16* y, int32_t* acc,
                              void* workspace, size_t ws_bytes, wq_stream_t stream);

/* App. D keeps GELU in BF16 between the FFN's quantized up- and down-projections.
 * This call is the up-projection with the down-projection's activation
 * quantization moved into its epilogue, so the bf16 hidden state never goes
 * through device memory:
 *   y[m,n]  = the fused linear's output, as wq_linear_w4a8 / w4a4 compute it
 *             (bf16; act_bits of the up-projection's own activations, 8 or 4)
 *   h[m,n]  = bf16(GELU(y[m,n])), GELU(v) = v * Phi(v) with Phi the standard
 *             normal distribution function (fp32, CUDA's erfcf)
 *   s_next[m] = (thr_next[step] / gain_next[step][stream_id[m]]) / qmax_next
 *             (static clipping of §4.3 for the down-projection: IEEE divisions,
 *             0 when the gain is not positive; qmax_next 127 for act_bits_next 8,
 *             7 for 4)
 *   codes_next[m,n] = clamp(rint_half_even(h[m,n] * cinv_next[n] / s_next[m]),
 *             -qmax_next, qmax_next), int8 [M][N], one code per byte for both
 *             widths; 0 when s_next[m] is 0.
 * Dynamic clipping needs the maximum over the whole row before any code, which
 * spans every output tile, so only static clipping can be fused here.
 * The down-projection then runs wq_gemm_w4ax(codes_next, s_next, 8, ...), or
 * wq_gemm_w4ax_ws for few tokens (int8 operands for both widths; the int32 sums
 * are the same).
 *   cinv_next [N] fp32 or NULL (= 1); thr_next [T]; gain_next [T][S];
 *   s_next [M] fp32 out; h [M][N] bf16 out or NULL (a debug copy; not needed).
 * Workspace and other arguments as wq_linear_w4a8.
 * The first call on a device also builds a 7 KB table of bf16(GELU(y)) for the
 * bf16 values 2^-10 <= |y| < 16 (one small kernel on `stream`, then a wait for
 * it); make that first call outside stream capture.  (Inside a capture the table
 * kernel is captured too and reruns with every replay, which is correct but
 * slower.) */
wq_status wq_linear_gelu_quant(const wq_bf16* x, int M, int K, int N, const float* cinv,
                               const uint8_t* stream_id, const float* alpha, const float* beta,
                               int S, int T, int step, int act_bits, const uint8_t* qw,
                               const float* s_w, const float* bias, const float* cinv_next,
                               const float* thr_next, const float* gain_next, int act_bits_next,
                               int8_t* codes_next, float* s_next, wq_bf16* h, void* workspace,
                               size_t ws_bytes, wq_stream_t stream);

/* Test hook for the GEMM's bounded waits (off by default; a test of failure
 * handling, never for production).  enable != 0: in every later GEMM launch on
 * the current device, CTA 0 leaves out the activation copy of its first K block,
 * so that pipeline stage never completes, and every wait gives up after limit_us
 * microseconds (> 0) instead of 2 s.  The launch then ends with the
 * WQ_DEVICE_ERR_TIMEOUT bit set (wq_device_status), its output undefined, and the
 * GPU context intact.  enable == 0 restores both defaults.  Synchronizes the
 * device; call it with no kernel of this library running. */
wq_status wq_debug_inject_stall(int enable, unsigned limit_us);

/* The fused W4A8 linear for callers that cannot allocate device memory.  The
 * paper has no counterpart to this entry point.
 *
 * Some callers may not allocate while they run: a robot controller's real-time
 * inference loop, where cudaMalloc can synchronize the device and take an
 * unbounded time; or a host application that owns all device memory and hands
 * the library no allocator.  This call takes no workspace.  The int8 codes and
 * token scales that pass between the two kernels live instead in a fixed
 * scratch array inside the library: 16 MiB, declared at file scope, so every
 * GPU that loads the library holds it until the process exits.  No cudaMalloc,
 * cudaFree or other allocating routine is called.
 *
 * Limit: wq_workspace_bytes(M, K, N, 8) <= 16 MiB (16777216 bytes): the codes
 * (M*K bytes), the token scales (4*M bytes) and, for token counts small enough
 * to split K, the split-K scratch, each rounded up to 256 bytes.  For example,
 * at K = 4096 and N = 4096, M = 4092 tokens fits exactly and M = 4093 does not.
 * Larger sizes return WQ_ERR_SCRATCH before anything is launched.
 * The first call on a device looks up the scratch array's device address with
 * that device current (cudaGetSymbolAddress) and caches it for the process;
 * make that first call before any stream capture on the device.  A device reset
 * (cudaDeviceReset) or any other teardown of the device's primary context
 * invalidates the cached address: do not call this entry point on that device
 * after one.
 * Every call shares the one array and reuses it as it stands: each call
 * rewrites all of the scratch it reads before reading it, so nothing needs
 * clearing, but calls whose work overlaps on the GPU (concurrent streams, or
 * concurrent host threads on the same device) race on it.
 * Other arguments and all results are exactly as in wq_linear_w4a8. */
wq_status wq_linear_w4a8_noalloc(const wq_bf16* x, int M, int K, int N, const float* cinv,
                                 const uint8_t* stream_id, const float* alpha,
                                 const float* beta, int S, int T, int step, const uint8_t* qw,
                                 const float* s_w, const float* bias, wq_bf16* y,
                                 wq_stream_t stream);

/* Reads and clears the device error word of the current device (synchronizes
 * the device).  *flags receives the WQ_DEVICE_ERR_* bits seen since the last
 * call (may be NULL).  Returns WQ_OK, WQ_ERR_TIMEOUT, WQ_ERR_DEVICE or
 * WQ_ERR_CUDA.  While a WQ_DEVICE_ERR_TIMEOUT bit is set, later GEMM launches
 * stop at their first wait that does not complete at once (their outputs are
 * then undefined), so clear it before relying on further results. */
wq_status wq_device_status(unsigned* flags);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */
