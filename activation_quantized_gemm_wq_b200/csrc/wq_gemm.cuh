// The second Rudder kernel (SteerQuant §4.4): low-bit GEMM of integer activation
// codes with one static int4 weight matrix, int32 accumulation, and a fused
// epilogue doing dequantization (s_tok * s_w), bias and the per-(step, stream)
// output compensation beta (§1: Rudder fuses scaling and output compensation).
//
// sm_100a design (one persistent CTA per SM, warp-specialised):
//   warp 0      TMA producer: packed int4 weight tile [128 n][64 B] (64-byte
//               swizzle) and the activation tile [BN tokens][BK] (int8: 128-byte
//               swizzle, consumed directly by the MMA; int4: 64-byte swizzle)
//   warp 1      TMEM allocator and the single MMA-issuing thread:
//               tcgen05.mma kind::i8, M=128 (output channels), N=BN (tokens),
//               K=32 per instruction, accumulators in TMEM, double-buffered so the
//               epilogue of tile i overlaps the mainloop of tile i+1
//   unpack      int4 -> int8 conversion in shared memory, written in the 128-byte
//   warps       swizzled K-major layout the MMA descriptors expect (weights, and
//               activations when they are int4)
//   epilogue    tcgen05.ld of the accumulator, y = bf16((s_tok*s_w)*acc + bias +
//   warps       beta[step][stream][n]), staged in shared memory and written with
//               TMA stores (tails clipped by the tensor map).  A second instance
//               (EPI = 8 or 4) continues from y: h = bf16(GELU(y)), then h is
//               quantized as the NEXT linear's activation (its channel scale and
//               static clip), and int8 codes are stored instead of y.  Any instance
//               can also copy the raw int32 accumulators to a debug buffer.
// The output-channel dimension is the MMA's M ("swap AB"), so the same kernel
// serves any token count from 1 to the full batch, with token tiles of 16..256.
//
// Every mbarrier wait is bounded (see wq_ptx.cuh): on timeout the kernel raises
// a device error bit, drains, frees its TMEM and returns.
#pragma once
#include <cuda_bf16.h>

#include <mutex>

#include "wq_internal.h"
#include "wq_ptx.cuh"
#include "wq_quant.cuh"

namespace wq {

// bf16(GELU(y)) for every bf16 y with 2^-10 <= |y| < 16 (exponent field 117..130),
// indexed [sign][exponent - 117][mantissa]: the GELU-and-quantize epilogue looks
// values up here instead of evaluating erfcf for each element.  Built on the GPU
// with the fp32 arithmetic the epilogue evaluates where neither the table nor a
// closed form applies (gelu_table_kernel), so a lookup returns exactly what the
// evaluation would; below and above the table h has closed forms (emit_codes).
constexpr int kGeluTabExp0 = 117, kGeluTabExps = 14, kGeluTabEnd = kGeluTabExp0 + kGeluTabExps;
__device__ uint16_t g_gelu_tab[2 * kGeluTabExps * 128];

namespace {

__global__ void gelu_table_kernel() {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 2 * kGeluTabExps * 128) return;
  const uint32_t sign = static_cast<uint32_t>(i / (kGeluTabExps * 128));
  const uint32_t e = static_cast<uint32_t>((i / 128) % kGeluTabExps + kGeluTabExp0);
  const uint32_t bits = (sign << 15) | (e << 7) | static_cast<uint32_t>(i % 128);
  const float y = __uint_as_float(bits << 16);
  g_gelu_tab[i] = __bfloat16_as_ushort(__float2bfloat16_rn(gelu_f32(y)));
}

// h = bf16(GELU(y)) evaluated (the values the table does not cover).
__device__ __noinline__ uint32_t gelu_bf16_eval(uint32_t ybits) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(gelu_f32(__uint_as_float(ybits << 16))));
}

// The next linear's code of xv with scale sn, exactly (as the quantizer takes it):
// from the reciprocal rn where that is a finite positive scale's, else from the
// quotient.  Out of line: only elements near a half-integer, or with a bad
// scale, come here.
template <int QMAX>
__device__ __noinline__ uint32_t code_exact_next(float xv, float sn, float rn) {
  return (sn > 0.0f && isfinite(rn)) ? quantize1_recip<QMAX>(xv, sn, rn)
                                     : static_cast<uint32_t>(quantize<QMAX>(xv, sn));
}

// v clamped to [-q, q], NaN kept (PTX min/max with .NaN propagate it).
__device__ __forceinline__ float clamp_nan(float v, float q) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(v), "f"(-q));
  asm("min.NaN.f32 %0, %0, %1;" : "+f"(r) : "f"(q));
  return r;
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) {
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct TileArgs {
  void* out;  // y [M][N] bf16, or acc [M][N] int32
  int M, N, K;
  int tiles_m, tiles_n, num_tiles;
  int n_fastest;
  int splits;     // K ranges per tile (1: no split)
  int num_units;  // num_tiles * splits work units, unit = tile * splits + split
  int32_t* partial;  // bf16 split: [tiles][BN][128] int32 sums of the splits (zeroed)
  int* counters;     // split K: [tiles][kMaxEpiWarps] arrivals per epilogue-warp slice
  int w_prefetch;    // weights of the first NS K blocks loaded before griddep_wait()
  // single-kernel linear (Cfg QBITS > 0): the bf16 activations, the channel
  // scale [K] (or null) and the clip ratios [T][S] the kernel quantizes with
  const uint16_t* q_x;
  const float* q_cinv;
  const float* q_alpha;  // clip ratios [T][S]; with q_thr, the stream gains [T][S]
  const float* q_thr;    // static clipping thresholds [T], or null (dynamic)
  EpilogueArgs ep;
  int has_y;             // 0: no y / codes store (the int32 debug view alone)
  int32_t* acc_out;      // int32 [M][N] copy of the accumulators (debug), or null
  // EPI > 0: the next linear's static clipping (thr [T], gain [T][S]), its channel
  // scale [N] (or null), the codes' scales s_next [M] out, h [M][N] bf16 out or null
  const float* g_thr;
  const float* g_gain;
  const float* g_cinv;
  float* g_s;
  uint16_t* g_h;
};

// K-block range of split `sp` of `splits` (balanced).
__device__ __forceinline__ void split_range(int num_k, int splits, int sp, int& kb0, int& kb1) {
  kb0 = (sp * num_k) / splits;
  kb1 = ((sp + 1) * num_k) / splits;
}

// Upper bound on the TMA stages in flight per CTA (the shared-memory budget
// decides below it).
#ifndef WQ_MAX_STAGES
#define WQ_MAX_STAGES 8
#endif
#ifndef WQ_UNPACK_WARPS_A8
#define WQ_UNPACK_WARPS_A8 4
#endif

// QBITS > 0: the single-kernel linear for token counts that fit one tile.  The
// producer also stages the bf16 activation tile; the epilogue warps compute each
// token's scale once (its row maximum over all of K) before the first tile; the
// unpack warps quantize every K block (qmax 127 or 7) straight into the int8
// tile the MMA reads.  No codes go through HBM.
// EPI > 0: the up-projection of an FFN whose epilogue emits the down-projection's
// activation codes (qmax 127 for EPI 8, 7 for EPI 4) instead of y.
// PAIR: two CTAs (a cluster) share one tile of 256 output channels x BN tokens
// (BN = 224 with the weights in TMEM, 256 for the GELU-and-quantize epilogue)
// through the pair MMA (tcgen05 cta_group::2): each CTA unpacks its own 128
// weight rows and loads half of the token rows (BN/2), rank 0 issues the MMAs, and
// each CTA's TMEM receives the accumulators of its own 128 channels for all BN
// tokens, which its epilogue writes.  Per SM this halves the activation tile's
// copy and the tensor core's reads of it from shared memory.
// KS: 128-deep K sub-blocks per pipeline stage.  The TMA engine moves a box row by
// row, and a 64-byte row of packed weights (128 K) streams at about 40 GB/s per
// SM, a 128-byte row at about 70: narrow token tiles, whose time is the weights'
// stream, take 256-deep stages (KS = 2) so that each weight row is 128 bytes.
template <int BN_, int ACT_BITS_, int QBITS_ = 0, int EPI_ = 0, bool PAIR_ = false, int KS_ = 1>
struct Cfg {
  static constexpr int BN = BN_;
  static constexpr bool PAIR = PAIR_;
  static constexpr int BNX = PAIR ? BN / 2 : BN;  // token rows of the activation tile here
  static constexpr int TILE_N = PAIR ? 256 : 128;  // output channels per work unit
  static constexpr int ACT_BITS = ACT_BITS_;
  static constexpr int QBITS = QBITS_;
  static constexpr int QMAX = QBITS == 4 ? 7 : 127;
  static constexpr int EPI = EPI_;
  static constexpr int QMAX_NEXT = EPI == 4 ? 7 : 127;
  static_assert(QBITS == 0 || (ACT_BITS == 8 && BN <= 64),
                "the single-kernel linear quantizes into the int8 mainloop, one token tile");
  static_assert(EPI == 0 || ((EPI == 8 || EPI == 4) && QBITS == 0 && ACT_BITS == 8),
                "the GELU-and-quantize epilogue follows the int8-activation mainloop");
  static_assert(!PAIR || (QBITS == 0 && (BN == 256 || BN == 224) && ACT_BITS == 8),
                "CTA pairs serve the 224- and 256-token tiles of int8 activation codes");
  static constexpr int KS = KS_;
  static_assert(KS == 1 || (KS == 2 && !PAIR && QBITS == 0 && BN <= 64),
                "256-deep stages serve the narrow token tiles of the two-kernel path");
  static constexpr int BM = 128;       // output channels per tile (MMA M)
  static constexpr int BK = 128 * KS;  // K elements per pipeline stage
  static constexpr int UNPACK_WARPS = ACT_BITS == 4 ? 8 : WQ_UNPACK_WARPS_A8;
  // epilogue warps per TMEM lane quadrant: three for the GELU-and-quantize
  // epilogue, whose longer per-element path would otherwise outlast the mainloop
  static constexpr int EPI_PER_Q = EPI ? 3 : 2;
  static constexpr int EPI_WARPS = 4 * EPI_PER_Q;
  static_assert(EPI_WARPS <= kMaxEpiWarps, "split-K counters hold kMaxEpiWarps per tile");
  static constexpr int EPI_THREADS = EPI_WARPS * 32;
  // MMA-issuing warps.  One thread issues a K block's four MMAs and its commit in
  // about 235 cycles, and its wait (with acquire) for the unpacked operands costs
  // about 200 more while its earlier MMAs are in flight: 440 cycles per K block,
  // above the tensor work of a tile narrower than 256 tokens (4 x N/2 cycles).
  // Narrow tiles therefore spread their K blocks over several issuing warps, each
  // accumulating into its own TMEM columns; the epilogue adds the partial sums.
  // (The GELU-and-quantize epilogue's twelve warps leave registers for two.)
  static constexpr int MMA_WARPS =
      PAIR ? 1 : BN <= 64 ? (EPI || KS == 2 ? 2 : 4) : BN == 128 ? 2 : 1;
  // Warp roles: warp 0 issues TMA, warps 1..MMA_WARPS issue MMAs, then the unpack
  // warps, then the epilogue warps (EPI_PER_Q per TMEM lane quadrant, warp % 4).
  static constexpr int NUM_WARPS = 1 + MMA_WARPS + UNPACK_WARPS + EPI_WARPS;
  static constexpr int THREADS = NUM_WARPS * 32;
  // index among the MMA-issuing warps, or -1
  __device__ static int mma_index(int w) { return (w >= 1 && w <= MMA_WARPS) ? w - 1 : -1; }
  // index among the unpack warps, or -1
  __device__ static int unpack_index(int w) {
    return (w > MMA_WARPS && w <= MMA_WARPS + UNPACK_WARPS) ? w - 1 - MMA_WARPS : -1;
  }
  // index among the epilogue warps (quadrant w % 4, chunk phase e / 4), or -1
  __device__ static int epi_index(int w) {
    return (w > MMA_WARPS + UNPACK_WARPS && w < NUM_WARPS) ? w - 1 - MMA_WARPS - UNPACK_WARPS
                                                           : -1;
  }

  // ATMEM (the 256-deep stages of narrow token tiles, and the 224-token CTA pairs):
  // the unpack warps write the int8 weight tile into TMEM (tcgen05.st) and the MMA
  // reads its A operand from there.  Shared memory then carries 2 bytes per packed
  // weight byte (the copy in, the unpack's read) instead of 6 (also the int8 tile's
  // write and the MMA's read of it), which bounded the narrow tiles at about 40 GB/s
  // of weights per SM and left the wide tiles' tensor pipe waiting on shared memory.
  // A pair's TMEM then holds two 224-column accumulators and two weight tiles.
  static constexpr bool ATMEM = (KS == 2 && EPI == 0) || (PAIR && BN == 224);
  static constexpr int A_COLS = KS * 32;  // TMEM columns of one int8 weight tile
  static constexpr int WP_BYTES = BM * BK / 2;                               // packed W
  static constexpr int WU_BYTES = ATMEM ? 0 : BM * BK;                       // int8 W
  static constexpr int XS_BYTES = ACT_BITS == 8 ? BNX * BK : BNX * BK / 2;   // staged x
  static constexpr int XU_BYTES = ACT_BITS == 8 ? 0 : BNX * BK;             // int8 x (A4)
  // one 128-deep sub-block of an int8 operand tile: [rows][128 B], 128-byte swizzle
  static constexpr int SUB_W = BM * 128;
  static constexpr int SUB_X = BNX * 128;
  static constexpr int XB_BYTES = QBITS ? BN * BK * 2 : 0;                  // staged bf16 x
  static constexpr int STAGE_BYTES = WP_BYTES + (QBITS ? XB_BYTES : XS_BYTES);  // TMA bytes
  static constexpr int STAGE_SMEM = WP_BYTES + XS_BYTES + XB_BYTES;
  // Pipeline: NS TMA stages (packed weights + activation tile), NU unpacked
  // buffers, and one "MMA done with K block g" barrier per stage (a ring of NS).
  // Each MMA-issuing thread does one wait and one commit per K block of its own.
  // (224-token pairs: two 32-column weight tiles beside 2 x 224 accumulator columns)
  static constexpr int NU_BASE = PAIR && ATMEM ? 2 : (ACT_BITS == 8 && KS == 1) || ATMEM ? 3 : 2;
  static constexpr int NU = MMA_WARPS > NU_BASE ? MMA_WARPS : NU_BASE;
  static constexpr int EPI_ELEM = 2;  // bf16 y (the codes of EPI > 0 use half of it)
  // The tensor cores accumulate 16x (int8 activations) or 256x (both operands
  // unpacked from int4) the code products; see unpack32.
  static constexpr int ACC_SHIFT = ACT_BITS == 8 ? 4 : 8;
  static constexpr int EPI_CHUNK = 16;  // token columns per TMEM load / TMA store
  static constexpr int NUM_CHUNKS = BN / EPI_CHUNK;
  static constexpr int EPI_BUF_BYTES = EPI_CHUNK * 32 * EPI_ELEM;
  // staged s_tok and stream ids, x2; then (QBITS) each token's scale and its
  // reciprocal; then (EPI) the next linear's token scales and reciprocals, x2
  static constexpr int GELU_TAB_BYTES = 2 * 14 * 128 * 2;  // EPI: the GELU table, copied here
  static constexpr int TOK_BYTES = 2 * BN * 4 + 2 * BN + (QBITS ? 2 * BN * 4 : 0) +
                                   (EPI ? 2 * 2 * BN * 4 + GELU_TAB_BYTES : 0);
  static constexpr int OFF_TOK_NEXT = 2 * BN * 4 + 2 * BN + (QBITS ? 2 * BN * 4 : 0);
  static constexpr int OFF_GELU_TAB = OFF_TOK_NEXT + 2 * 2 * BN * 4;  // EPI
  static constexpr int SMEM_LIMIT = 232448;  // 227 KB opt-in per CTA
  static constexpr int RESERVED = 1024 /*alignment slack*/ + 512 /*barriers*/;
  static constexpr int FIXED = RESERVED + NU * (WU_BYTES + XU_BYTES) + TOK_BYTES;
  // double-buffered epilogue staging unless that would cost a TMA stage below 4
  static constexpr int NS_WITH_2 =
      (SMEM_LIMIT - FIXED - EPI_WARPS * 2 * EPI_BUF_BYTES) / STAGE_SMEM;
  static constexpr int EPI_NBUF = NS_WITH_2 >= 4 ? 2 : 1;
  static constexpr int EPI_BYTES = EPI_WARPS * EPI_NBUF * EPI_BUF_BYTES;
  static constexpr int NS_FIT = (SMEM_LIMIT - FIXED - EPI_BYTES) / STAGE_SMEM;
  // narrow tiles stream weights with little else to do: let more copies fly
  static constexpr int NS_CAP = BN <= 64 ? 2 * WQ_MAX_STAGES : WQ_MAX_STAGES;
  static constexpr int NS = NS_FIT > NS_CAP ? NS_CAP : NS_FIT;
  static_assert(NS >= NU && NS >= 2, "the done ring needs NS >= NU");
  static_assert(BN % EPI_CHUNK == 0 && NUM_CHUNKS >= 1, "token tile is a multiple of 16");

  static constexpr int OFF_WP = 0;
  static constexpr int OFF_XS = OFF_WP + NS * WP_BYTES;
  static constexpr int OFF_XB = OFF_XS + NS * XS_BYTES;
  static constexpr int OFF_WU = OFF_XB + NS * XB_BYTES;
  static constexpr int OFF_XU = OFF_WU + NU * WU_BYTES;
  static constexpr int OFF_EPI = OFF_XU + NU * XU_BYTES;
  static constexpr int OFF_TOK = OFF_EPI + EPI_BYTES;
  static constexpr int OFF_BAR = OFF_TOK + TOK_BYTES;
  static constexpr int NUM_BARS = 2 * NS + NU + 8;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
  static_assert(OFF_XS % 1024 == 0 && XS_BYTES % 512 == 0 && OFF_WU % 1024 == 0 &&
                    OFF_XU % 1024 == 0 && OFF_EPI % 1024 == 0 && OFF_BAR % 8 == 0,
                "swizzled tiles need 1024-byte alignment");

  // two tile buffers x MMA_WARPS partial accumulators of BN columns
  static constexpr int ACC_COLS = 2 * MMA_WARPS * BN;
  // ATMEM: NU int8 weight tiles after the accumulators
  static constexpr int A_COL0 = ACC_COLS;
  static constexpr int USED_COLS = ACC_COLS + (ATMEM ? NU * A_COLS : 0);
  static_assert(USED_COLS <= 512, "TMEM holds 512 columns");
  static constexpr uint32_t TMEM_COLS = USED_COLS <= 32    ? 32
                                        : USED_COLS <= 64  ? 64
                                        : USED_COLS <= 128 ? 128
                                        : USED_COLS <= 256 ? 256
                                                           : 512;
  static_assert(!ATMEM || UNPACK_WARPS % 4 == 0, "unpack warps cover the lane quadrants");
};

__device__ __forceinline__ void decode_tile(const TileArgs& a, int tile, int& n_tile,
                                            int& m_tile) {
  if (a.n_fastest) {
    n_tile = tile % a.tiles_n;
    m_tile = tile / a.tiles_n;
  } else {
    m_tile = tile % a.tiles_m;
    n_tile = tile / a.tiles_m;
  }
}

// 16 packed bytes (32 int4 codes, low nibble first) -> 32 bytes holding 16 * code,
// in k order.  Moving each nibble into the high half of its byte makes the byte
// the two's-complement value 16 * code, so no sign extension is needed; the
// factor 16 per unpacked operand is exact in int32 and is divided out in the
// epilogue.
// NATURAL = false leaves each group of 8 codes in the order 0 2 4 6 1 3 5 7:
// valid when both MMA operands are unpacked the same way (a common permutation of
// k does not change the dot product), and two byte permutes cheaper per word.
template <bool NATURAL>
__device__ __forceinline__ void unpack32(const uint4 p, uint4& lo16, uint4& hi16) {
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t e = (w[i] << 4) & 0xF0F0F0F0u;  // 16 * codes k0 k2 k4 k6
    const uint32_t f = w[i] & 0xF0F0F0F0u;         // 16 * codes k1 k3 k5 k7
    if constexpr (NATURAL) {
      o[2 * i] = __byte_perm(e, f, 0x5140);        // k0 k1 k2 k3
      o[2 * i + 1] = __byte_perm(e, f, 0x7362);    // k4 k5 k6 k7
    } else {
      o[2 * i] = e;
      o[2 * i + 1] = f;
    }
  }
  lo16 = make_uint4(o[0], o[1], o[2], o[3]);
  hi16 = make_uint4(o[4], o[5], o[6], o[7]);
}

// Packed tile [ROWS][64 KS bytes] (KS = 1: 64-byte rows, 64-byte swizzle; KS = 2:
// 128-byte rows, 128-byte swizzle) -> KS int8 sub-tiles [ROWS][128 B] with the
// 128-byte swizzle, ROWS * 128 bytes apart.  Task i covers row i / (4 KS), packed
// 16-byte chunk p = i % (4 KS), which holds k = 32p .. 32p + 31: sub-tile p / 4.
// Each thread issues all of its loads before converting (latency hiding).
template <int ROWS, int NT, bool NATURAL, int KS = 1>
__device__ __forceinline__ void unpack_tile(const uint8_t* src, uint8_t* dst, int tid) {
  constexpr int CPR = 4 * KS;  // packed chunks per row
  constexpr int TASKS = ROWS * CPR;
  constexpr int PER = (TASKS + NT - 1) / NT;
  uint4 v[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = tid + k * NT;
    if (TASKS % NT == 0 || i < TASKS) {
      const int r = i / CPR, p = i % CPR;
      const int sw = KS == 1 ? (p ^ ((r >> 1) & 3)) : (p ^ (r & 7));
      v[k] = *reinterpret_cast<const uint4*>(src + r * (16 * CPR) + (sw << 4));
    }
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = tid + k * NT;
    if (TASKS % NT == 0 || i < TASKS) {
      const int r = i / CPR, p = i % CPR, pp = p & 3;
      uint4 lo, hi;
      unpack32<NATURAL>(v[k], lo, hi);
      uint8_t* row = dst + (p >> 2) * (ROWS * 128) + r * 128;
      *reinterpret_cast<uint4*>(row + (((2 * pp) ^ (r & 7)) << 4)) = lo;
      *reinterpret_cast<uint4*>(row + (((2 * pp + 1) ^ (r & 7)) << 4)) = hi;
    }
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                const __grid_constant__ CUtensorMap tm_out, const TileArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // TMA landed, stage s
  uint64_t* done = full + C::NS;     // MMA finished K block g, slot g % NS (one commit)
  uint64_t* ufull = done + C::NS;    // unpacked buffer u ready
  uint64_t* tfull = ufull + C::NU;
  uint64_t* tempty = tfull + 2;
  uint64_t* tokbar = tempty + 2;  // epilogue warps: token staging of buffer i complete
  uint64_t* qready = tokbar + 2;  // QBITS: every token scale of the tile is in shared memory
  uint64_t* mma_drained = qready + 1;  // every MMA this CTA issued has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_drained + 1);
  float* q_s = reinterpret_cast<float*>(smem + C::OFF_TOK + 2 * C::BN * 4 + 2 * C::BN);
  float* q_r = q_s + C::BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_k = args.K / C::BK;
  // work units: one per CTA, or one per CTA pair (rank 0 issues the pair's MMAs)
  const uint32_t rank = C::PAIR ? cluster_ctarank() : 0u;
  const int unit0 = C::PAIR ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int ustep = C::PAIR ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&done[s], 1);
    }
    // a pair's unpack and epilogue warps of both CTAs arrive on rank 0's barriers
    for (int u = 0; u < C::NU; ++u) mbar_init(&ufull[u], C::UNPACK_WARPS * (C::PAIR ? 2 : 1));
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], C::MMA_WARPS);
      mbar_init(&tempty[b], C::EPI_WARPS * (C::PAIR ? 2 : 1));
      mbar_init(&tokbar[b], C::EPI_WARPS);
    }
    mbar_init(qready, C::EPI_WARPS);
    mbar_init(mma_drained, C::MMA_WARPS);
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == 1) {
    if constexpr (C::PAIR) {
      tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (C::PAIR) cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // Every CTA of this grid is resident (at most one per SM): the next kernel may
  // be launched now; it waits for this one before touching its data.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // K block g (counted over all of this CTA's tiles) goes to stage g % NS once
    // the MMA has finished K block g - NS, the previous user of that stage.
    if (lane == 0) {
      // The first NS stages' weights do not depend on the previous kernel when
      // the caller says so: start streaming them before waiting for it.
      uint32_t pre = 0;
      if (args.w_prefetch) {
        for (int unit = unit0; unit < args.num_units && pre < C::NS; unit += ustep) {
          int n_tile, m_tile, kb0, kb1;
          decode_tile(args, unit / args.splits, n_tile, m_tile);
          split_range(num_k, args.splits, unit % args.splits, kb0, kb1);
          for (int kb = kb0; kb < kb1 && pre < C::NS; ++kb, ++pre) {
            mbar_arrive_expect_tx(&full[pre], C::STAGE_BYTES);
            tma_load_2d(smem + C::OFF_WP + pre * C::WP_BYTES, &tm_w, &full[pre],
                        kb * (C::BK / 2), n_tile * C::TILE_N + rank * C::BM);
          }
        }
      }
      griddep_wait();
      // test hook (normally -1): K block whose activation copy CTA 0 leaves out
      const int stall = blockIdx.x == 0 ? *reinterpret_cast<volatile int*>(&g_stall_kblock) : -1;
      uint32_t g = 0;
      bool ok = true;
      for (int unit = unit0; ok && unit < args.num_units; unit += ustep) {
        int n_tile, m_tile, kb0, kb1;
        decode_tile(args, unit / args.splits, n_tile, m_tile);
        split_range(num_k, args.splits, unit % args.splits, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const uint32_t s = g % C::NS;
          if (g >= pre) {  // else: expect_tx and the weight load were issued above
            if (g >= static_cast<uint32_t>(C::NS) &&
                !mbar_wait(&done[s], ((g / C::NS) - 1) & 1u)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
            tma_load_2d(smem + C::OFF_WP + s * C::WP_BYTES, &tm_w, &full[s], kb * (C::BK / 2),
                        n_tile * C::TILE_N + rank * C::BM);
          }
          if (static_cast<int>(g) == stall) {
            // leave the stage one copy short: its phase never completes
          } else if constexpr (C::QBITS > 0) {  // bf16 x, two boxes of 64 channels
            tma_load_2d(smem + C::OFF_XB + s * C::XB_BYTES, &tm_x, &full[s], kb * C::BK,
                        m_tile * C::BN);
            tma_load_2d(smem + C::OFF_XB + s * C::XB_BYTES + C::BN * 128, &tm_x, &full[s],
                        kb * C::BK + 64, m_tile * C::BN);
          } else if constexpr (C::ACT_BITS == 8) {  // KS boxes of 128 channels
#pragma unroll
            for (int i = 0; i < C::KS; ++i)
              tma_load_2d(smem + C::OFF_XS + s * C::XS_BYTES + i * C::SUB_X, &tm_x, &full[s],
                          kb * C::BK + i * 128, m_tile * C::BN + rank * C::BNX);
          } else {  // packed int4: one box of BK / 2 bytes per token row
            tma_load_2d(smem + C::OFF_XS + s * C::XS_BYTES, &tm_x, &full[s], kb * (C::BK / 2),
                        m_tile * C::BN + rank * C::BNX);
          }
        }
      }
      // Drain: the copies of every issued stage must have landed before the CTA
      // exits (normally all were consumed already and these waits return at once;
      // after an error elsewhere they still wait, bounded, for copies in flight).
      // The stage the test hook left short never completes and is not waited for.
      for (uint32_t i = 0; i < static_cast<uint32_t>(C::NS) && i < g; ++i) {
        const uint32_t j = g - 1 - i;
        if (static_cast<int>(j) != stall) mbar_wait_drain(&full[j % C::NS], (j / C::NS) & 1u);
      }
    }
    __syncwarp();
  } else if (C::mma_index(warp) >= 0) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer i takes the K blocks kb0 + i, kb0 + i + MMA_WARPS, ... of each tile
    // into its own accumulator.  Per K block: one wait (its unpacked buffer; the
    // unpack warps arrive there only after the stage's TMA landed, which orders
    // the activation tile too), four MMAs, one commit (frees the stage and the
    // unpacked buffer).  Every issuer commits the tile's tfull once.
    const int mi = C::mma_index(warp);
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_i8(C::BN, C::PAIR ? 256u : 128u);
      uint32_t g = 0;
      int b = 0;
      uint32_t ph_b = 0;
      bool ok = true;
      for (int unit = unit0; ok && unit < args.num_units; unit += ustep) {
        int kb0, kb1;
        split_range(num_k, args.splits, unit % args.splits, kb0, kb1);
        if (!mbar_wait(&tempty[b], ph_b ^ 1u)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem =
            tmem_base + static_cast<uint32_t>((b * C::MMA_WARPS + mi) * C::BN);
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          if ((kb - kb0) % C::MMA_WARPS != mi) continue;
          const uint32_t s = g % C::NS, u = g % C::NU;
          if (!mbar_wait(&ufull[u], (g / C::NU) & 1u)) { ok = false; break; }
          tc_fence_after();
          const uint32_t b_addr =
              C::ACT_BITS == 8 ? smem_u32(smem + C::OFF_XS + s * C::XS_BYTES)
                               : smem_u32(smem + C::OFF_XU + u * C::XU_BYTES);
          const uint32_t a_addr = smem_u32(smem + C::OFF_WU + u * C::WU_BYTES);
          // ATMEM: the int8 weight tile u in TMEM, 8 columns per 32-deep MMA
          const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(C::A_COL0 + u * C::A_COLS);
#pragma unroll
          for (int kk = 0; kk < C::BK / 32; ++kk) {  // sub-block kk / 4, 32 deep each
            const uint64_t bd = smem_desc_sw128(b_addr + (kk >> 2) * C::SUB_X + (kk & 3) * 32);
            const uint32_t acc = (kb - kb0 >= C::MMA_WARPS || kk != 0) ? 1u : 0u;
            if constexpr (C::ATMEM && C::PAIR) {
              mma_i8_ts_pair(d_tmem, a_tmem + static_cast<uint32_t>(kk * 8), bd, idesc, acc);
            } else if constexpr (C::ATMEM) {
              mma_i8_ts(d_tmem, a_tmem + static_cast<uint32_t>(kk * 8), bd, idesc, acc);
            } else {
              const uint64_t ad =
                  smem_desc_sw128(a_addr + (kk >> 2) * C::SUB_W + (kk & 3) * 32);
              if constexpr (C::PAIR) mma_i8_ss_pair(d_tmem, ad, bd, idesc, acc);
              else mma_i8_ss(d_tmem, ad, bd, idesc, acc);
            }
          }
          if constexpr (C::PAIR) mma_commit_pair(&done[s], 3);  // both CTAs' stage s
          else mma_commit(&done[s]);
        }
        if (!ok) break;
        if constexpr (C::PAIR) mma_commit_pair(&tfull[b], 3);
        else mma_commit(&tfull[b]);
        if (++b == 2) { b = 0; ph_b ^= 1u; }
      }
      // Every MMA issued has completed before the TMEM is freed (after an error the
      // epilogue may not have waited for the last ones).
      if constexpr (C::PAIR) mma_commit_pair(mma_drained, 1);
      else mma_commit(mma_drained);
      mbar_wait_drain(mma_drained, 0);
    }
    __syncwarp();
  } else if (C::unpack_index(warp) >= 0) {
    // ------------------------------------------------------------ int4 -> int8
    // K block g: wait for its TMA stage and for the MMA to have finished K block
    // g - NU (the previous user of unpacked buffer g % NU).
    const int tid = C::unpack_index(warp) * 32 + lane;
    constexpr int NT = C::UNPACK_WARPS * 32;
    uint32_t g = 0;
    bool ok = true;
    if constexpr (C::QBITS > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(qready, 0));
    for (int unit = unit0; ok && unit < args.num_units; unit += ustep) {
      int kb0, kb1;
      split_range(num_k, args.splits, unit % args.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const uint32_t s = g % C::NS, u = g % C::NU;
        bool w = mbar_wait(&full[s], (g / C::NS) & 1u);
        if (g >= static_cast<uint32_t>(C::NU)) {
          const uint32_t j = g - C::NU;
          w = w && mbar_wait(&done[j % C::NS], (j / C::NS) & 1u);
        }
        if (!__all_sync(0xFFFFFFFFu, w)) {  // keep the warp's decision uniform
          ok = false;
          break;
        }
        // int8 activations arrive in k order, so the weights must too; int4
        // activations are unpacked exactly like the weights, so both may keep
        // the cheaper permuted order.
        if constexpr (C::ATMEM) {
          // Weight row r = 32q + lane of the tile, q = warp % 4 (the TMEM lane quadrant
          // this warp reaches); with 8 unpack warps two share a quadrant, each taking
          // half of the row's 16-byte packed chunks.  Chunk p (128-byte swizzle) holds
          // k = 32p .. 32p + 31: columns 8p .. 8p + 7 of the tile in TMEM.
          constexpr int PER_Q = C::UNPACK_WARPS / 4;
          constexpr int CH = 4 * C::KS / PER_Q;
          static_assert(CH % 2 == 0, "16-column TMEM stores");
          tc_fence_after();  // the MMA that read this tile before has completed
          const int q = warp & 3, part = C::unpack_index(warp) / 4;
          const int r = q * 32 + lane;
          const uint8_t* src = smem + C::OFF_WP + s * C::WP_BYTES + r * (C::BK / 2);
          uint4 v[CH];
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const int p = part * CH + i;
            // 64-byte rows: 64-byte swizzle; 128-byte rows: 128-byte swizzle
            const int sw = C::KS == 1 ? (p ^ ((r >> 1) & 3)) : (p ^ (r & 7));
            v[i] = *reinterpret_cast<const uint4*>(src + (sw << 4));
          }
          const uint32_t ta = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                              static_cast<uint32_t>(C::A_COL0 + u * C::A_COLS + part * CH * 8);
#pragma unroll
          for (int i = 0; i < CH; i += 2) {
            uint32_t w[16];
            uint4 lo, hi;
            unpack32<C::ACT_BITS == 8>(v[i], lo, hi);
            w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
            w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
            unpack32<C::ACT_BITS == 8>(v[i + 1], lo, hi);
            w[8] = lo.x; w[9] = lo.y; w[10] = lo.z; w[11] = lo.w;
            w[12] = hi.x; w[13] = hi.y; w[14] = hi.z; w[15] = hi.w;
            tmem_st_32x32b_x16(ta + static_cast<uint32_t>(i * 8), w);
          }
          tmem_wait_st();
          tc_fence_before();  // the stores, before the arrival the MMA waits for
        } else {
          unpack_tile<C::BM, NT, C::ACT_BITS == 8, C::KS>(smem + C::OFF_WP + s * C::WP_BYTES,
                                                          smem + C::OFF_WU + u * C::WU_BYTES,
                                                          tid);
        }
        if constexpr (C::ACT_BITS == 4) {
          unpack_tile<C::BNX, NT, false, C::KS>(smem + C::OFF_XS + s * C::XS_BYTES,
                                                smem + C::OFF_XU + u * C::XU_BYTES, tid);
        }
        if constexpr (C::QBITS > 0) {
          // chunk i: token row i / 16, channels 8*(i % 16) .. +7 of this K block
          const uint8_t* xb = smem + C::OFF_XB + s * C::XB_BYTES;
          uint8_t* xs = smem + C::OFF_XS + s * C::XS_BYTES;
          for (int i = tid; i < C::BN * 16; i += NT) {
            const int m = i >> 4, j = i & 15;
            const uint4 raw = *reinterpret_cast<const uint4*>(xb + (j >> 3) * (C::BN * 128) +
                                                               m * 128 + (j & 7) * 16);
            const int k0 = kb * C::BK + 8 * j;
            float ci[8];
            if (args.q_cinv) {
              const float4 a = __ldg(reinterpret_cast<const float4*>(args.q_cinv + k0));
              const float4 b = __ldg(reinterpret_cast<const float4*>(args.q_cinv + k0 + 4));
              ci[0] = a.x; ci[1] = a.y; ci[2] = a.z; ci[3] = a.w;
              ci[4] = b.x; ci[5] = b.y; ci[6] = b.z; ci[7] = b.w;
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) ci[e] = 1.0f;
            }
            float v[8];
            scale8(raw, ci, v);
            const float sm = q_s[m], rm = q_r[m];
            uint32_t q[8];
            if (sm > 0.0f && isfinite(rm)) {
              quantize8_recip<C::QMAX>(v, sm, rm, q);
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) q[e] = static_cast<uint32_t>(quantize<C::QMAX>(v[e], sm));
            }
            // 8 codes -> bytes 8*(j%2) .. of 16-byte chunk j/2 of row m (128-byte swizzle)
            *reinterpret_cast<uint2*>(xs + m * 128 + (((j >> 1) ^ (m & 7)) << 4) + (j & 1) * 8) =
                make_uint2(pack_low_bytes(q[0], q[1], q[2], q[3]),
                           pack_low_bytes(q[4], q[5], q[6], q[7]));
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        __syncwarp();
        if (lane == 0) {
          if constexpr (C::PAIR) mbar_arrive_cluster(mapa_shared(&ufull[u], 0));
          else mbar_arrive(&ufull[u]);
        }
      }
    }
  } else if (C::epi_index(warp) >= 0) {
    // ------------------------------------------------------------ epilogue
    // Warp e covers TMEM lanes 32q..32q+31 (output channels) and every other
    // 16-column chunk (tokens) of the tile, starting at chunk h.
    const int e = C::epi_index(warp);
    const int q = warp & 3;
    const int h = e >> 2;
    const int et = e * 32 + lane;
    uint8_t* ebuf = smem + C::OFF_EPI + e * C::EPI_NBUF * C::EPI_BUF_BYTES;
    float* tok_s = reinterpret_cast<float*>(smem + C::OFF_TOK);
    uint8_t* tok_id = smem + C::OFF_TOK + 2 * C::BN * 4;
    int b = 0, buf = 0, it = 0;
    uint32_t ph_b = 0;
    const EpilogueArgs& ep = args.ep;
    const bool small_s = ep.S <= 4;
    griddep_wait();  // token scales and split-K scratch come from the previous kernel
    if constexpr (C::QBITS > 0) {
      // Token scales of the (single) token tile: the 256 epilogue threads split
      // into BN groups of 256/BN lanes (within one warp), one token row per group;
      // s = alpha[step][stream] * max_k |x * cinv| / qmax, over all of K.
      constexpr int TPR = C::EPI_THREADS / C::BN;  // 4, 8 or 16 lanes per row
      const int m = et / TPR, part = et % TPR;
      const int nchunk = args.K >> 3;
      float amax = 0.0f;
      if (m < args.M && args.q_thr == nullptr) {  // static clipping needs no row maximum
        const uint4* xr = reinterpret_cast<const uint4*>(args.q_x + (size_t)m * args.K);
#pragma unroll 4
        for (int c = part; c < nchunk; c += TPR) {
          float ci[8], v[8];
          if (args.q_cinv) {
            const float4 a = __ldg(reinterpret_cast<const float4*>(args.q_cinv) + 2 * c);
            const float4 b = __ldg(reinterpret_cast<const float4*>(args.q_cinv) + 2 * c + 1);
            ci[0] = a.x; ci[1] = a.y; ci[2] = a.z; ci[3] = a.w;
            ci[4] = b.x; ci[5] = b.y; ci[6] = b.z; ci[7] = b.w;
          } else {
#pragma unroll
            for (int t = 0; t < 8; ++t) ci[t] = 1.0f;
          }
          scale8(__ldg(xr + c), ci, v);
#pragma unroll
          for (int t = 0; t < 8; ++t) amax = fmaxf(amax, fabsf(v[t]));
        }
      }
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1)  // within the row's lane group
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (part == 0) {
        float s_m = 0.0f;
        if (m < args.M) {
          const int sid = ep.stream_id[m];
          if (sid < ep.S) {
            const float tab = __ldg(args.q_alpha + ep.step * ep.S + sid);
            float clip;
            if (args.q_thr)  // clip = threshold / stream gain (0 when the gain is not positive)
              clip = tab > 0.0f ? __fdiv_rn(__ldg(args.q_thr + ep.step), tab) : 0.0f;
            else
              clip = __fmul_rn(tab, amax);
            s_m = __fdiv_rn(clip, static_cast<float>(C::QMAX));
          } else {
            raise_error(kErrBadStreamId);
          }
        }
        q_s[m] = s_m;
        q_r[m] = s_m > 0.0f ? __frcp_rn(s_m) : 0.0f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(qready);
      // every row's scale staged (after a timeout the waits below give up too)
      __all_sync(0xFFFFFFFFu, mbar_wait(qready, 0));
    }
    if constexpr (C::EPI > 0) {  // the GELU table into shared memory (read only below)
      uint32_t* tab_s = reinterpret_cast<uint32_t*>(smem + C::OFF_TOK + C::OFF_GELU_TAB);
      const uint32_t* tab_g = reinterpret_cast<const uint32_t*>(g_gelu_tab);
      for (int i = et; i < C::GELU_TAB_BYTES / 4; i += C::EPI_THREADS) tab_s[i] = tab_g[i];
    }
    const bool split = args.splits > 1;
    // y (or the next linear's codes) is written unless this is the int32 debug view
    const bool has_out = args.has_y != 0;
    float* nxt_s = reinterpret_cast<float*>(smem + C::OFF_TOK + C::OFF_TOK_NEXT);  // EPI
    for (int unit = unit0; unit < args.num_units; unit += ustep, ++it) {
      const int tile = unit / args.splits;
      int n_tile, m_tile;
      decode_tile(args, tile, n_tile, m_tile);
      const int n_base = n_tile * C::TILE_N + static_cast<int>(rank) * C::BM + q * 32;
      const int n = n_base + lane;
      const int m0 = m_tile * C::BN;
      float* sts = tok_s + (it & 1) * C::BN;
      uint8_t* sds = tok_id + (it & 1) * C::BN;
      float* g_s = nxt_s + (it & 1) * 2 * C::BN;  // EPI: next scale [BN], reciprocal [BN]
      // per-lane channel constants; bias and the compensation of each stream
      // combined once per tile.  A stream id >= S (a precondition violation the
      // quantizer reports) gets the bias alone: no table row is read for it.
      float sw = 0.0f, bs = 0.0f, bb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      float g_ci = 1.0f;  // EPI: the next linear's channel scale at channel n
      if (has_out) {
        for (int i = et; i < C::BN; i += C::EPI_THREADS) {
          const int m = m0 + i;
          if constexpr (C::QBITS > 0) sts[i] = q_s[i];  // the single token tile
          else sts[i] = m < args.M ? ep.s_tok[m] : 0.0f;
          const int sd = m < args.M ? ep.stream_id[m] : 0;
          sds[i] = static_cast<uint8_t>(sd);
          if constexpr (C::EPI > 0) {
            // static clip of the next linear: thr[step] / gain[step][stream]
            float sn = 0.0f;
            if (m < args.M && sd < ep.S) {
              const float gn = __ldg(args.g_gain + ep.step * ep.S + sd);
              const float clip = gn > 0.0f ? __fdiv_rn(__ldg(args.g_thr + ep.step), gn) : 0.0f;
              sn = __fdiv_rn(clip, static_cast<float>(C::QMAX_NEXT));
            }
            g_s[i] = sn;
            const float rn = sn > 0.0f ? __frcp_rn(sn) : 0.0f;
            g_s[C::BN + i] = sn > 0.0f && isfinite(rn) ? rn : __int_as_float(0x7FC00000);
            if (n_tile == 0 && unit % args.splits == 0 && m < args.M) args.g_s[m] = sn;
          }
        }
        if (n < args.N) {
          sw = ldexpf(ep.s_w[n], -C::ACC_SHIFT);  // exact power-of-two rescale
          bs = ep.bias ? ep.bias[n] : 0.0f;
          const float* brow = ep.beta ? ep.beta + (size_t)ep.step * ep.S * args.N + n : nullptr;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            bb[j] = (brow && j < ep.S && small_s) ? __fadd_rn(bs, brow[(size_t)j * args.N]) : bs;
          if constexpr (C::EPI > 0) g_ci = args.g_cinv ? args.g_cinv[n] : 1.0f;
        }
      }

      // bias + compensation of token stream sd at this lane's channel
      auto offset = [&](int sd) -> float {
        if (sd >= ep.S) return bs;
        if (small_s) return sd == 0 ? bb[0] : sd == 1 ? bb[1] : sd == 2 ? bb[2] : bb[3];
        return (ep.beta && n < args.N)
                   ? __fadd_rn(bs, ep.beta[((size_t)ep.step * ep.S + sd) * args.N + n])
                   : bs;
      };

      // This chunk's staging buffer, once its previous TMA store has read it.
      auto stage_buf = [&]() -> uint8_t* {
        uint8_t* sb = ebuf + buf * C::EPI_BUF_BYTES;
        if (lane == 0) {
          if constexpr (C::EPI_NBUF == 2) bulk_wait_group_read<1>();
          else bulk_wait_group_read<0>();
        }
        __syncwarp();
        return sb;
      };
      auto store_buf = [&](uint8_t* sb, int j0) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && n_base < args.N) {
          tma_store_2d(&tm_out, sb, n_base, m0 + j0);
          bulk_commit_group();
        }
        if constexpr (C::EPI_NBUF == 2) buf ^= 1;
      };

      // y for one 16-column chunk of accumulators (scaled by 2^ACC_SHIFT), through a
      // shared-memory staging buffer and a TMA store.
      auto emit_y = [&](const uint32_t (&r)[16], int j0) {
        uint8_t* sb = stage_buf();
        __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(sb);
        const float4* st4 = reinterpret_cast<const float4*>(sts + j0);
        const int sd_l = sds[j0 + (lane & 15)];
        const int sd0 = sds[j0];
        if (small_s && __all_sync(0xFFFFFFFFu, sd_l == sd0)) {
          // one stream in the whole chunk (the common case: streams are runs of rows)
          const float bsel = offset(sd0);
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 t = st4[j4];
            const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int j = 4 * j4 + k;
              const float v = fmaf(tv[k] * sw, __int2float_rn(static_cast<int>(r[j])), bsel);
              ob[j * 32 + lane] = __float2bfloat16_rn(v);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float v =
                fmaf(sts[j0 + j] * sw, __int2float_rn(static_cast<int>(r[j])), offset(sds[j0 + j]));
            ob[j * 32 + lane] = __float2bfloat16_rn(v);
          }
        }
        store_buf(sb, j0);
      };

      // EPI > 0: y as above, then h = bf16(GELU(y)) and the next linear's code of
      // h * cinv_next[n] with its static scale, staged as int8 [16 tokens][32
      // channels] and written with a TMA store; h itself only to the debug buffer.
      // The 16 elements go through each step together, two at a time in packed
      // fp32x2 arithmetic (the same IEEE roundings per element) and without a
      // branch inside a step; the rare cases (a value outside the GELU table, a code
      // near a half-integer, a zero, tiny or infinite scale, whose reciprocal is
      // staged as NaN) take a second pass that calls out of line.
      auto emit_codes = [&](const uint32_t (&r)[16], int j0) {
        uint8_t* sb = stage_buf();
        const uint16_t* tab = reinterpret_cast<const uint16_t*>(smem + C::OFF_TOK + C::OFF_GELU_TAB);
        float off[16];
        const int sd_l = sds[j0 + (lane & 15)];
        const int sd0 = sds[j0];
        if (__all_sync(0xFFFFFFFFu, sd_l == sd0)) {  // one stream in the chunk (the usual case)
          const float o = offset(sd0);
#pragma unroll
          for (int j = 0; j < 16; ++j) off[j] = o;
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) off[j] = offset(sds[j0 + j]);
        }
        const float4* st4 = reinterpret_cast<const float4*>(sts + j0);
        const float2 sw2 = make_float2(sw, sw);
        uint32_t hb[16];
        uint32_t rare = 0;
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          const float4 t = st4[j4];
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            const int j = 4 * j4 + 2 * p;
            const float2 s2 = __fmul2_rn(p ? make_float2(t.z, t.w) : make_float2(t.x, t.y), sw2);
            const float2 a2 = make_float2(__int2float_rn(static_cast<int>(r[j])),
                                          __int2float_rn(static_cast<int>(r[j + 1])));
            const float2 v2 = __ffma2_rn(s2, a2, make_float2(off[j], off[j + 1]));
            const uint32_t y2 = bf162_bits(__floats2bfloat162_rn(v2.x, v2.y));
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const uint32_t yb = k ? y2 >> 16 : y2 & 0xFFFFu;
              // table row: exponent field kGeluTabExp0.., either sign
              const uint32_t mag = yb & 0x7FFFu;
              const uint32_t u = mag - (kGeluTabExp0 << 7);
              const bool in = u < static_cast<uint32_t>(kGeluTabExps * 128);
              const uint32_t ti = in ? u + (yb >> 15) * (kGeluTabExps * 128) : 0u;
              const uint32_t hv = tab[ti];
              // Outside the table, the correctly rounded GELU in closed form:
              //  * normal |y| < 2^-10: GELU(y) = y/2 (1 + erf(y/sqrt2)) with
              //    |erf(y/sqrt2)| < 0.0008, under half of bf16's relative spacing (2^-9),
              //    so h = y/2 exactly: the exponent field minus one;
              //  * finite |y| >= 16: 1 - Phi(16) < 2^-60, so h = y for y > 0, and h = -0
              //    for y < 0 (|GELU(y)| < 2^-180, far below bf16's smallest subnormal).
              // Zeros, subnormals, infinities and NaN are evaluated.
              const bool tiny = mag - 0x100u < (kGeluTabExp0 << 7) - 0x100u;
              const bool wide = mag - (kGeluTabEnd << 7) < 0x7F80u - (kGeluTabEnd << 7);
              const uint32_t hx = tiny ? yb - 0x80u : yb & (0xFFFFu ^ ((yb >> 15) * 0x7FFFu));
              hb[j + k] = in               ? hv
                          : (tiny || wide) ? hx
                                           : (yb | 0x80000000u);  // high bit: evaluate below
              rare |= hb[j + k];
            }
          }
        }
        if (rare & 0x80000000u) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (hb[j] & 0x80000000u) hb[j] = gelu_bf16_eval(hb[j] & 0xFFFFu);
        }
        if (args.g_h != nullptr && n < args.N) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (m0 + j0 + j < args.M) args.g_h[(size_t)(m0 + j0 + j) * args.N + n] = hb[j];
        }
        constexpr float kq = static_cast<float>(C::QMAX_NEXT);
        const float4* rn4 = reinterpret_cast<const float4*>(g_s + C::BN + j0);
        const float2 ci2 = make_float2(g_ci, g_ci);
        const float2 m2 = make_float2(kRoundMagic, kRoundMagic);
        const float2 nm2 = make_float2(-kRoundMagic, -kRoundMagic);
        const float2 neg1 = make_float2(-1.0f, -1.0f);
        uint32_t code[16];
        bool ok = true;
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          const float4 rv = rn4[j4];
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            const int j = 4 * j4 + 2 * p;
            const float2 x2 = __fmul2_rn(
                make_float2(__uint_as_float(hb[j] << 16), __uint_as_float(hb[j + 1] << 16)), ci2);
            const float2 t = __fmul2_rn(x2, p ? make_float2(rv.z, rv.w) : make_float2(rv.x, rv.y));
            // clamp first: beyond +-QMAX the exact quotient (within |t| 2^-22 of t)
            // rounds to the same end, so only t inside the range is rounded; the clamp
            // keeps a NaN t (NaN h, a bad scale staged as a NaN reciprocal)
            const float2 tc = make_float2(clamp_nan(t.x, kq), clamp_nan(t.y, kq));
            const float2 u = __fadd2_rn(tc, m2);                         // magic + rint(tc)
            const float2 d = __ffma2_rn(__fadd2_rn(u, nm2), neg1, tc);   // tc - rint(tc)
            // exact unless tc lies near a half-integer; NaN fails the test too
            ok = ok && fabsf(d.x) < 0.5f - 0x1p-12f && fabsf(d.y) < 0.5f - 0x1p-12f;
            code[j] = __float_as_uint(u.x);
            code[j + 1] = __float_as_uint(u.y);
          }
        }
        if (!ok) {  // exact codes where the fast one may differ
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float xv = __fmul_rn(__uint_as_float(hb[j] << 16), g_ci);
            const float rn = g_s[C::BN + j0 + j];
            const float t = clamp_nan(__fmul_rn(xv, rn), kq);
            const float d = __fsub_rn(t, __fsub_rn(__fadd_rn(t, kRoundMagic), kRoundMagic));
            if (!(fabsf(d) < 0.5f - 0x1p-12f))
              code[j] = code_exact_next<C::QMAX_NEXT>(xv, g_s[j0 + j], rn);
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) sb[j * 32 + lane] = static_cast<uint8_t>(code[j]);
        store_buf(sb, j0);
      };

      // Everything one chunk of finished accumulators produces.
      auto finish = [&](const uint32_t (&r)[16], int j0) {
        if (args.acc_out != nullptr && n < args.N) {
          // int32 debug view: exact, the scaled sums are multiples of 2^ACC_SHIFT
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (m0 + j0 + j < args.M)
              args.acc_out[(size_t)(m0 + j0 + j) * args.N + n] =
                  static_cast<int32_t>(r[j]) >> C::ACC_SHIFT;
        }
        if (!has_out) return;
        if constexpr (C::EPI > 0) emit_codes(r, j0);
        else emit_y(r, j0);
      };

      // staging visible to every epilogue warp (and the warps kept within one tile)
      __syncwarp();
      if (lane == 0) mbar_arrive(&tokbar[it & 1]);
      bool w = mbar_wait(&tokbar[it & 1], (it >> 1) & 1);
      w = w && mbar_wait(&tfull[b], ph_b);
      if (!__all_sync(0xFFFFFFFFu, w)) break;  // uniform, and converged for tcgen05.ld
      tc_fence_after();
      if (h >= C::NUM_CHUNKS) {  // no chunk for this warp (token tiles of 16)
        tc_fence_before();
        if (lane == 0) {
          if constexpr (C::PAIR) mbar_arrive_cluster(mapa_shared(&tempty[b], 0));
          else mbar_arrive(&tempty[b]);
        }
      }
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(b * C::MMA_WARPS * C::BN);
      // issuers that accumulated into this tile (one per K block, up to MMA_WARPS)
      int nparts = 1;
      if constexpr (C::MMA_WARPS > 1) {
        int kb0, kb1;
        split_range(num_k, args.splits, unit % args.splits, kb0, kb1);
        nparts = kb1 - kb0 < C::MMA_WARPS ? kb1 - kb0 : C::MMA_WARPS;
      }
      // split K: the tile's int32 accumulator (2^ACC_SHIFT-scaled), summed by red.add
      int32_t* tile_acc =
          split ? args.partial + (size_t)tile * C::BN * C::BM + q * 32 + lane : nullptr;
      for (int c = h; c < C::NUM_CHUNKS; c += C::EPI_PER_Q) {
        const int j0 = c * C::EPI_CHUNK;
        uint32_t r[16];
        tmem_ld_32x32b_x16(tbase + j0, r);
#pragma unroll
        for (int p = 1; p < C::MMA_WARPS; ++p) {  // the other issuers' partial sums
          if (p < nparts) {
            uint32_t t[16];
            tmem_ld_32x32b_x16(tbase + p * C::BN + j0, t);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] += t[j];  // int32 sums: exact in any order
          }
        }
        tmem_wait_ld();
        if (c + C::EPI_PER_Q >= C::NUM_CHUNKS) {  // last chunk of this warp: hand the accumulator back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (C::PAIR) mbar_arrive_cluster(mapa_shared(&tempty[b], 0));
            else mbar_arrive(&tempty[b]);
          }
        }
        if (m0 + j0 >= args.M) continue;  // whole chunk beyond the last token
        if (!split) {
          finish(r, j0);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)  // exact in any order; no return value needed
            atomicAdd(tile_acc + (j0 + j) * C::BM, static_cast<int32_t>(r[j]));
        }
      }
      if (split && h < C::NUM_CHUNKS) {
        // The last of the tile's splits to finish this warp slice sums the
        // partials (int32: exact in any order) and finishes them.
        __threadfence();
        __syncwarp();
        int* counter = args.counters + tile * C::EPI_WARPS + e;
        int prev = 0;
        if (lane == 0) prev = atomicAdd(counter, 1);
        prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
        if (prev == args.splits - 1) {
          __threadfence();
          for (int c = h; c < C::NUM_CHUNKS; c += C::EPI_PER_Q) {
            const int j0 = c * C::EPI_CHUNK;
            if (m0 + j0 >= args.M) continue;
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              r[j] = static_cast<uint32_t>(__ldcg(tile_acc + (j0 + j) * C::BM));
            finish(r, j0);
          }
        }
      }
      if (++b == 2) { b = 0; ph_b ^= 1u; }
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // a pair: neither CTA leaves (or frees the TMEM) while the other may still
  // arrive on its barriers or have the pair MMA read its shared memory
  if constexpr (C::PAIR) cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (C::PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major 2-D tensor [rows][cols] of `esize`-byte elements.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int cols,
              int rows, int box_cols, int box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esize};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int bn_for(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256; }

// Token tile of a CTA pair on the plain epilogue.  224-token tiles (weights in TMEM)
// run a little faster per token than 256-token tiles, but every pair works through
// whole tiles, so the busiest pair does ceil(tiles / pairs) x BN token columns per
// 256 output channels: where 224 leaves it more of them (4288 tokens on 2048 channels:
// 160 tiles, three per pair, against 136 tiles, two per pair), 256 is taken.
int pair_bn(int M, int N) {
  const long long pairs = sm_count() / 2;
  const long long ch = (N + 255) / 256;
  const auto busiest = [&](long long bn) {
    const long long tiles = ch * ((M + bn - 1) / bn);
    return (tiles + pairs - 1) / pairs * bn;
  };
  return busiest(224) <= busiest(256) ? 224 : 256;
}

// Inputs of the single-kernel linear (Cfg QBITS > 0).
struct SingleArgs {
  const uint16_t* x;   // bf16 [M][K]
  const float* cinv;   // [K] or null
  const float* table;  // clip ratios [T][S], or the stream gains [T][S] with thr
  const float* thr;    // static clipping thresholds [T], or null
};

template <class C>
cudaError_t run_gemm(const void* qx, const uint8_t* qw, int M, int N, int K,
                     const EpilogueArgs& ep, void* out, const SplitScratch* scratch,
                     cudaStream_t st, bool w_prefetch, const SingleArgs* single,
                     const GemmExtras* ex) {
  CUtensorMap tm_w, tm_x, tm_out;
  // packed rows of BK / 2 bytes: 64 (64-byte swizzle) or 128 (128-byte swizzle)
  constexpr CUtensorMapSwizzle kPackedSwizzle =
      C::KS == 1 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = make_map(&tm_w, qw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, C::BK / 2, C::BM,
                     kPackedSwizzle);
  if (C::QBITS > 0)  // bf16 activations, boxes of 64 channels x BN tokens
    ok = ok && single && make_map(&tm_x, single->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, 64,
                                  C::BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  else if (C::ACT_BITS == 8)  // each CTA of a pair loads half of the token tile
    ok = ok && make_map(&tm_x, qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 128, C::BNX,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_map(&tm_x, qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, C::BK / 2, C::BNX,
                        kPackedSwizzle);
  int32_t* acc_out = ex ? ex->acc_out : nullptr;
  if (out == nullptr && acc_out == nullptr) return cudaErrorInvalidValue;
  if (C::EPI > 0)  // the next linear's int8 codes [M][N], boxes of 32 channels x 16 tokens
    ok = ok && out && make_map(&tm_out, out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, M, 32,
                               C::EPI_CHUNK, CU_TENSOR_MAP_SWIZZLE_NONE);
  else  // y; the int32 debug view alone maps its own buffer here, and never stores to it
    ok = ok && make_map(&tm_out, out ? out : static_cast<void*>(acc_out),
                        CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, 32, C::EPI_CHUNK,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;

  TileArgs a;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.tiles_m = (M + C::BN - 1) / C::BN;
  a.tiles_n = (N + C::TILE_N - 1) / C::TILE_N;
  a.num_tiles = a.tiles_m * a.tiles_n;
  // Keep the smaller operand resident in L2: sweep output channels fastest when
  // the packed weights fit comfortably, so each activation tile streams once.
  a.n_fastest = (static_cast<size_t>(N) * K / 2) <= (48u << 20) ? 1 : 0;
  a.splits = (scratch != nullptr && !C::PAIR) ? gemm_splits(M, N, K) : 1;
  a.num_units = a.num_tiles * a.splits;
  a.partial = scratch ? scratch->partial : nullptr;
  a.counters = scratch ? scratch->counters : nullptr;
  a.w_prefetch = w_prefetch ? 1 : 0;
  a.q_x = single ? single->x : nullptr;
  a.q_cinv = single ? single->cinv : nullptr;
  a.q_alpha = single ? single->table : nullptr;
  a.q_thr = single ? single->thr : nullptr;
  a.ep = ep;
  a.has_y = out != nullptr ? 1 : 0;
  a.acc_out = acc_out;
  a.g_thr = ex ? ex->next_thr : nullptr;
  a.g_gain = ex ? ex->next_gain : nullptr;
  a.g_cinv = ex ? ex->next_cinv : nullptr;
  a.g_s = ex ? ex->next_s : nullptr;
  a.g_h = ex ? ex->h : nullptr;
  if (C::EPI > 0 && (a.g_thr == nullptr || a.g_gain == nullptr || a.g_s == nullptr))
    return cudaErrorInvalidValue;

  static std::atomic<bool> attr_set[kAttrDevices] = {};  // per template instance and device
  const cudaError_t e = set_smem_once(gemm_kernel<C>, C::SMEM_BYTES, attr_set);
  if (e != cudaSuccess) return e;
  if constexpr (C::PAIR) {  // clusters of two CTAs, one unit per pair at a time
    static std::atomic<int> max_pairs[kAttrDevices] = {};  // resident pairs, per device
    int dev = 0;
    cudaGetDevice(&dev);
    int fit = (dev >= 0 && dev < kAttrDevices) ? max_pairs[dev].load() : 0;
    if (fit == 0) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * (sm_count() / 2));
      q.blockDim = dim3(C::THREADS);
      q.dynamicSmemBytes = C::SMEM_BYTES;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      q.attrs = at;
      q.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&fit, gemm_kernel<C>, &q) != cudaSuccess || fit < 1)
        fit = sm_count() / 2;
      if (dev >= 0 && dev < kAttrDevices) max_pairs[dev].store(fit);
    }
    const int pairs = a.num_units < fit ? a.num_units : fit;
    return launch_pdl(gemm_kernel<C>, 2 * pairs, C::THREADS, C::SMEM_BYTES, st, 2, tm_w, tm_x,
                      tm_out, a);
  }
  const int grid = a.num_units < sm_count() ? a.num_units : sm_count();
  return launch_pdl(gemm_kernel<C>, grid, C::THREADS, C::SMEM_BYTES, st, 1, tm_w, tm_x, tm_out, a);
}

// More than 128 tokens go to CTA pairs unless K is split (few tiles, long K): tiles
// of 224 tokens with the weights in TMEM (measured 4 % faster per step than 256-token
// pairs with the weights in shared memory on the hidden-4096 block) where pair_bn
// finds them no worse balanced, else 256; always 256 for the GELU-and-quantize
// epilogue, whose twelve warps keep the shared-memory design.  gemm_plan writes
// these choices out for reporting; a change here changes it too.
template <int ACT_BITS, int EPI = 0>
cudaError_t dispatch_bn(const void* qx, const uint8_t* qw, int M, int N, int K,
                        const EpilogueArgs& ep, void* out, const SplitScratch* sc,
                        cudaStream_t st, bool wp, const GemmExtras* ex) {
  if constexpr (ACT_BITS == 8) {
    if (bn_for(M) == 256 && (sc == nullptr || gemm_splits(M, N, K) == 1)) {
      if constexpr (EPI == 0) {
        if (pair_bn(M, N) == 224)
          return run_gemm<Cfg<224, 8, 0, 0, true>>(qx, qw, M, N, K, ep, out, nullptr, st, wp,
                                                   nullptr, ex);
        return run_gemm<Cfg<256, 8, 0, 0, true>>(qx, qw, M, N, K, ep, out, nullptr, st, wp,
                                                 nullptr, ex);
      } else {
        return run_gemm<Cfg<256, 8, 0, EPI, true>>(qx, qw, M, N, K, ep, out, nullptr, st, wp,
                                                   nullptr, ex);
      }
    }
  }
  // narrow token tiles stream 256-deep stages when K allows
  const bool ks2 = K % 256 == 0;
  switch (bn_for(M)) {
    case 16:
      return ks2 ? run_gemm<Cfg<16, ACT_BITS, 0, EPI, false, 2>>(qx, qw, M, N, K, ep, out, sc, st,
                                                                  wp, nullptr, ex)
                 : run_gemm<Cfg<16, ACT_BITS, 0, EPI>>(qx, qw, M, N, K, ep, out, sc, st, wp,
                                                       nullptr, ex);
    case 32:
      return ks2 ? run_gemm<Cfg<32, ACT_BITS, 0, EPI, false, 2>>(qx, qw, M, N, K, ep, out, sc, st,
                                                                  wp, nullptr, ex)
                 : run_gemm<Cfg<32, ACT_BITS, 0, EPI>>(qx, qw, M, N, K, ep, out, sc, st, wp,
                                                       nullptr, ex);
    case 64:
      return ks2 ? run_gemm<Cfg<64, ACT_BITS, 0, EPI, false, 2>>(qx, qw, M, N, K, ep, out, sc, st,
                                                                  wp, nullptr, ex)
                 : run_gemm<Cfg<64, ACT_BITS, 0, EPI>>(qx, qw, M, N, K, ep, out, sc, st, wp,
                                                       nullptr, ex);
    case 128:
      return run_gemm<Cfg<128, ACT_BITS, 0, EPI>>(qx, qw, M, N, K, ep, out, sc, st, wp, nullptr,
                                                   ex);
    default:
      return run_gemm<Cfg<256, ACT_BITS, 0, EPI>>(qx, qw, M, N, K, ep, out, sc, st, wp, nullptr,
                                                   ex);
  }
}

template <int QBITS>
cudaError_t dispatch_single(const SingleArgs& sa, const uint8_t* qw, int M, int N, int K,
                            const EpilogueArgs& ep, void* y, cudaStream_t st) {
  switch (bn_for(M)) {
    case 16: return run_gemm<Cfg<16, 8, QBITS>>(nullptr, qw, M, N, K, ep, y, nullptr, st, false,
                                                &sa, nullptr);
    case 32: return run_gemm<Cfg<32, 8, QBITS>>(nullptr, qw, M, N, K, ep, y, nullptr, st, false,
                                                &sa, nullptr);
    default: return run_gemm<Cfg<64, 8, QBITS>>(nullptr, qw, M, N, K, ep, y, nullptr, st, false,
                                                &sa, nullptr);
  }
}

}  // namespace

cudaError_t launch_linear_single(const uint16_t* x, const float* cinv, const float* table,
                                 const float* thr, int act_bits, const uint8_t* qw, int M, int N,
                                 int K, const EpilogueArgs& ep, void* y, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (M > kSingleKernelMaxM) return cudaErrorInvalidValue;
  const SingleArgs sa{x, cinv, table, thr};
  return act_bits == 8 ? dispatch_single<8>(sa, qw, M, N, K, ep, y, st)
                       : dispatch_single<4>(sa, qw, M, N, K, ep, y, st);
}

int gemm_splits(int M, int N, int K) {
  const int BN = bn_for(M);
  const int tiles = ((M + BN - 1) / BN) * ((N + 127) / 128);
  const int num_k = K / 128;
  if (tiles * 2 > kSplitTargetCtas) return 1;
  // Splitting pays only when each tile's K loop is long: measured at 16-256 tokens,
  // K = 2048 ran faster unsplit (the partial sums, their reduction and the lost CTA
  // pairs of 256-token tiles outweigh the extra SMs), K = 4096 about even (split
  // kept for the narrow tiles), K >= 8192 up to twice as fast split.
  if (num_k < 32 || (num_k < 64 && BN > 64)) return 1;
  int s = kSplitTargetCtas / tiles;
  const int cap = num_k / 2 > 1 ? num_k / 2 : 1;  // at least two K blocks per split
  s = s < cap ? s : cap;
  return s > 1 ? s : 1;
}

// Output tiles of the single-CTA instances (128 channels each), and the split
// scratch's two parts, each rounded up to 256 bytes.
size_t split_tiles(int M, int N) {
  const int BN = bn_for(M);
  return static_cast<size_t>((M + BN - 1) / BN) * ((N + 127) / 128);
}
size_t split_partial_bytes(int M, int N) {
  const size_t partial = split_tiles(M, N) * bn_for(M) * 128 * sizeof(int32_t);
  return (partial + 255) / 256 * 256;
}

size_t gemm_split_scratch_bytes(int M, int N, int K) {
  if (gemm_splits(M, N, K) == 1) return 0;
  const size_t counters = split_tiles(M, N) * kMaxEpiWarps * sizeof(int);
  return split_partial_bytes(M, N) + (counters + 255) / 256 * 256;
}

SplitScratch split_scratch_at(void* base, int M, int N) {
  uint8_t* p = static_cast<uint8_t*>(base);
  return SplitScratch{reinterpret_cast<int32_t*>(p),
                      reinterpret_cast<int*>(p + split_partial_bytes(M, N))};
}

// The choices of dispatch_bn and run_gemm, written out.
GemmPlan gemm_plan(int M, int N, int K, int act_bits, bool split_scratch, bool gelu_quant) {
  GemmPlan p{};
  if (M <= 0) return p;
  const int BN = bn_for(M);
  const int splits = split_scratch ? gemm_splits(M, N, K) : 1;
  if (act_bits == 8 && BN == 256 && splits == 1) {  // CTA pairs
    p.tile_tokens = gelu_quant ? 256 : pair_bn(M, N);
    p.tile_channels = 256;
    p.ctas_per_tile = 2;
    p.k_splits = 1;
    p.k_stage = 128;
    p.weights_in_tmem = p.tile_tokens == 224 ? 1 : 0;
  } else {
    p.tile_tokens = BN;
    p.tile_channels = 128;
    p.ctas_per_tile = 1;
    p.k_splits = splits;
    p.k_stage = BN <= 64 && K % 256 == 0 ? 256 : 128;
    p.weights_in_tmem = p.k_stage == 256 && !gelu_quant ? 1 : 0;
  }
  p.tiles = ((M + p.tile_tokens - 1) / p.tile_tokens) *
            ((N + p.tile_channels - 1) / p.tile_channels);
  return p;
}

cudaError_t launch_gemm(const void* qx, int act_bits, const uint8_t* qw, int M, int N, int K,
                        const EpilogueArgs& ep, void* y, const SplitScratch* scratch,
                        cudaStream_t st, bool w_prefetch, const GemmExtras* extras) {
  if (M == 0) return cudaSuccess;
  return act_bits == 8
             ? dispatch_bn<8>(qx, qw, M, N, K, ep, y, scratch, st, w_prefetch, extras)
             : dispatch_bn<4>(qx, qw, M, N, K, ep, y, scratch, st, w_prefetch, extras);
}

// The GELU table, once per device: launched on the caller's stream, and marked
// built only after a launch outside stream capture has completed (a launch inside a
// capture becomes part of the graph and rebuilds the table on every replay).
cudaError_t ensure_gelu_table(cudaStream_t st) {
  static std::atomic<bool> built[kAttrDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
  const bool cached = dev >= 0 && dev < kAttrDevices;
  if (cached && built[dev].load(std::memory_order_acquire)) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return cudaGetLastError();
  constexpr int n = 2 * kGeluTabExps * 128;
  gelu_table_kernel<<<(n + 127) / 128, 128, 0, st>>>();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || cs != cudaStreamCaptureStatusNone) return e;
  e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && cached) built[dev].store(true, std::memory_order_release);
  return e;
}

cudaError_t launch_gemm_gelu_quant(const void* qx, const uint8_t* qw, int M, int N, int K,
                                   const EpilogueArgs& ep, int next_bits, int8_t* codes,
                                   const SplitScratch* scratch, cudaStream_t st, bool w_prefetch,
                                   const GemmExtras& extras) {
  if (M == 0) return cudaSuccess;
  return next_bits == 8
             ? dispatch_bn<8, 8>(qx, qw, M, N, K, ep, codes, scratch, st, w_prefetch, &extras)
             : dispatch_bn<8, 4>(qx, qw, M, N, K, ep, codes, scratch, st, w_prefetch, &extras);
}

}  // namespace wq
