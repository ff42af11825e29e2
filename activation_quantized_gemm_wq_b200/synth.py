"""Seeded synthetic inputs for the fused low-bit linear.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no scaling, clipping, quantization or GEMM).  Both the CUDA
path and the CPU oracle consume exactly the arrays produced here.

Workloads (the paper's LIBERO/RoboLab/DROID activations are not available; these
stand in for them with the token-stream structure of a world-action-model
denoiser: video, proprio and action rows sharing one weight matrix):

  tiny        K=N=256, M=64 (48 video, 8 proprio, 8 action), W4A8, 1 step
  block2048   hidden 2048 block: QKV 2048->6144, attn-out 2048->2048,
              MLP-up 2048->8192, MLP-down 8192->2048; M=4096+64+128
  block4096   hidden 4096 block: 4096->12288, 4096->4096, 4096->16384,
              16384->4096; M=8192+64+256, per-(step, stream) activation stds
  small-M     the eight weight shapes above with M in {16..256} action-only or
              proprio+action rows

Distributions: x ~ N(0, std_stream^2) with stds video 1.0, proprio 3.0,
action 0.5 (block4096: std per (step, stream) ~ U[0.5, 3.0]); a seeded subset of
input channels (tiny: 4 of 256 x30; block2048: 1% x U[20, 50]; block4096: 1% x50)
is scaled in every stream, in both the runtime rows and the 256-row calibration
batch; W ~ N(0, 0.02^2); bias ~ N(0, 0.01^2); beta ~ N(0, 1e-3^2) per
(step, stream, n); clip ratio alpha per (step, stream) ~ U[0.85, 1.0]
(tiny: {1.0, 0.95, 0.9}).  bf16 tensors are returned as raw uint16 patterns.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import List, Optional, Sequence, Tuple

import numpy as np

VIDEO, PROPRIO, ACTION = 0, 1, 2
N_STREAMS = 3
CAL_ROWS = 256


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest-even); returns uint16 patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    K: int
    N: int


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    linears: Tuple[Linear, ...]
    rows: Tuple[Tuple[int, int], ...]        # ordered (stream id, row count) runs
    act_bits: int
    T: int
    stds: Optional[Tuple[float, float, float]]  # None: drawn per (step, stream)
    outlier_frac: float                        # fraction of K (tiny: exact count below)
    outlier_count: Optional[int]
    outlier_range: Tuple[float, float]
    alpha_fixed: Optional[Tuple[float, ...]] = None
    fresh_x_per_step: bool = True

    @property
    def M(self) -> int:
        return sum(n for _, n in self.rows)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


_H2048 = (Linear("qkv", 2048, 6144), Linear("attn_out", 2048, 2048),
          Linear("mlp_up", 2048, 8192), Linear("mlp_down", 8192, 2048))
_H4096 = (Linear("qkv", 4096, 12288), Linear("attn_out", 4096, 4096),
          Linear("mlp_up", 4096, 16384), Linear("mlp_down", 16384, 4096))

TINY = Workload("tiny_w4a8", (Linear("linear", 256, 256),),
                ((VIDEO, 48), (PROPRIO, 8), (ACTION, 8)), 8, 1, (1.0, 3.0, 0.5),
                0.0, 4, (30.0, 30.0), alpha_fixed=(1.0, 0.95, 0.9))
BLOCK2048_A8 = Workload("block2048_w4a8", _H2048,
                        ((VIDEO, 4096), (PROPRIO, 64), (ACTION, 128)), 8, 1,
                        (1.0, 3.0, 0.5), 0.01, None, (20.0, 50.0))
BLOCK2048_A4 = BLOCK2048_A8.with_(name="block2048_w4a4_t10", act_bits=4, T=10)
BLOCK4096_A8 = Workload("block4096_w4a8_t10", _H4096,
                        ((VIDEO, 8192), (PROPRIO, 64), (ACTION, 256)), 8, 10, None,
                        0.01, None, (50.0, 50.0))
BLOCK4096_A4 = BLOCK4096_A8.with_(name="block4096_w4a4_t10", act_bits=4)

WORKLOADS = {w.name: w for w in (TINY, BLOCK2048_A8, BLOCK2048_A4, BLOCK4096_A8, BLOCK4096_A4)}

SMALL_M = (16, 32, 64, 128, 256)


def small_m(parent: Workload, M: int, mix: str, act_bits: int) -> Workload:
    """Small-M weight-streaming batch: 'action' rows only, or M/4 proprio then 3M/4 action."""
    if mix == "action":
        rows = ((ACTION, M),)
    elif mix == "proprio_action":
        rows = ((PROPRIO, M // 4), (ACTION, M - M // 4))
    else:
        raise ValueError(mix)
    return parent.with_(name=f"{parent.name.split('_')[0]}_m{M}_{mix}_a{act_bits}", rows=rows,
                        act_bits=act_bits, T=10)


# the small-M batches by name (weights and tables of the parent block)
for _parent in (BLOCK2048_A8, BLOCK4096_A8):
    for _bits in (8, 4):
        for _M in SMALL_M:
            _w = small_m(_parent, _M, "action", _bits)
            WORKLOADS[_w.name] = _w


def custom(name: str, K: int, N: int, rows: Sequence[Tuple[int, int]], act_bits: int = 8,
           T: int = 1, stds=(1.0, 3.0, 0.5), outlier_frac: float = 0.01,
           outlier_range=(20.0, 50.0)) -> Workload:
    """A one-linear workload of arbitrary shape with the block2048 distributions."""
    return Workload(name, (Linear("linear", K, N),), tuple(rows), act_bits, T, stds,
                    outlier_frac, None, outlier_range)


def _rng(seed: int, wl: Workload, *key: int) -> np.random.Generator:
    tag = zlib.crc32(wl.name.split("_m")[0].encode())
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, *key])))


# tensor ids inside the seed key
_T_W, _T_CAL, _T_OUT, _T_BIAS, _T_ALPHA, _T_BETA, _T_X, _T_STD = range(8)


def stream_ids(wl: Workload) -> np.ndarray:
    return np.concatenate([np.full(n, s, np.uint8) for s, n in wl.rows])


def _cal_rows(wl: Workload) -> np.ndarray:
    """Stream ids of the 256-row calibration batch, in the runtime proportions."""
    M = wl.M
    want = [(s, n * CAL_ROWS / M) for s, n in wl.rows]
    base = [(s, int(np.floor(v))) for s, v in want]
    short = CAL_ROWS - sum(n for _, n in base)
    order = sorted(range(len(want)), key=lambda i: -(want[i][1] - base[i][1]))
    counts = [n for _, n in base]
    for i in order[:short]:
        counts[i] += 1
    return np.concatenate([np.full(c, s, np.uint8) for (s, _), c in zip(base, counts)])


def _stds(wl: Workload, seed: int) -> np.ndarray:
    """[T][3] activation std per (step, stream)."""
    if wl.stds is not None:
        return np.tile(np.asarray(wl.stds, np.float32), (wl.T, 1))
    return _rng(seed, wl, 0, 0, _T_STD).uniform(0.5, 3.0, size=(wl.T, N_STREAMS)).astype(np.float32)


def _outliers(wl: Workload, layer: int, K: int, seed: int) -> np.ndarray:
    """Per-input-channel multiplier (1 except on the seeded outlier channels)."""
    g = _rng(seed, wl, layer, 0, _T_OUT)
    n = wl.outlier_count if wl.outlier_count is not None else int(round(wl.outlier_frac * K))
    mult = np.ones(K, np.float32)
    if n:
        idx = g.choice(K, size=n, replace=False)
        lo, hi = wl.outlier_range
        mult[idx] = g.uniform(lo, hi, size=n) if hi > lo else lo
    return mult


def _draw_x(g: np.random.Generator, sids: np.ndarray, std_row: np.ndarray,
            mult: np.ndarray) -> np.ndarray:
    K = mult.shape[0]
    z = g.standard_normal(size=(sids.shape[0], K), dtype=np.float32)
    z *= std_row[sids][:, None]
    z *= mult[None, :]
    return f32_to_bf16_bits(z)


@dataclasses.dataclass
class LayerInputs:
    """Static inputs of one linear: bf16 W [N][K], calibration batch, bias, tables."""
    W: np.ndarray
    x_cal: np.ndarray
    bias: np.ndarray
    alpha: np.ndarray   # [T][S]
    beta: np.ndarray    # [T][S][N]


def layer_inputs(wl: Workload, layer: int, seed: int = 0) -> LayerInputs:
    lin = wl.linears[layer]
    K, N, T = lin.K, lin.N, wl.T
    W = f32_to_bf16_bits(_rng(seed, wl, layer, 0, _T_W).normal(0.0, 0.02, size=(N, K))
                         .astype(np.float32))
    mult = _outliers(wl, layer, K, seed)
    stds = _stds(wl, seed)
    cal_sid = _cal_rows(wl)
    g = _rng(seed, wl, layer, 0, _T_CAL)
    z = g.standard_normal(size=(CAL_ROWS, K), dtype=np.float32)
    cal_step = np.arange(CAL_ROWS) % T
    z *= stds[cal_step, cal_sid][:, None]
    z *= mult[None, :]
    x_cal = f32_to_bf16_bits(z)
    bias = _rng(seed, wl, layer, 0, _T_BIAS).normal(0.0, 0.01, size=N).astype(np.float32)
    if wl.alpha_fixed is not None:
        alpha = np.tile(np.asarray(wl.alpha_fixed, np.float32), (T, 1))
    else:
        alpha = _rng(seed, wl, layer, 0, _T_ALPHA).uniform(0.85, 1.0, size=(T, N_STREAMS)) \
            .astype(np.float32)
    beta = _rng(seed, wl, layer, 0, _T_BETA).normal(0.0, 1e-3, size=(T, N_STREAMS, N)) \
        .astype(np.float32)
    return LayerInputs(W, x_cal, bias, alpha, beta)


def activations(wl: Workload, layer: int, step: int = 0, seed: int = 0) -> np.ndarray:
    """Runtime bf16 activations x [M][K] for (layer, step); fresh draw per step."""
    lin = wl.linears[layer]
    sids = stream_ids(wl)
    stds = _stds(wl, seed)
    mult = _outliers(wl, layer, lin.K, seed)
    key_step = step if wl.fresh_x_per_step else 0
    g = _rng(seed, wl, layer, key_step, _T_X, wl.M)
    return _draw_x(g, sids, stds[step], mult)


def total_ops(wl: Workload) -> int:
    """Multiply-accumulate count x2 of one pass over every linear of the workload."""
    return sum(2 * wl.M * l.N * l.K for l in wl.linears)
