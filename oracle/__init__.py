"""ctypes front end of the plain-C CPU oracle.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``activation_quantized_gemm_wq_b200``) never imports it and shares no code
with it.

All array arguments are numpy arrays; bf16 tensors travel as their raw uint16
bit patterns.  See ``oracle.h`` for the definitions and their citations.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int


def load(path=None):
    """Load (building first if needed) the oracle shared library."""
    global _LIB
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _LIB is None:
        if _build.needs_build():
            _build.build()
        _LIB = _bind(ctypes.CDLL(_build.LIB))
    return _LIB


def _bind(lib):
    lib.oracle_channel_scale.argtypes = [_P, _I, _P, _I, _I, _P, _P]
    lib.oracle_pack_int4.argtypes = [_P, _P, _I, _I, _P, _P]
    lib.oracle_act_quant.argtypes = [_P, _I, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P]
    lib.oracle_act_quant_static.argtypes = [_P, _I, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P,
                                            _P]
    lib.oracle_gemm_s32.argtypes = [_P, _I, _P, _I, _I, _I, _P]
    lib.oracle_epilogue.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]
    lib.oracle_linear.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P,
                                  _P, _P, _P, _P, _P]
    lib.oracle_gelu.argtypes = [ctypes.c_double]
    lib.oracle_gelu.restype = ctypes.c_double
    lib.oracle_gelu_bf16.argtypes = [_P, ctypes.c_size_t, _P]
    lib.oracle_gelu_bf16.restype = _I
    lib.oracle_bf16_to_float.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_float.restype = ctypes.c_float
    lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_double_to_bf16.restype = ctypes.c_uint16
    for f in ("oracle_channel_scale", "oracle_pack_int4", "oracle_act_quant",
              "oracle_act_quant_static", "oracle_gemm_s32", "oracle_epilogue", "oracle_linear"):
        getattr(lib, f).restype = _I
    return lib


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


class Oracle:
    """Typed wrappers over one loaded oracle library (the real one or a test build)."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def channel_scale(self, x_cal, W):
        x_cal = _c(x_cal, np.uint16)
        W = _c(W, np.uint16)
        K = W.shape[1]
        c = np.empty(K, np.float32)
        cinv = np.empty(K, np.float32)
        _check(self.lib.oracle_channel_scale(_ptr(x_cal), x_cal.shape[0], _ptr(W), W.shape[0],
                                             K, _ptr(c), _ptr(cinv)), "channel_scale")
        return c, cinv

    def pack_int4(self, W, c=None):
        W = _c(W, np.uint16)
        c = _c(c, np.float32)
        N, K = W.shape
        qw = np.empty((N, K // 2), np.uint8)
        s_w = np.empty(N, np.float32)
        _check(self.lib.oracle_pack_int4(_ptr(W), _ptr(c), N, K, _ptr(qw), _ptr(s_w)),
               "pack_int4")
        return qw, s_w

    def act_quant(self, x, cinv, stream_id, alpha, step, act_bits):
        x = _c(x, np.uint16)
        cinv = _c(cinv, np.float32)
        stream_id = _c(stream_id, np.uint8)
        alpha = _c(alpha, np.float32)
        T, S = alpha.shape
        M, K = x.shape
        qx = np.empty((M, K) if act_bits == 8 else (M, K // 2),
                      np.int8 if act_bits == 8 else np.uint8)
        s_tok = np.empty(M, np.float32)
        _check(self.lib.oracle_act_quant(_ptr(x), M, K, _ptr(cinv), _ptr(stream_id), _ptr(alpha),
                                         S, T, step, act_bits, _ptr(qx), _ptr(s_tok)),
               "act_quant")
        return qx, s_tok

    def act_quant_static(self, x, cinv, stream_id, thr, gain, step, act_bits):
        """Static clipping (shared threshold thr [T], stream gains gain [T][S])."""
        x = _c(x, np.uint16)
        cinv = _c(cinv, np.float32)
        stream_id = _c(stream_id, np.uint8)
        thr = _c(thr, np.float32)
        gain = _c(gain, np.float32)
        T, S = gain.shape
        M, K = x.shape
        qx = np.empty((M, K) if act_bits == 8 else (M, K // 2),
                      np.int8 if act_bits == 8 else np.uint8)
        s_tok = np.empty(M, np.float32)
        _check(self.lib.oracle_act_quant_static(_ptr(x), M, K, _ptr(cinv), _ptr(stream_id),
                                                _ptr(thr), _ptr(gain), S, T, step, act_bits,
                                                _ptr(qx), _ptr(s_tok)), "act_quant_static")
        return qx, s_tok

    def linear_static(self, x, cinv, stream_id, thr, gain, beta, step, act_bits, qw, s_w, bias):
        """The fused linear with static clipping, as the three steps in order:
        act_quant_static, gemm_s32, epilogue.  Returns (y bf16 bits, qx, s_tok, acc)."""
        qx, s_tok = self.act_quant_static(x, cinv, stream_id, thr, gain, step, act_bits)
        acc = self.gemm_s32(qx, act_bits, qw, np.asarray(x).shape[1])
        if beta is None:  # the epilogue's table shape comes from the gains
            y = self.epilogue(acc, s_tok, s_w, bias,
                              np.zeros((np.asarray(gain).shape[0], np.asarray(gain).shape[1],
                                        np.asarray(qw).shape[0]), np.float32),
                              stream_id, step)
        else:
            y = self.epilogue(acc, s_tok, s_w, bias, beta, stream_id, step)
        return y, qx, s_tok, acc

    def gemm_s32(self, qx, act_bits, qw, K):
        qx = np.ascontiguousarray(qx)
        qw = _c(qw, np.uint8)
        M = qx.shape[0]
        N = qw.shape[0]
        acc = np.empty((M, N), np.int32)
        _check(self.lib.oracle_gemm_s32(_ptr(qx), act_bits, _ptr(qw), M, N, K, _ptr(acc)),
               "gemm_s32")
        return acc

    def epilogue(self, acc, s_tok, s_w, bias, beta, stream_id, step):
        acc = _c(acc, np.int32)
        s_tok = _c(s_tok, np.float32)
        s_w = _c(s_w, np.float32)
        bias = _c(bias, np.float32)
        stream_id = _c(stream_id, np.uint8)
        M, N = acc.shape
        if beta is not None:
            beta = _c(beta, np.float32)
            T, S = beta.shape[0], beta.shape[1]
        else:
            T, S = step + 1, int(stream_id.max()) + 1 if M else 1
        y = np.empty((M, N), np.uint16)
        _check(self.lib.oracle_epilogue(_ptr(acc), _ptr(s_tok), _ptr(s_w), _ptr(bias),
                                        _ptr(beta), _ptr(stream_id), M, N, S, T, step,
                                        _ptr(y)), "epilogue")
        return y

    def linear(self, x, cinv, stream_id, alpha, beta, step, act_bits, qw, s_w, bias):
        """The whole fused linear; returns (y bf16 bits, qx, s_tok, acc)."""
        x = _c(x, np.uint16)
        cinv = _c(cinv, np.float32)
        stream_id = _c(stream_id, np.uint8)
        alpha = _c(alpha, np.float32)
        beta = _c(beta, np.float32)
        qw = _c(qw, np.uint8)
        s_w = _c(s_w, np.float32)
        bias = _c(bias, np.float32)
        M, K = x.shape
        N = qw.shape[0]
        T, S = alpha.shape
        y = np.empty((M, N), np.uint16)
        qx = np.empty((M, K) if act_bits == 8 else (M, K // 2),
                      np.int8 if act_bits == 8 else np.uint8)
        s_tok = np.empty(M, np.float32)
        acc = np.empty((M, N), np.int32)
        _check(self.lib.oracle_linear(_ptr(x), M, K, N, _ptr(cinv), _ptr(stream_id), _ptr(alpha),
                                      _ptr(beta), S, T, step, act_bits, _ptr(qw), _ptr(s_w),
                                      _ptr(bias), _ptr(y), _ptr(qx), _ptr(s_tok), _ptr(acc)),
               "linear")
        return y, qx, s_tok, acc


    def gelu(self, v):
        """GELU(v) in fp64 (App. D keeps GELU in BF16; exact erf form)."""
        return float(self.lib.oracle_gelu(float(v)))

    def gelu_bf16(self, v):
        """bf16(GELU(v)) elementwise for raw bf16 patterns v, one rounding."""
        v = _c(v, np.uint16)
        h = np.empty_like(v)
        _check(self.lib.oracle_gelu_bf16(_ptr(v), v.size, _ptr(h)), "gelu_bf16")
        return h

    def linear_gelu_quant_static(self, x, cinv, stream_id, alpha, beta, step, act_bits, qw,
                                 s_w, bias, cinv_next, thr_next, gain_next, act_bits_next):
        """An FFN up-projection whose output is quantized for the down-projection:
        y = the fused linear (bf16, App. D keeps the linear's output in BF16),
        h = bf16(GELU(y)), then h quantized as the next linear's activation with its
        channel scale cinv_next and static clipping (thr_next [T], gain_next [T][S]:
        one shared threshold per step, a gain per stream; no row maximum, so each
        code depends only on its own element).  Returns (codes, s_next, h, y)."""
        y = self.linear(x, cinv, stream_id, alpha, beta, step, act_bits, qw, s_w, bias)[0]
        h = self.gelu_bf16(y)
        codes, s_next = self.act_quant_static(h, cinv_next, stream_id, thr_next, gain_next,
                                              step, act_bits_next)
        return codes, s_next, h, y


def bf16_bits_to_f32(bits):
    """Widen raw bf16 patterns to float32 (exact)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)
