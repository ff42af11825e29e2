"""Python binding of libwq (include/wq.h): the fused W4A8 / W4A4 linear of
SteerQuant's Rudder kernels on B200 (sm_100a).

Argument marshalling only: every step runs in the CUDA library.  Tensors are
torch CUDA tensors (device memory and streams come from PyTorch); bf16 tensors
may be torch.bfloat16 or raw 16-bit integer tensors.  Each function has the
name and argument order of its C entry point, with sizes taken from the tensor
shapes.  The C entry points take plain pointers and cannot see how large a
buffer is, so before each call the binding checks every tensor against what the
call will read or write there: on the current CUDA device, contiguous, of the
element type the header names, and holding at least that many elements.  A
tensor that fails raises here (TypeError for the type, ValueError otherwise)
instead of reaching a kernel that would run past its end.  There is no CPU
fallback: if libwq.so is missing or fails to load, calling the functions raises.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwq.so")

_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int

WQ_OK = 0
STATUS = {0: "WQ_OK", 1: "WQ_ERR_NULL", 2: "WQ_ERR_SHAPE", 3: "WQ_ERR_ALIGN", 4: "WQ_ERR_ARG",
          5: "WQ_ERR_CUDA", 6: "WQ_ERR_TIMEOUT", 7: "WQ_ERR_DEVICE", 8: "WQ_ERR_SCRATCH"}



class GemmPlan(ctypes.Structure):
    """struct wq_gemm_plan of include/wq.h."""
    _fields_ = [(n, ctypes.c_int) for n in ("tile_tokens", "tile_channels", "ctas_per_tile",
                                             "k_splits", "k_stage", "tiles", "weights_in_tmem")]


PLAN_CALLS = {"gemm": 0, "gemm_ws": 1, "linear": 2, "gelu_quant": 3}

# name -> (restype, argtypes); mirrors include/wq.h
_SIGS = {
    "wq_status_string": (ctypes.c_char_p, [_I]),
    "wq_version": (_I, []),
    "wq_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "wq_channel_scale": (_I, [_P, _I, _P, _I, _I, _P, _P, _P]),
    "wq_pack_int4": (_I, [_P, _P, _I, _I, _P, _P, _P]),
    "wq_act_quant": (_I, [_P, _I, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "wq_gemm_w4ax": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "wq_gemm_scratch_bytes": (ctypes.c_size_t, [_I, _I, _I]),
    "wq_gemm_plan_query": (_I, [_I, _I, _I, _I, _I, ctypes.POINTER(GemmPlan)]),
    "wq_gemm_w4ax_ws": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P,
                             ctypes.c_size_t, _P]),
    "wq_linear_w4a8": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P,
                            ctypes.c_size_t, _P]),
    "wq_linear_w4a4": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P,
                            ctypes.c_size_t, _P]),
    "wq_linear_w4a8_noalloc": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P,
                                    _P]),
    "wq_act_quant_static": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "wq_linear_w4ax_static": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P,
                                   _P, _P, _P, ctypes.c_size_t, _P]),
    "wq_linear_w4ax_single": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P,
                                   _P, _P, _P]),
    "wq_debug_gemm_s32": (_I, [_P, _I, _P, _I, _I, _I, _P, _P, ctypes.c_size_t, _P]),
    "wq_debug_linear_s32": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P,
                                 _P, _P, _P, ctypes.c_size_t, _P]),
    "wq_linear_gelu_quant": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P,
                                  _P, _P, _P, _I, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "wq_debug_inject_stall": (_I, [_I, ctypes.c_uint]),
    "wq_device_status": (_I, [ctypes.POINTER(ctypes.c_uint)]),
}


class WQError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


def lib():
    """The loaded libwq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m activation_quantized_gemm_wq_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


# element types the header names for each kind of tensor
_BF16 = frozenset({"torch.bfloat16", "torch.int16", "torch.uint16"})
_F32 = frozenset({"torch.float32"})
_BYTES = frozenset({"torch.uint8", "torch.int8"})
_I32 = frozenset({"torch.int32"})


def _current_device():
    import torch
    return torch.cuda.current_device()


def _ptr(t, name, kinds=None, count=0):
    """Device address of tensor `t`, which the C call reads or writes as `count`
    elements of one of the element types `kinds` (None: any type, e.g. the
    workspace).  None passes through: the library decides which pointers may be
    NULL and returns WQ_ERR_NULL for the others."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name}: libwq takes device tensors")
    if not t.is_contiguous():
        raise ValueError(f"{name}: libwq takes contiguous tensors")
    if kinds is not None and str(t.dtype) not in kinds:
        raise TypeError(f"{name}: element type {t.dtype}, expected one of {sorted(kinds)}")
    if t.numel() < count:
        raise ValueError(f"{name}: {t.numel()} elements, the call uses {count}")
    if t.get_device() != _current_device():
        raise ValueError(f"{name}: on cuda:{t.get_device()}, the current device is "
                         f"cuda:{_current_device()}")
    return t.data_ptr()


def _codes_per_row(K, act_bits):
    """Bytes per token row of activation codes: K int8 codes, or K/2 packed int4."""
    return K // 2 if act_bits == 4 else K


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    if st != WQ_OK:
        raise WQError(name, st)


def _nbytes(t):
    return t.numel() * t.element_size()


def wq_version():
    return lib().wq_version()


def wq_workspace_bytes(M, K, N, act_bits):
    return int(lib().wq_workspace_bytes(M, K, N, act_bits))


def wq_channel_scale(x_cal, W, c, cinv, stream=None):
    Mcal, K = x_cal.shape
    N = W.shape[0]
    _call("wq_channel_scale", _ptr(x_cal, "x_cal", _BF16, Mcal * K), Mcal,
          _ptr(W, "W", _BF16, N * K), N, K, _ptr(c, "c", _F32, K), _ptr(cinv, "cinv", _F32, K),
          _stream(stream))


def wq_pack_int4(W, c, qw, s_w, stream=None):
    N, K = W.shape
    _call("wq_pack_int4", _ptr(W, "W", _BF16, N * K), _ptr(c, "c", _F32, K), N, K,
          _ptr(qw, "qw", _BYTES, N * (K // 2)), _ptr(s_w, "s_w", _F32, N), _stream(stream))


def wq_act_quant(x, cinv, stream_id, alpha, step, act_bits, qx, s_tok, stream=None):
    M, K = x.shape
    T, S = alpha.shape
    _call("wq_act_quant", _ptr(x, "x", _BF16, M * K), M, K, _ptr(cinv, "cinv", _F32, K),
          _ptr(stream_id, "stream_id", _BYTES, M), _ptr(alpha, "alpha", _F32, T * S), S, T, step,
          act_bits, _ptr(qx, "qx", _BYTES, M * _codes_per_row(K, act_bits)),
          _ptr(s_tok, "s_tok", _F32, M), _stream(stream))


def wq_act_quant_static(x, cinv, stream_id, thr, gain, step, act_bits, qx, s_tok, stream=None):
    M, K = x.shape
    T, S = gain.shape
    _call("wq_act_quant_static", _ptr(x, "x", _BF16, M * K), M, K, _ptr(cinv, "cinv", _F32, K),
          _ptr(stream_id, "stream_id", _BYTES, M), _ptr(thr, "thr", _F32, T),
          _ptr(gain, "gain", _F32, T * S), S, T, step, act_bits,
          _ptr(qx, "qx", _BYTES, M * _codes_per_row(K, act_bits)),
          _ptr(s_tok, "s_tok", _F32, M), _stream(stream))


def _token_and_weight_args(x, cinv, stream_id, beta, S, T, qw, s_w, bias, y):
    """The pointers every fused linear takes, checked for x [M][K], qw [N][K/2]."""
    M, K = x.shape
    N = qw.shape[0]
    return dict(M=M, K=K, N=N,
                x=_ptr(x, "x", _BF16, M * K), cinv=_ptr(cinv, "cinv", _F32, K),
                sid=_ptr(stream_id, "stream_id", _BYTES, M),
                beta=_ptr(beta, "beta", _F32, T * S * N), qw=_ptr(qw, "qw", _BYTES, N * (K // 2)),
                s_w=_ptr(s_w, "s_w", _F32, N), bias=_ptr(bias, "bias", _F32, N),
                y=_ptr(y, "y", _BF16, M * N))


def wq_linear_w4ax_static(x, cinv, stream_id, thr, gain, beta, step, act_bits, qw, s_w, bias, y,
                          workspace, stream=None):
    T, S = gain.shape
    a = _token_and_weight_args(x, cinv, stream_id, beta, S, T, qw, s_w, bias, y)
    _call("wq_linear_w4ax_static", a["x"], a["M"], a["K"], a["N"], a["cinv"], a["sid"],
          _ptr(thr, "thr", _F32, T), _ptr(gain, "gain", _F32, T * S), a["beta"], S, T, step,
          act_bits, a["qw"], a["s_w"], a["bias"], a["y"], _ptr(workspace, "workspace"),
          _nbytes(workspace), _stream(stream))


def wq_linear_w4ax_single(x, cinv, stream_id, table, thr, beta, step, act_bits, qw, s_w, bias, y,
                          stream=None):
    """The fused linear as one kernel, for M <= 64 tokens (no workspace).  thr None:
    dynamic clipping, table = alpha; else static clipping, table = the stream gains."""
    T, S = table.shape
    a = _token_and_weight_args(x, cinv, stream_id, beta, S, T, qw, s_w, bias, y)
    _call("wq_linear_w4ax_single", a["x"], a["M"], a["K"], a["N"], a["cinv"], a["sid"],
          _ptr(table, "table", _F32, T * S), _ptr(thr, "thr", _F32, T), a["beta"], S, T, step,
          act_bits, a["qw"], a["s_w"], a["bias"], a["y"], _stream(stream))


def wq_gemm_w4ax(qx, s_tok, act_bits, K, stream_id, beta, S, T, step, qw, s_w, bias, y,
                 stream=None):
    M, N = y.shape
    _call("wq_gemm_w4ax", _ptr(qx, "qx", _BYTES, M * _codes_per_row(K, act_bits)),
          _ptr(s_tok, "s_tok", _F32, M), act_bits, M, K, N,
          _ptr(stream_id, "stream_id", _BYTES, M), _ptr(beta, "beta", _F32, T * S * N), S, T,
          step, _ptr(qw, "qw", _BYTES, N * (K // 2)), _ptr(s_w, "s_w", _F32, N),
          _ptr(bias, "bias", _F32, N), _ptr(y, "y", _BF16, M * N), _stream(stream))


def wq_gemm_scratch_bytes(M, K, N):
    return int(lib().wq_gemm_scratch_bytes(M, K, N))


def wq_gemm_plan_query(M, K, N, act_bits=8, call="linear"):
    """Which GEMM instance `call` ("gemm", "gemm_ws", "linear" or "gelu_quant") runs
    for an (M, K, N) shape, as a dict of the wq_gemm_plan fields (no device work)."""
    plan = GemmPlan()
    _call("wq_gemm_plan_query", M, K, N, act_bits, PLAN_CALLS[call], ctypes.byref(plan))
    return {n: getattr(plan, n) for n, _ in GemmPlan._fields_}


def wq_gemm_w4ax_ws(qx, s_tok, act_bits, K, stream_id, beta, S, T, step, qw, s_w, bias, y,
                    workspace=None, stream=None):
    """wq_gemm_w4ax splitting K over every SM for few tokens, through `workspace`
    (at least wq_gemm_scratch_bytes(M, K, N) bytes; None when that is 0)."""
    M, N = y.shape
    _call("wq_gemm_w4ax_ws", _ptr(qx, "qx", _BYTES, M * _codes_per_row(K, act_bits)),
          _ptr(s_tok, "s_tok", _F32, M), act_bits, M, K, N,
          _ptr(stream_id, "stream_id", _BYTES, M), _ptr(beta, "beta", _F32, T * S * N), S, T,
          step, _ptr(qw, "qw", _BYTES, N * (K // 2)), _ptr(s_w, "s_w", _F32, N),
          _ptr(bias, "bias", _F32, N), _ptr(y, "y", _BF16, M * N),
          _ptr(workspace, "workspace"), 0 if workspace is None else _nbytes(workspace),
          _stream(stream))


def _linear(name, x, cinv, stream_id, alpha, beta, step, qw, s_w, bias, y, workspace, stream):
    T, S = alpha.shape
    a = _token_and_weight_args(x, cinv, stream_id, beta, S, T, qw, s_w, bias, y)
    _call(name, a["x"], a["M"], a["K"], a["N"], a["cinv"], a["sid"],
          _ptr(alpha, "alpha", _F32, T * S), a["beta"], S, T, step, a["qw"], a["s_w"], a["bias"],
          a["y"], _ptr(workspace, "workspace"), _nbytes(workspace), _stream(stream))


def wq_linear_w4a8(x, cinv, stream_id, alpha, beta, step, qw, s_w, bias, y, workspace,
                   stream=None):
    _linear("wq_linear_w4a8", x, cinv, stream_id, alpha, beta, step, qw, s_w, bias, y,
            workspace, stream)


def wq_linear_w4a4(x, cinv, stream_id, alpha, beta, step, qw, s_w, bias, y, workspace,
                   stream=None):
    _linear("wq_linear_w4a4", x, cinv, stream_id, alpha, beta, step, qw, s_w, bias, y,
            workspace, stream)


def wq_linear_w4a8_noalloc(x, cinv, stream_id, alpha, beta, step, qw, s_w, bias, y,
                           stream=None):
    """wq_linear_w4a8 without a workspace: for callers that cannot allocate device
    memory while they run.  Uses the library's fixed 16 MiB scratch (see wq.h)."""
    T, S = alpha.shape
    a = _token_and_weight_args(x, cinv, stream_id, beta, S, T, qw, s_w, bias, y)
    _call("wq_linear_w4a8_noalloc", a["x"], a["M"], a["K"], a["N"], a["cinv"], a["sid"],
          _ptr(alpha, "alpha", _F32, T * S), a["beta"], S, T, step, a["qw"], a["s_w"],
          a["bias"], a["y"], _stream(stream))


def wq_debug_gemm_s32(qx, act_bits, qw, K, acc, workspace=None, stream=None):
    """The product GEMM's int32 accumulators on codes qx.  workspace: as for the
    fused linear (wq_workspace_bytes); only needed when K is split (few tokens)."""
    M, N = acc.shape
    _call("wq_debug_gemm_s32", _ptr(qx, "qx", _BYTES, M * _codes_per_row(K, act_bits)),
          act_bits, _ptr(qw, "qw", _BYTES, N * (K // 2)), M, N, K, _ptr(acc, "acc", _I32, M * N),
          _ptr(workspace, "workspace"), 0 if workspace is None else _nbytes(workspace),
          _stream(stream))


def wq_debug_linear_s32(x, cinv, stream_id, alpha, beta, step, act_bits, qw, s_w, bias, y, acc,
                        workspace, stream=None):
    """wq_linear_w4a8 / w4a4 (by act_bits) with the int32 accumulators also written."""
    T, S = alpha.shape
    a = _token_and_weight_args(x, cinv, stream_id, beta, S, T, qw, s_w, bias, y)
    _call("wq_debug_linear_s32", a["x"], a["M"], a["K"], a["N"], a["cinv"], a["sid"],
          _ptr(alpha, "alpha", _F32, T * S), a["beta"], S, T, step, act_bits, a["qw"], a["s_w"],
          a["bias"], a["y"], _ptr(acc, "acc", _I32, a["M"] * a["N"]),
          _ptr(workspace, "workspace"), _nbytes(workspace), _stream(stream))


def wq_linear_gelu_quant(x, cinv, stream_id, alpha, beta, step, act_bits, qw, s_w, bias,
                         cinv_next, thr_next, gain_next, act_bits_next, codes_next, s_next, h,
                         workspace, stream=None):
    """FFN up-projection whose epilogue writes the down-projection's codes:
    codes_next int8 [M][N] and s_next [M] (static clipping thr_next [T], gain_next
    [T][S]); h [M][N] bf16 (debug copy of bf16(GELU(y))) may be None."""
    T, S = alpha.shape
    M, K = x.shape
    N = qw.shape[0]
    _call("wq_linear_gelu_quant", _ptr(x, "x", _BF16, M * K), M, K, N,
          _ptr(cinv, "cinv", _F32, K), _ptr(stream_id, "stream_id", _BYTES, M),
          _ptr(alpha, "alpha", _F32, T * S), _ptr(beta, "beta", _F32, T * S * N), S, T, step,
          act_bits, _ptr(qw, "qw", _BYTES, N * (K // 2)), _ptr(s_w, "s_w", _F32, N),
          _ptr(bias, "bias", _F32, N), _ptr(cinv_next, "cinv_next", _F32, N),
          _ptr(thr_next, "thr_next", _F32, T), _ptr(gain_next, "gain_next", _F32, T * S),
          act_bits_next, _ptr(codes_next, "codes_next", _BYTES, M * N),
          _ptr(s_next, "s_next", _F32, M), _ptr(h, "h", _BF16, M * N),
          _ptr(workspace, "workspace"), _nbytes(workspace), _stream(stream))


def wq_debug_inject_stall(enable, limit_us=0):
    """Test hook: make every later GEMM launch stall on its first stage and give up
    after limit_us (enable=True), or restore the defaults (enable=False)."""
    _call("wq_debug_inject_stall", 1 if enable else 0, int(limit_us))


def wq_device_status():
    """(status name, flag bits) of the device error word; clears it."""
    flags = ctypes.c_uint(0)
    st = lib().wq_device_status(ctypes.byref(flags))
    return STATUS.get(st, st), flags.value


def alloc_workspace(M, K, N, act_bits, device="cuda"):
    """A device workspace of wq_workspace_bytes() bytes (256-byte aligned by torch)."""
    import torch
    n = wq_workspace_bytes(M, K, N, act_bits)
    if n == 0:
        raise ValueError("invalid sizes for a workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)
