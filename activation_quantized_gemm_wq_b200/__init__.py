"""Python binding of libwq (include/wq.h): the fused W4A8 / W4A4 linear of
SteerQuant's Rudder kernels on B200 (sm_100a).

Argument marshalling only: every step runs in the CUDA library.  Tensors are
torch CUDA tensors (device memory and streams come from PyTorch); bf16 tensors
may be torch.bfloat16 or raw 16-bit integer tensors.  Each function has the
name and argument order of its C entry point, with sizes taken from the tensor
shapes.  There is no CPU fallback: if libwq.so is missing or fails to load,
importing the functions raises.
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

# name -> (restype, argtypes); mirrors include/wq.h
_SIGS = {
    "wq_status_string": (ctypes.c_char_p, [_I]),
    "wq_version": (_I, []),
    "wq_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "wq_channel_scale": (_I, [_P, _I, _P, _I, _I, _P, _P, _P]),
    "wq_pack_int4": (_I, [_P, _P, _I, _I, _P, _P, _P]),
    "wq_act_quant": (_I, [_P, _I, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "wq_gemm_w4ax": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P]),
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
    "wq_debug_gemm_s32": (_I, [_P, _I, _P, _I, _I, _I, _P, _P]),
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


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libwq takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libwq takes contiguous tensors")
    return t.data_ptr()


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
    _call("wq_channel_scale", _ptr(x_cal), Mcal, _ptr(W), W.shape[0], K, _ptr(c), _ptr(cinv),
          _stream(stream))


def wq_pack_int4(W, c, qw, s_w, stream=None):
    N, K = W.shape
    _call("wq_pack_int4", _ptr(W), _ptr(c), N, K, _ptr(qw), _ptr(s_w), _stream(stream))


def wq_act_quant(x, cinv, stream_id, alpha, step, act_bits, qx, s_tok, stream=None):
    M, K = x.shape
    T, S = alpha.shape
    _call("wq_act_quant", _ptr(x), M, K, _ptr(cinv), _ptr(stream_id), _ptr(alpha), S, T, step,
          act_bits, _ptr(qx), _ptr(s_tok), _stream(stream))


def wq_act_quant_static(x, cinv, stream_id, thr, gain, step, act_bits, qx, s_tok, stream=None):
    M, K = x.shape
    T, S = gain.shape
    _call("wq_act_quant_static", _ptr(x), M, K, _ptr(cinv), _ptr(stream_id), _ptr(thr),
          _ptr(gain), S, T, step, act_bits, _ptr(qx), _ptr(s_tok), _stream(stream))


def wq_linear_w4ax_static(x, cinv, stream_id, thr, gain, beta, step, act_bits, qw, s_w, bias, y,
                          workspace, stream=None):
    M, K = x.shape
    N = qw.shape[0]
    T, S = gain.shape
    _call("wq_linear_w4ax_static", _ptr(x), M, K, N, _ptr(cinv), _ptr(stream_id), _ptr(thr),
          _ptr(gain), _ptr(beta), S, T, step, act_bits, _ptr(qw), _ptr(s_w), _ptr(bias), _ptr(y),
          _ptr(workspace), _nbytes(workspace), _stream(stream))


def wq_linear_w4ax_single(x, cinv, stream_id, table, thr, beta, step, act_bits, qw, s_w, bias, y,
                          stream=None):
    """The fused linear as one kernel, for M <= 64 tokens (no workspace).  thr None:
    dynamic clipping, table = alpha; else static clipping, table = the stream gains."""
    M, K = x.shape
    N = qw.shape[0]
    T, S = table.shape
    _call("wq_linear_w4ax_single", _ptr(x), M, K, N, _ptr(cinv), _ptr(stream_id), _ptr(table),
          _ptr(thr), _ptr(beta), S, T, step, act_bits, _ptr(qw), _ptr(s_w), _ptr(bias), _ptr(y),
          _stream(stream))


def wq_gemm_w4ax(qx, s_tok, act_bits, K, stream_id, beta, S, T, step, qw, s_w, bias, y,
                 stream=None):
    M, N = y.shape
    _call("wq_gemm_w4ax", _ptr(qx), _ptr(s_tok), act_bits, M, K, N, _ptr(stream_id), _ptr(beta),
          S, T, step, _ptr(qw), _ptr(s_w), _ptr(bias), _ptr(y), _stream(stream))


def _linear(name, x, cinv, stream_id, alpha, beta, step, qw, s_w, bias, y, workspace, stream):
    M, K = x.shape
    N = qw.shape[0]
    T, S = alpha.shape
    _call(name, _ptr(x), M, K, N, _ptr(cinv), _ptr(stream_id), _ptr(alpha), _ptr(beta), S, T,
          step, _ptr(qw), _ptr(s_w), _ptr(bias), _ptr(y), _ptr(workspace), _nbytes(workspace),
          _stream(stream))


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
    M, K = x.shape
    N = qw.shape[0]
    T, S = alpha.shape
    _call("wq_linear_w4a8_noalloc", _ptr(x), M, K, N, _ptr(cinv), _ptr(stream_id), _ptr(alpha),
          _ptr(beta), S, T, step, _ptr(qw), _ptr(s_w), _ptr(bias), _ptr(y), _stream(stream))


def wq_debug_gemm_s32(qx, act_bits, qw, K, acc, stream=None):
    M, N = acc.shape
    _call("wq_debug_gemm_s32", _ptr(qx), act_bits, _ptr(qw), M, N, K, _ptr(acc), _stream(stream))


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
