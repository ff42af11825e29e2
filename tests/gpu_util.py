"""Helpers shared by the GPU tests: moving numpy arrays to and from the device,
running the library's entry points, and comparing with the oracle."""
import numpy as np
import torch

import activation_quantized_gemm_wq_b200 as wq


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def host(t, dtype=None):
    a = t.detach().cpu().numpy()
    if dtype is not None:
        a = a.view(dtype)
    return a


def bf16_to_f64(bits):
    return (np.asarray(bits).view(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def within_tolerance(y_bits, ref_bits):
    """max |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref), element-wise; returns
    (ok, worst ratio of error to allowance)."""
    y = bf16_to_f64(y_bits)
    ref = bf16_to_f64(ref_bits)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    allow = 2.0 ** -7 * np.abs(ref) + 1e-3 * rms
    err = np.abs(y - ref)
    worst = float(np.max(err / np.maximum(allow, 1e-300))) if ref.size else 0.0
    return bool(np.all(err <= allow)), worst


def gpu_prep(W, x_cal):
    """Channel scale and packed weights computed on the GPU."""
    N, K = W.shape
    c = torch.empty(K, dtype=torch.float32, device="cuda")
    cinv = torch.empty_like(c)
    qw = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    s_w = torch.empty(N, dtype=torch.float32, device="cuda")
    dW = dev(W)
    wq.wq_channel_scale(dev(x_cal), dW, c, cinv)
    wq.wq_pack_int4(dW, c, qw, s_w)
    return c, cinv, qw, s_w


def gpu_act_quant(x, cinv, sid, alpha, step, bits):
    M, K = x.shape
    qx = torch.empty((M, K) if bits == 8 else (M, K // 2),
                     dtype=torch.int8 if bits == 8 else torch.uint8, device="cuda")
    s_tok = torch.empty(M, dtype=torch.float32, device="cuda")
    wq.wq_act_quant(dev(x), None if cinv is None else dev(cinv), dev(sid), dev(alpha), step, bits,
                    qx, s_tok)
    return host(qx), host(s_tok)


def gpu_linear(x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias):
    """The fused linear through the C ABI; qw/s_w/cinv may be numpy or device tensors."""
    M, K = x.shape
    N = qw.shape[0]
    t = lambda a: None if a is None else (a if isinstance(a, torch.Tensor) else dev(a))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = wq.alloc_workspace(M, K, N, bits)
    fn = wq.wq_linear_w4a8 if bits == 8 else wq.wq_linear_w4a4
    fn(t(x), t(cinv), t(sid), t(alpha), t(beta), step, t(qw), t(s_w), t(bias), y, ws)
    return host(y.view(torch.int16), np.uint16)


def gpu_gemm_s32(qx, bits, qw, K):
    """The product GEMM's int32 accumulators on codes qx (K split as the fused linear
    splits it for these sizes, through a workspace)."""
    M, N = qx.shape[0], qw.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    ws = wq.alloc_workspace(M, K, N, bits)
    wq.wq_debug_gemm_s32(dev(qx), bits, dev(qw), K, acc, ws)
    return host(acc)


def unpack_codes(packed):
    """Packed int4 codes [M][K/2] (low nibble = even k, two's complement) -> int8 [M][K]."""
    p = np.asarray(packed, np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo -= (lo >= 8) * 16
    hi -= (hi >= 8) * 16
    out = np.empty((p.shape[0], p.shape[1] * 2), np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def _round256(n):
    return (n + 255) // 256 * 256


def gpu_linear_debug(x, cinv, sid, alpha, beta, step, bits, qw, s_w, bias, rows=None):
    """wq_debug_linear_s32 (the fused linear with its accumulators also written).
    Returns host copies of (y bf16 bits, acc int32, workspace codes int8 [.][K],
    workspace token scales), restricted to `rows` when given."""
    M, K = x.shape
    N = qw.shape[0]
    t = lambda a: None if a is None else (a if isinstance(a, torch.Tensor) else dev(a))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    ws = wq.alloc_workspace(M, K, N, bits)
    wq.wq_debug_linear_s32(t(x), t(cinv), t(sid), t(alpha), t(beta), step, bits, t(qw), t(s_w),
                           t(bias), y, acc, ws)
    codes = ws[: M * K].view(torch.int8).view(M, K)
    off = _round256(M * K)
    s_tok = ws[off: off + 4 * M].view(torch.float32)
    if rows is not None:
        idx = torch.as_tensor(np.asarray(rows), device="cuda", dtype=torch.long)
        y, acc, codes, s_tok = y[idx], acc[idx], codes[idx], s_tok[idx]
    return host(y.view(torch.int16), np.uint16), host(acc), host(codes), host(s_tok)


def gpu_gemm_w4ax(qx, s_tok, bits, K, sid, beta, step, qw, s_w, bias):
    """wq_gemm_w4ax on codes qx (int8 [M][K] or packed int4 [M][K/2])."""
    M, N = qx.shape[0], qw.shape[0]
    T, S_, _ = beta.shape
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    wq.wq_gemm_w4ax(dev(qx), dev(s_tok), bits, K, dev(sid), dev(beta), S_, T, step, dev(qw),
                    dev(s_w), None if bias is None else dev(bias), y)
    return host(y.view(torch.int16), np.uint16)


def gpu_gemm_w4ax_ws(qx, s_tok, bits, K, sid, beta, step, qw, s_w, bias):
    """wq_gemm_w4ax_ws: the GEMM-only call splitting K through a workspace.  The
    workspace is filled with garbage first: the call must clear what it uses."""
    M, N = qx.shape[0], qw.shape[0]
    T, S_, _ = beta.shape
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    n = wq.wq_gemm_scratch_bytes(M, K, N)
    ws = torch.full((max(n, 256),), 0xA5, dtype=torch.uint8, device="cuda") if n else None
    wq.wq_gemm_w4ax_ws(dev(qx), dev(s_tok), bits, K, dev(sid), dev(beta), S_, T, step, dev(qw),
                       dev(s_w), None if bias is None else dev(bias), y, ws)
    return host(y.view(torch.int16), np.uint16), n


def gpu_act_quant_static(x, cinv, sid, thr, gain, step, bits):
    M, K = x.shape
    qx = torch.empty((M, K) if bits == 8 else (M, K // 2),
                     dtype=torch.int8 if bits == 8 else torch.uint8, device="cuda")
    s_tok = torch.empty(M, dtype=torch.float32, device="cuda")
    wq.wq_act_quant_static(dev(x), None if cinv is None else dev(cinv), dev(sid), dev(thr),
                           dev(gain), step, bits, qx, s_tok)
    return host(qx), host(s_tok)


def gpu_linear_static(x, cinv, sid, thr, gain, beta, step, bits, qw, s_w, bias):
    M, K = x.shape
    N = qw.shape[0]
    t = lambda a: None if a is None else (a if isinstance(a, torch.Tensor) else dev(a))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = wq.alloc_workspace(M, K, N, bits)
    wq.wq_linear_w4ax_static(t(x), t(cinv), t(sid), t(thr), t(gain), t(beta), step, bits, t(qw),
                             t(s_w), t(bias), y, ws)
    return host(y.view(torch.int16), np.uint16)


def gpu_linear_single(x, cinv, sid, table, beta, step, bits, qw, s_w, bias, thr=None):
    M, K = x.shape
    N = qw.shape[0]
    t = lambda a: None if a is None else (a if isinstance(a, torch.Tensor) else dev(a))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    wq.wq_linear_w4ax_single(t(x), t(cinv), t(sid), t(table), t(thr), t(beta), step, bits, t(qw),
                             t(s_w), t(bias), y)
    return host(y.view(torch.int16), np.uint16)
