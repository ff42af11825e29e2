"""The FFN up-projection whose epilogue quantizes for the down-projection
(wq_linear_gelu_quant): App. D keeps GELU in BF16 between the quantized FFN
projections; here h = bf16(GELU(y)) is formed in the up-projection's epilogue and
quantized there with the down-projection's channel scale and static clip.

Parity (both sides decide each code from the same bf16 value):
  - y of the same inputs (wq_linear_w4a8 / w4a4) within the tolerance of the oracle;
  - the GPU's h within one bf16 step of the oracle's GELU of the GPU's own y (fp32
    erfcf against fp64 erfc may straddle a bf16 rounding boundary);
  - codes and s_next bit for bit against the oracle's static quantizer applied to
    the GPU's h;
  - the down-projection on those codes (wq_gemm_w4ax with int8 operands, and the
    int32 debug view) against the oracle's GEMM and epilogue.
"""
import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

from gpu_util import (dev, gpu_gemm_s32, gpu_gemm_w4ax, gpu_linear, host, unpack_codes,
                      within_tolerance)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wq.wq_device_status()
    yield
    assert wq.wq_device_status() == ("WQ_OK", 0)


def _f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _ordered(bits):
    """bf16 patterns -> integers in the order of their values (adjacent values differ by 1)."""
    b = np.asarray(bits, np.uint16).astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def _f32bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


@pytest.mark.parametrize("bits_up,bits_next", [(8, 8), (8, 4), (4, 8)])
@pytest.mark.parametrize("M,K,N,wide", [(300, 512, 384, False), (33, 1024, 256, True),
                                        (16, 4096, 1024, False), (4288, 2048, 8192, False)],
                         ids=["300x512x384", "33x1024x256_wide", "16x4096x1024_split",
                              "block2048_mlp_up"])
def test_gelu_quant_against_oracle(oracle, M, K, N, wide, bits_up, bits_next):
    g = np.random.default_rng(M + K + N + 10 * bits_up + bits_next)
    T, step = 3, 2
    rows_ = ((0, M - M // 4 - M // 8), (1, M // 8), (2, M // 4))
    wl = S.custom(f"gelu{M}x{K}x{N}", K, N, tuple(r for r in rows_ if r[1] > 0),
                  act_bits=bits_up, T=T)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0, step=step)
    sid = S.stream_ids(wl)
    # wide: biases from -14 to 6 put y on GELU's whole curve, tails included
    bias = g.uniform(-14.0, 6.0, N).astype(np.float32) if wide else L.bias
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    cinv_next = g.uniform(0.5, 2.0, N).astype(np.float32)
    gain_next = g.uniform(0.85, 1.0, (T, 3)).astype(np.float32)

    y = gpu_linear(x, cinv, sid, L.alpha, L.beta, step, bits_up, qw, s_w, bias)
    h_of_y = oracle.gelu_bf16(y)
    # one shared threshold per step: 0.8 of the largest |h * cinv_next| (some codes clip)
    peak = float(np.max(np.abs(_f32(h_of_y) * cinv_next)))
    thr_next = np.full(T, 0.8 * peak, np.float32)

    codes = torch.empty((M, N), dtype=torch.int8, device="cuda")
    s_next = torch.empty(M, dtype=torch.float32, device="cuda")
    h = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = wq.alloc_workspace(M, K, N, bits_up)
    wq.wq_linear_gelu_quant(dev(x), dev(cinv), dev(sid), dev(L.alpha), dev(L.beta), step,
                            bits_up, dev(qw), dev(s_w), dev(bias), dev(cinv_next), dev(thr_next),
                            dev(gain_next), bits_next, codes, s_next, h, ws)
    codes, s_next, h = host(codes), host(s_next), host(h.view(torch.int16), np.uint16)

    # y against the oracle (every row, or sampled rows at full size)
    sel = np.arange(M) if M <= 600 else np.sort(np.concatenate(
        [[0, 4095, 4096, 4159, 4160, M - 1], g.choice(M, 10, replace=False)]))
    y_ref = oracle.linear(x[sel], cinv, sid[sel], L.alpha, L.beta, step, bits_up, qw, s_w,
                          bias)[0]
    ok, worst = within_tolerance(y[sel], y_ref)
    assert ok, worst
    # h within one bf16 step of the oracle's GELU of the same y
    d = np.abs(_ordered(h) - _ordered(h_of_y))
    assert d.max() <= 1, f"h off by {d.max()} bf16 steps"
    assert np.mean(d == 0) > 0.99
    # codes and scales bit for bit from the GPU's h
    q_ref, s_ref = oracle.act_quant_static(h, cinv_next, sid, thr_next, gain_next, step,
                                           bits_next)
    assert np.array_equal(_f32bits(s_next), _f32bits(s_ref))
    assert np.array_equal(codes, q_ref if bits_next == 8 else unpack_codes(q_ref))
    qmax = 127 if bits_next == 8 else 7
    assert np.abs(codes.astype(np.int32)).max() == qmax  # the clip was reached

    # the down-projection on those codes (int8 operands for both widths)
    N2 = 256
    wl2 = S.custom(f"geludown{N}", N, N2, tuple(r for r in rows_ if r[1] > 0), T=T)
    L2 = S.layer_inputs(wl2, 0)
    qw2, s_w2 = oracle.pack_int4(L2.W, None)
    acc = gpu_gemm_s32(codes, 8, qw2, N)
    acc_ref = oracle.gemm_s32(codes, 8, qw2, N)
    assert np.array_equal(acc, acc_ref)
    y2 = gpu_gemm_w4ax(codes, s_next, 8, N, sid, L2.beta, step, qw2, s_w2, L2.bias)
    y2_ref = oracle.epilogue(acc_ref, s_next, s_w2, L2.bias, L2.beta, sid, step)
    ok, worst = within_tolerance(y2, y2_ref)
    assert ok, worst


def test_gelu_quant_without_h_matches_with_h(oracle):
    """The debug copy of h changes nothing: codes and scales are the same without it."""
    M, K, N, T = 200, 256, 512, 1
    wl = S.custom("gelu_noh", K, N, ((0, 150), (2, 50)), T=T)
    L = S.layer_inputs(wl, 0)
    x, sid = S.activations(wl, 0), S.stream_ids(wl)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    thr, gain = np.full(T, 0.05, np.float32), np.ones((T, 3), np.float32)
    outs = []
    for with_h in (True, False):
        codes = torch.empty((M, N), dtype=torch.int8, device="cuda")
        s_next = torch.empty(M, dtype=torch.float32, device="cuda")
        h = torch.empty((M, N), dtype=torch.bfloat16, device="cuda") if with_h else None
        wq.wq_linear_gelu_quant(dev(x), dev(cinv), dev(sid), dev(L.alpha), dev(L.beta), 0, 8,
                                dev(qw), dev(s_w), dev(L.bias), None, dev(thr), dev(gain), 8,
                                codes, s_next, h, wq.alloc_workspace(M, K, N, 8))
        outs.append((host(codes), host(s_next)))
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])
