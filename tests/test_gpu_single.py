"""The single-kernel linear (quantization inside the GEMM, token counts up to one
64-token tile) against the oracle and against the two-kernel linear."""
import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

from gpu_util import gpu_linear, gpu_linear_single, gpu_linear_static, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wq.wq_device_status()
    yield
    assert wq.wq_device_status() == ("WQ_OK", 0)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (16, 2048, 1024), (37, 1024, 384),
                                   (64, 4096, 512), (5, 128, 48)])
def test_single_kernel_linear(oracle, M, K, N, bits):
    rows = ((1, M // 4), (2, M - M // 4))
    wl = S.custom(f"one{M}x{K}x{N}", K, N, tuple(r for r in rows if r[1] > 0), act_bits=bits,
                  T=3)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0, step=2)
    if M > 3:
        x[1] = 0  # a zero row
    sid = S.stream_ids(wl)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    for ci, bias, beta, step in ((cinv, L.bias, L.beta, 2), (None, None, None, 0)):
        y_ref, _, _, _ = oracle.linear(x, ci, sid, L.alpha, beta, step, bits, qw, s_w, bias)
        y = gpu_linear_single(x, ci, sid, L.alpha, beta, step, bits, qw, s_w, bias)
        ok, worst = within_tolerance(y, y_ref)
        assert ok, worst
        # the same codes and scales as the two-kernel path, so the same bf16 outputs
        y2 = gpu_linear(x, ci, sid, L.alpha, beta, step, bits, qw, s_w, bias)
        assert np.array_equal(y, y2)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,K,N", [(16, 2048, 1024), (37, 1024, 384), (1, 256, 16)])
def test_single_kernel_linear_static_clipping(oracle, M, K, N, bits):
    g = np.random.default_rng(M + 3 * K)
    rows = ((1, M // 4), (2, M - M // 4))
    wl = S.custom(f"ones{M}x{K}x{N}", K, N, tuple(r for r in rows if r[1] > 0), act_bits=bits,
                  T=3)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0, step=1)
    sid = S.stream_ids(wl)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    xp = (x.astype(np.uint32) << 16).view(np.float32) * cinv[None, :]
    thr = (float(np.median(np.abs(xp).max(axis=1))) * g.uniform(0.6, 1.2, 3)).astype(np.float32)
    gain = g.uniform(0.5, 2.0, (3, 3)).astype(np.float32)
    gain[1, 2] = 0.0  # a zero gain: zero codes for that stream
    y_ref, _, _, _ = oracle.linear_static(x, cinv, sid, thr, gain, L.beta, 1, bits, qw, s_w,
                                          L.bias)
    y = gpu_linear_single(x, cinv, sid, gain, L.beta, 1, bits, qw, s_w, L.bias, thr=thr)
    ok, worst = within_tolerance(y, y_ref)
    assert ok, worst
    y2 = gpu_linear_static(x, cinv, sid, thr, gain, L.beta, 1, bits, qw, s_w, L.bias)
    assert np.array_equal(y, y2)
