"""Static clipping (the layer-step table read as a shared threshold per step and a
gain per stream, SteerQuant §4.3) on the GPU against the oracle: codes and token
scales bit for bit, the fused linear within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

from gpu_util import gpu_act_quant_static, gpu_linear_static, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wq.wq_device_status()
    yield
    assert wq.wq_device_status() == ("WQ_OK", 0)


def _bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


def _tables(g, T, Sn, x, cinv, qmax):
    """Thresholds near the activations' typical row maxima (so some elements
    saturate and most do not), gains in [0.5, 2], and one zero gain."""
    xp = (x.astype(np.uint32) << 16).view(np.float32) * (1.0 if cinv is None else cinv[None, :])
    typical = float(np.median(np.abs(xp).max(axis=1))) or 1.0
    thr = (typical * g.uniform(0.6, 1.2, T)).astype(np.float32)
    gain = g.uniform(0.5, 2.0, (T, Sn)).astype(np.float32)
    gain[0, Sn - 1] = 0.0
    return thr, gain


@pytest.mark.parametrize("bits,qmax", [(8, 127), (4, 7)])
@pytest.mark.parametrize("M,K", [(64, 256), (300, 2048), (16, 8192), (3, 32768), (37, 384),
                                 (1200, 2048), (1030, 4096), (515, 8192), (601, 16384)])
def test_act_quant_static_bit_exact(oracle, M, K, bits, qmax):
    g = np.random.default_rng(M * 13 + K)
    wl = S.custom(f"st{M}x{K}", K, 16, ((0, M),), act_bits=bits, T=3)
    x = S.activations(wl, 0)
    sid = g.integers(0, 3, M).astype(np.uint8)
    cinv = g.uniform(0.2, 4.0, K).astype(np.float32)
    thr, gain = _tables(g, 3, 3, x, cinv, qmax)
    for ci, step in ((cinv, 2), (None, 0)):
        q_ref, s_ref = oracle.act_quant_static(x, ci, sid, thr, gain, step, bits)
        q, s = gpu_act_quant_static(x, ci, sid, thr, gain, step, bits)
        assert np.array_equal(_bits(s), _bits(s_ref))
        assert np.array_equal(q.view(np.uint8), q_ref.view(np.uint8))


@pytest.mark.parametrize("bits,qmax", [(8, 127), (4, 7)])
@pytest.mark.parametrize("M,K,N", [(300, 512, 384), (16, 2048, 1024), (1, 256, 16),
                                   (700, 4096, 256)])
def test_linear_static_matches_oracle(oracle, M, K, N, bits, qmax):
    g = np.random.default_rng(M + K + N)
    rows = ((0, M - M // 4), (2, M // 4))
    wl = S.custom(f"ls{M}x{K}x{N}", K, N, tuple(r for r in rows if r[1] > 0), act_bits=bits, T=3)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0, step=1)
    sid = S.stream_ids(wl)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    thr, gain = _tables(g, 3, 3, x, cinv, qmax)
    for step in (1, 0):
        y_ref, _, _, _ = oracle.linear_static(x, cinv, sid, thr, gain, L.beta, step, bits, qw,
                                              s_w, L.bias)
        y = gpu_linear_static(x, cinv, sid, thr, gain, L.beta, step, bits, qw, s_w, L.bias)
        ok, worst = within_tolerance(y, y_ref)
        assert ok, worst
