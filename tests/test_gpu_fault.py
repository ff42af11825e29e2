"""Failure handling of the GEMM's bounded waits, without a GPU fault: a test hook
leaves one pipeline stage of CTA 0 a copy short, so the waits on it can never
complete.  With the wait limit lowered to 50 ms the launch must end on its own
(every wait bounded, copies and MMAs in flight drained, tensor memory freed), the
device error word must read WQ_ERR_TIMEOUT, and, once the hook is off and the word
cleared, the next call on the same context must be correct."""
import time

import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

from gpu_util import gpu_linear, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wq.wq_device_status()
    yield
    wq.wq_debug_inject_stall(False)
    assert wq.wq_device_status() == ("WQ_OK", 0)


# one CTA and one tile; a split of K over many CTAs (few tiles, long K); many CTAs with
# several tiles each
@pytest.mark.parametrize("M,K,N", [(64, 256, 128), (300, 8192, 384), (4288, 2048, 2048)])
def test_stalled_stage_times_out_and_the_context_recovers(oracle, M, K, N):
    rows = ((0, M - M // 4), (2, M // 4))
    wl = S.custom(f"stall{M}x{K}x{N}", K, N, rows, act_bits=8, T=1)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0)
    sid = S.stream_ids(wl)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    assert wq.wq_device_status() == ("WQ_OK", 0)
    wq.wq_debug_inject_stall(True, 50_000)
    try:
        t0 = time.perf_counter()
        gpu_linear(x, cinv, sid, L.alpha, L.beta, 0, 8, qw, s_w, L.bias)  # synchronizes
        elapsed = time.perf_counter() - t0
        status, flags = wq.wq_device_status()
    finally:
        wq.wq_debug_inject_stall(False)
    assert status == "WQ_ERR_TIMEOUT" and flags & 1, (status, flags)
    assert elapsed < 1.5, f"the stalled launch took {elapsed:.2f} s to end"
    # the same context, hook off and error word cleared: correct results again
    y = gpu_linear(x, cinv, sid, L.alpha, L.beta, 0, 8, qw, s_w, L.bias)
    assert wq.wq_device_status() == ("WQ_OK", 0)
    sel = np.arange(M) if M <= 512 else np.arange(0, M, 97)
    y_ref = oracle.linear(x[sel], cinv, sid[sel], L.alpha, L.beta, 0, 8, qw, s_w, L.bias)[0]
    ok, worst = within_tolerance(y[sel], y_ref)
    assert ok, worst
