"""A stream id outside the table (>= S) is a precondition the device checks: that
row gets scale 0 and all-zero codes, its output is the bias alone (no row of the
compensation table is read for it), and wq_device_status reports
WQ_ERR_DEVICE with the stream-id bit.  The other rows are unaffected."""
import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

from gpu_util import gpu_linear_debug, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wq.wq_device_status()
    yield
    assert wq.wq_device_status() == ("WQ_OK", 0)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("Sn,bad_id", [(3, 3), (3, 200), (4, 4), (6, 6), (7, 9)])
def test_bad_stream_id_gives_bias_and_device_error(oracle, Sn, bad_id, bits):
    g = np.random.default_rng(Sn * 31 + bad_id)
    M, K, N, T = 96, 256, 160, 3
    wl = S.custom(f"badid{Sn}", K, N, ((0, M),), act_bits=bits, T=T)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0)
    sid = g.integers(0, Sn, M).astype(np.uint8)
    bad = np.array([5, 17, M - 1])
    sid[bad] = bad_id
    alpha = g.uniform(0.8, 1.0, (T, Sn)).astype(np.float32)
    beta = g.normal(0, 1e-2, (T, Sn, N)).astype(np.float32)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    step = T - 1  # the last table row: a bad id there would read past the table
    wq.wq_device_status()
    y, acc, codes, s_tok = gpu_linear_debug(x, cinv, sid, alpha, beta, step, bits, qw, s_w,
                                            L.bias)
    torch.cuda.synchronize()
    assert wq.wq_device_status() == ("WQ_ERR_DEVICE", 2)
    # the bad rows: scale 0, codes 0, sums 0, y = bf16(bias) exactly
    assert np.all(s_tok[bad] == 0) and not codes[bad].any() and not acc[bad].any()
    bias_bf16 = ((L.bias.astype(np.float32).view(np.uint32) + 0x7FFF +
                  ((L.bias.astype(np.float32).view(np.uint32) >> 16) & 1)) >> 16).astype(np.uint16)
    assert np.array_equal(y[bad], np.broadcast_to(bias_bf16, (len(bad), N)))
    # every other row as the oracle computes it
    good = np.setdiff1d(np.arange(M), bad)
    y_ref, _, _, acc_ref = oracle.linear(x[good], cinv, sid[good], alpha, beta, step, bits, qw,
                                         s_w, L.bias)
    assert np.array_equal(acc[good], acc_ref)
    ok, worst = within_tolerance(y[good], y_ref)
    assert ok, worst
