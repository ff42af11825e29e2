"""wq_linear_w4a8_noalloc: the fused W4A8 linear for callers that cannot
allocate device memory while they run (a real-time controller loop, or a host
that gives the library no allocator).  It keeps the codes and token scales in
the library's fixed 16 MiB scratch instead of a caller workspace.

Checked through the C ABI against wq_linear_w4a8 (which uses a caller
workspace) on two calls in a row with different inputs, so stale scratch
contents from the first call cannot leak into the second.  Both run the same two
kernels on the same inputs, so their outputs must be equal bit for bit; the
first call is also compared with the CPU oracle, within the tolerance the other
tests use.  This file is collected last, and it needs nothing from the other test
files, so it passes alone in a fresh process as well as after them."""
import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

pytestmark = pytest.mark.gpu


def _dev(a):
    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()


def _f64(y):
    return y.float().cpu().numpy().astype(np.float64)


def _within_tolerance(y, ref):
    """max |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref), element-wise."""
    rms = np.sqrt(np.mean(ref ** 2))
    return bool(np.all(np.abs(y - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-3 * rms))


def _oracle_y(wl, x_host, step):
    """The oracle's y (as float64) for the first linear of `wl` on activations x_host."""
    from oracle import Oracle
    orc = Oracle()
    L = S.layer_inputs(wl, 0)
    c, cinv = orc.channel_scale(L.x_cal, L.W)
    qw, s_w = orc.pack_int4(L.W, c)
    rows = np.arange(x_host.shape[0]) if x_host.shape[0] <= 512 else \
        np.arange(0, x_host.shape[0], 61)
    y = orc.linear(x_host[rows], cinv, S.stream_ids(wl)[rows], L.alpha, L.beta, step, 8, qw,
                   s_w, L.bias)[0]
    return rows, (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _prepared(wl):
    L = S.layer_inputs(wl, 0)
    K, N = L.W.shape[1], L.W.shape[0]
    c = torch.empty(K, dtype=torch.float32, device="cuda")
    cinv = torch.empty_like(c)
    qw = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    s_w = torch.empty(N, dtype=torch.float32, device="cuda")
    W = _dev(L.W)
    wq.wq_channel_scale(_dev(L.x_cal), W, c, cinv)
    wq.wq_pack_int4(W, c, qw, s_w)
    return L, cinv, qw, s_w


@pytest.mark.parametrize("wl", [
    S.TINY,
    S.custom("noalloc_mid", 512, 384, ((0, 200), (1, 40), (2, 60)), T=3),
    S.custom("noalloc_big", 2048, 2048, ((0, 4096), (1, 64), (2, 128)), T=1),
], ids=["tiny", "mid", "4288x2048"])
def test_noalloc_matches_workspace_linear_twice(wl):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L, cinv, qw, s_w = _prepared(wl)
    sid = _dev(S.stream_ids(wl))
    alpha, beta, bias = _dev(L.alpha), _dev(L.beta), _dev(L.bias)
    M, K, N = wl.M, wl.linears[0].K, wl.linears[0].N
    ws = wq.alloc_workspace(M, K, N, 8)
    step = wl.T - 1
    for call in range(2):  # two calls in a row, different activations each time
        x_host = S.activations(wl, 0, step=call % wl.T, seed=call)
        x = _dev(x_host)
        y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        wq.wq_linear_w4a8(x, cinv, sid, alpha, beta, step, qw, s_w, bias, y_ref, ws)
        wq.wq_linear_w4a8_noalloc(x, cinv, sid, alpha, beta, step, qw, s_w, bias, y)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: equal bit for bit
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), f"call {call} differs"
        if call == 0:  # and right, as the oracle computes it
            rows, y_orc = _oracle_y(wl, x_host, step)
            assert _within_tolerance(_f64(y)[rows], y_orc), "differs from the oracle"
    assert wq.wq_device_status() == ("WQ_OK", 0)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = wq.lib()
    fake = 1 << 20  # never dereferenced: the size check comes first
    # 4096 tokens x 8192 channels of int8 codes = 32 MiB > 16 MiB
    st = lib.wq_linear_w4a8_noalloc(fake, 4096, 8192, 256, None, fake, fake, None, 3, 1, 0, fake,
                                    fake, None, fake, None)
    assert wq.STATUS[st] == "WQ_ERR_SCRATCH"
    assert wq.lib().wq_status_string(st).decode().startswith("WQ_ERR_SCRATCH")
