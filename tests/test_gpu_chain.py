"""Back-to-back fused linears in one stream, as a model runs them: each linear's
output is the next one's input, so the quantizer of linear i+1 must wait for the
GEMM of linear i (programmatic dependent launch lets it start early), and the
GEMM's early weight loads must not overtake anything the stream wrote before.
Also: the same chain captured in a CUDA graph and replayed gives the same bits."""
import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

from gpu_util import dev, host, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wq.wq_device_status()
    yield
    assert wq.wq_device_status() == ("WQ_OK", 0)


def _chain_layers(oracle, dims, M, bits, seed):
    """Weights packed on the GPU (so the pack kernel immediately precedes the chain
    in the stream) and the same weights packed by the oracle."""
    g = np.random.default_rng(seed)
    layers = []
    for i in range(len(dims) - 1):
        K, N = dims[i], dims[i + 1]
        W = S.f32_to_bf16_bits(g.normal(0, 0.05, (N, K)).astype(np.float32))
        c = g.uniform(0.5, 2.0, K).astype(np.float32)
        cinv = (np.float32(1.0) / c).astype(np.float32)
        qw_ref, sw_ref = oracle.pack_int4(W, c)
        qw = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        s_w = torch.empty(N, dtype=torch.float32, device="cuda")
        wq.wq_pack_int4(dev(W), dev(c), qw, s_w)
        bias = g.normal(0, 0.01, N).astype(np.float32)
        alpha = g.uniform(0.85, 1.0, (2, 3)).astype(np.float32)
        beta = g.normal(0, 1e-3, (2, 3, N)).astype(np.float32)
        layers.append(dict(K=K, N=N, cinv=cinv, qw=qw, s_w=s_w, qw_ref=qw_ref, sw_ref=sw_ref,
                           bias=bias, alpha=alpha, beta=beta))
    return layers


def _run_chain(layers, x_dev, sid_dev, bits, step, outs, wss):
    fn = wq.wq_linear_w4a8 if bits == 8 else wq.wq_linear_w4a4
    cur = x_dev
    for L, y, ws in zip(layers, outs, wss):
        fn(cur, L["cinv_d"], sid_dev, L["alpha_d"], L["beta_d"], step, L["qw"], L["s_w"],
           L["bias_d"], y, ws)
        cur = y
    return cur


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M", [16, 300])
def test_dependent_chain_matches_oracle_and_graph(oracle, bits, M):
    dims = [512, 1024, 384, 2048, 256]
    layers = _chain_layers(oracle, dims, M, bits, seed=M + bits)
    for L in layers:
        L["cinv_d"], L["bias_d"] = dev(L["cinv"]), dev(L["bias"])
        L["alpha_d"], L["beta_d"] = dev(L["alpha"]), dev(L["beta"])
    g = np.random.default_rng(7)
    x = S.f32_to_bf16_bits(g.normal(0, 1.0, (M, dims[0])).astype(np.float32))
    sid = np.sort(g.integers(0, 3, M)).astype(np.uint8)
    x_dev, sid_dev = dev(x), dev(sid)
    outs = [torch.empty((M, L["N"]), dtype=torch.bfloat16, device="cuda") for L in layers]
    wss = [wq.alloc_workspace(M, L["K"], L["N"], bits) for L in layers]
    step = 1

    # eager, right after the weights were packed on the GPU in the same stream
    y_last = _run_chain(layers, x_dev, sid_dev, bits, step, outs, wss)
    eager = [host(o.view(torch.int16), np.uint16).copy() for o in outs]

    # the oracle, layer by layer on the GPU's own bf16 outputs: each layer checked
    # against the oracle given the same input, so errors do not compound
    inp = x
    for L, y in zip(layers, eager):
        y_ref, _, _, _ = oracle.linear(inp, L["cinv"], sid, L["alpha"], L["beta"], step, bits,
                                       L["qw_ref"], L["sw_ref"], L["bias"])
        ok, worst = within_tolerance(y, y_ref)
        assert ok, worst
        inp = y
    assert np.array_equal(eager[-1], host(y_last.view(torch.int16), np.uint16))

    # the same chain as one CUDA graph, replayed twice
    for o in outs:
        o.zero_()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _run_chain(layers, x_dev, sid_dev, bits, step, outs, wss)  # warm outside capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        _run_chain(layers, x_dev, sid_dev, bits, step, outs, wss)
    for _ in range(2):
        for o in outs:
            o.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for o, e in zip(outs, eager):
            assert np.array_equal(host(o.view(torch.int16), np.uint16), e)
    del graph
