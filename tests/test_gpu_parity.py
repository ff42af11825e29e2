"""CUDA path against the CPU oracle, element by element, through the C ABI.

Bit-exact: channel scales, packed weight codes and scales, activation codes and
token scales, int32 accumulators.  bf16 outputs: within
max |y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref) (the GPU epilogue is fp32, the
oracle's fp64).  Small sizes run the oracle on every element; the full block
shapes run on the GPU at full size and are checked on sampled token rows (each
row's result depends only on that row).
"""
import numpy as np
import pytest
import torch

import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

import oracle_pins as P
from gpu_util import (dev, gpu_act_quant, gpu_gemm_s32, gpu_gemm_w4ax, gpu_gemm_w4ax_ws,
                      gpu_linear, gpu_linear_debug, gpu_prep, host, unpack_codes,
                      within_tolerance)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wq.wq_device_status()  # clear any stale error bits
    yield
    assert wq.wq_device_status() == ("WQ_OK", 0)


def _f32bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


# ------------------------------------------------------------------ offline prep

@pytest.mark.parametrize("wl,layer", [(S.TINY, 0), (S.BLOCK2048_A8, 1), (S.BLOCK2048_A8, 3)])
def test_channel_scale_and_pack_bit_exact(oracle, wl, layer):
    L = S.layer_inputs(wl, layer)
    c_ref, cinv_ref = oracle.channel_scale(L.x_cal, L.W)
    qw_ref, sw_ref = oracle.pack_int4(L.W, c_ref)
    c, cinv, qw, s_w = gpu_prep(L.W, L.x_cal)
    assert np.array_equal(_f32bits(host(c)), _f32bits(c_ref))
    assert np.array_equal(_f32bits(host(cinv)), _f32bits(cinv_ref))
    assert np.array_equal(host(qw), qw_ref)
    assert np.array_equal(_f32bits(host(s_w)), _f32bits(sw_ref))


# ------------------------------------------------------------------ activation codes

# M >= 512 with K = 4096 takes the staged-rows kernel (the last round of rows ragged
# here), other M >= 1024 with K <= 4096 the one-warp-per-row kernel, the rest the
# CTA-per-rows one
AQ_SHAPES = [(64, 256), (37, 384), (300, 2048), (16, 8192), (9, 16384), (3, 32768), (1, 128),
             (1100, 256), (1030, 4096), (2048, 2048), (1050, 8192), (1025, 32768),
             (513, 4096), (777, 16384), (600, 8192), (1111, 1024), (1031, 2048)]


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,K", AQ_SHAPES)
def test_act_quant_bit_exact(oracle, M, K, bits):
    g = np.random.default_rng(M * 7 + K)
    wl = S.custom(f"aq{M}x{K}", K, 16, ((0, M - M // 3), (2, M // 3)), act_bits=bits, T=4)
    x = S.activations(wl, 0)
    if M > 3:
        x[2] = 0  # zero row
    sid = g.integers(0, 3, M).astype(np.uint8)  # shuffled stream ids
    alpha = g.uniform(0.5, 1.2, (4, 3)).astype(np.float32)
    cinv = g.uniform(0.2, 4.0, K).astype(np.float32)
    for use_cinv, step in ((True, 3), (False, 0)):
        ci = cinv if use_cinv else None
        q_ref, s_ref = oracle.act_quant(x, ci, sid, alpha, step, bits)
        q, s = gpu_act_quant(x, ci, sid, alpha, step, bits)
        assert np.array_equal(_f32bits(s), _f32bits(s_ref))
        assert np.array_equal(q.view(np.uint8), q_ref.view(np.uint8))


@pytest.mark.parametrize("bits,qmax", [(8, 127), (4, 7)])
def test_act_quant_near_ties_many_rows(oracle, bits, qmax):
    """Near-tie rows tiled to 1024 rows (the one-warp-per-row kernel)."""
    x1, cinv = P.near_tie_inputs(21, K=4096, qmax=qmax)
    x = np.ascontiguousarray(np.repeat(x1, 1024, axis=0))
    sid = np.zeros(x.shape[0], np.uint8)
    alpha = np.ones((1, 1), np.float32)
    q_ref, s_ref = oracle.act_quant(x1, cinv, sid[:1], alpha, 0, bits)
    q, s = gpu_act_quant(x, cinv, sid, alpha, 0, bits)
    assert np.array_equal(_f32bits(s), np.repeat(_f32bits(s_ref), x.shape[0]))
    assert np.array_equal(q.view(np.uint8), np.repeat(q_ref.view(np.uint8), x.shape[0], axis=0))


@pytest.mark.parametrize("bits,qmax", [(8, 127), (4, 7)])
def test_act_quant_near_ties(oracle, bits, qmax):
    for seed in (11, 12, 13):
        x, cinv = P.near_tie_inputs(seed, K=4096, qmax=qmax)
        sid = np.zeros(1, np.uint8)
        alpha = np.ones((1, 1), np.float32)
        q_ref, s_ref = oracle.act_quant(x, cinv, sid, alpha, 0, bits)
        q, s = gpu_act_quant(x, cinv, sid, alpha, 0, bits)
        assert np.array_equal(_f32bits(s), _f32bits(s_ref))
        assert np.array_equal(q.view(np.uint8), q_ref.view(np.uint8))


# ------------------------------------------------------------------ int32 core

# the next four split K over several CTAs (few output tiles, long K), as the fused
# linear does: 16-, 64-, 128- and 256-token tiles
GEMM_SHAPES = [(1, 16, 128), (16, 144, 256), (17, 128, 512), (64, 256, 256), (100, 272, 384),
               (128, 128, 128), (129, 400, 256), (300, 384, 512), (513, 128, 1024),
               (16, 128, 4096), (40, 512, 8192), (100, 384, 8192), (256, 512, 8192),
               (256, 2048, 2048),
               # K % 256 == 128 at narrow token tiles: 128-deep stages over 2-4 issuers
               (33, 256, 384), (48, 192, 1152)]


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_s32_bit_exact(oracle, M, N, K, bits):
    g = np.random.default_rng(M + N + K + bits)
    qw = g.integers(0, 256, (N, K // 2), dtype=np.uint8)       # every nibble incl. -8
    if bits == 8:
        qx = g.integers(-128, 128, (M, K), dtype=np.int8)      # every int8 incl. -128
    else:
        qx = g.integers(0, 256, (M, K // 2), dtype=np.uint8)
    ref = oracle.gemm_s32(qx, bits, qw, K)
    got = gpu_gemm_s32(qx, bits, qw, K)
    assert np.array_equal(got, ref)


def test_gemm_s32_extreme_values(oracle):
    """All-max codes: the largest accumulators the format can produce."""
    M, N, K = 40, 32, 2048
    qx = np.full((M, K), -128, np.int8)
    qw = np.full((N, K // 2), 0x88, np.uint8)  # every code -8
    ref = oracle.gemm_s32(qx, 8, qw, K)
    assert ref[0, 0] == 128 * 8 * K
    assert np.array_equal(gpu_gemm_s32(qx, 8, qw, K), ref)


# ------------------------------------------------------------------ the fused linear

def _check_linear(oracle, x, sid, L, bits, step, rows=None, use_gpu_prep=True):
    """One fused linear through wq_debug_linear_s32 (the product's two launches, with
    the accumulators also written) against the oracle on `rows` (all by default):
    the workspace's codes and token scales bit for bit (4-bit codes are kept one per
    byte there), the int32 accumulators bit for bit, y within the tolerance."""
    c_ref, cinv_ref = oracle.channel_scale(L.x_cal, L.W)
    qw_ref, sw_ref = oracle.pack_int4(L.W, c_ref)
    if use_gpu_prep:
        _, cinv_d, qw_d, sw_d = gpu_prep(L.W, L.x_cal)
    else:
        cinv_d, qw_d, sw_d = cinv_ref, qw_ref, sw_ref
    if rows is None:
        rows = np.arange(x.shape[0])
    y, acc, codes, s_tok = gpu_linear_debug(x, cinv_d, sid, L.alpha, L.beta, step, bits, qw_d,
                                            sw_d, L.bias, rows=rows)
    y_ref, q_ref, s_ref, acc_ref = oracle.linear(x[rows], cinv_ref, sid[rows], L.alpha, L.beta,
                                                 step, bits, qw_ref, sw_ref, L.bias)
    assert np.array_equal(_f32bits(s_tok), _f32bits(s_ref)), "token scales"
    q_ref8 = q_ref if bits == 8 else unpack_codes(q_ref)
    assert np.array_equal(codes, q_ref8), "activation codes"
    assert np.array_equal(acc, acc_ref), "int32 accumulators"
    ok, worst = within_tolerance(y, y_ref)
    assert ok, f"bf16 outputs outside tolerance (worst error/allowance {worst:.3f})"
    return worst


def test_linear_tiny_workload_all_elements(oracle):
    wl = S.TINY
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0)
    _check_linear(oracle, x, S.stream_ids(wl), L, 8, 0)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,K,N", [(300, 512, 384), (1, 256, 16), (33, 1024, 144),
                                   (520, 256, 2048)])
def test_linear_ragged_all_elements(oracle, M, K, N, bits):
    rows = ((0, M - M // 4 - M // 8), (1, M // 8), (2, M // 4))
    wl = S.custom(f"lin{M}x{K}x{N}", K, N, tuple(r for r in rows if r[1] > 0), act_bits=bits, T=3)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0, step=2)
    sid = S.stream_ids(wl)
    _check_linear(oracle, x, sid, L, bits, 2)
    # the debug view is the product path: the plain call gives the same y bit for bit
    _, cinv, qw, s_w = gpu_prep(L.W, L.x_cal)
    y_plain = gpu_linear(x, cinv, sid, L.alpha, L.beta, 2, bits, qw, s_w, L.bias)
    y_dbg = gpu_linear_debug(x, cinv, sid, L.alpha, L.beta, 2, bits, qw, s_w, L.bias)[0]
    assert np.array_equal(y_plain, y_dbg)


@pytest.mark.parametrize("Sn", [4, 6, 7])
def test_linear_many_streams_and_optional_inputs(oracle, Sn):
    """S = 4 (the largest per-lane table), 6 and 7 (> 4: per-element table reads),
    shuffled ids, no bias, no beta, no cinv."""
    g = np.random.default_rng(5 + Sn)
    M, K, N, T = 200, 384, 272, 5
    wl = S.custom("many", K, N, ((0, M),), act_bits=8, T=T)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0)
    sid = g.integers(0, Sn, M).astype(np.uint8)
    alpha = g.uniform(0.7, 1.0, (T, Sn)).astype(np.float32)
    beta = g.normal(0, 1e-2, (T, Sn, N)).astype(np.float32)
    qw_ref, sw_ref = oracle.pack_int4(L.W, None)
    for bias, bt, step in ((L.bias, beta, 4), (None, beta, 1), (L.bias, None, 0), (None, None, 2)):
        y = gpu_linear(x, None, sid, alpha, bt, step, 8, qw_ref, sw_ref, bias)
        y_ref, _, _, _ = oracle.linear(x, None, sid, alpha, bt, step, 8, qw_ref, sw_ref, bias)
        ok, worst = within_tolerance(y, y_ref)
        assert ok, worst


def test_linear_empty_batch():
    K, N = 256, 64
    y = torch.zeros((0, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    x = torch.zeros((0, K), dtype=torch.bfloat16, device="cuda")
    sid = torch.zeros(1, dtype=torch.uint8, device="cuda")
    alpha = torch.ones((1, 3), dtype=torch.float32, device="cuda")
    qw = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    s_w = torch.ones(N, dtype=torch.float32, device="cuda")
    st = wq.lib().wq_linear_w4a8(x.data_ptr(), 0, K, N, None, sid.data_ptr(), alpha.data_ptr(),
                                 None, 3, 1, 0, qw.data_ptr(), s_w.data_ptr(), None, y.data_ptr(),
                                 ws.data_ptr(), 256, None)
    assert st == 0


# ------------------------------------------------------------------ full-size shapes, sampled
# Every layer of both blocks at full size (K up to 16384, M = 4288 and 8512), through
# the same two launches the benchmark times: codes, token scales and int32
# accumulators of the sampled token rows bit for bit, y within the tolerance.

def _sample_rows(wl, n_random, seed=0):
    """Every stream's first and last rows, the batch's last row, and random rows."""
    g = np.random.default_rng(seed)
    M = wl.M
    edges, start = [], 0
    for _, cnt in wl.rows:
        edges += [start, start + cnt - 1]
        start += cnt
    rows = set(edges) | {M - 1} | set(g.choice(M, n_random, replace=False).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("wl,step", [(S.BLOCK2048_A8, 0), (S.BLOCK2048_A4, 9)],
                         ids=["block2048_w4a8", "block2048_w4a4_step9"])
@pytest.mark.parametrize("layer", [0, 1, 2, 3])
def test_block2048_full_size_sampled_rows(oracle, wl, step, layer):
    L = S.layer_inputs(wl, layer)
    x = S.activations(wl, layer, step)
    _check_linear(oracle, x, S.stream_ids(wl), L, wl.act_bits, step,
                  rows=_sample_rows(wl, 24, seed=layer))


@pytest.mark.parametrize("wl", [S.BLOCK4096_A8, S.BLOCK4096_A4], ids=["w4a8", "w4a4"])
@pytest.mark.parametrize("layer", [0, 1, 2, 3])
def test_block4096_full_size_sampled_rows(oracle, wl, layer):
    L = S.layer_inputs(wl, layer)
    step = 5
    x = S.activations(wl, layer, step)
    _check_linear(oracle, x, S.stream_ids(wl), L, wl.act_bits, step,
                  rows=_sample_rows(wl, 4, seed=layer))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M", S.SMALL_M)
def test_small_m_weight_streaming(oracle, M, bits):
    for parent, layer, mix in ((S.BLOCK2048_A8, 0, "action"), (S.BLOCK4096_A8, 2, "proprio_action")):
        wl = S.small_m(parent, M, mix, bits)
        L = S.layer_inputs(wl, layer)
        x = S.activations(wl, layer, 0)
        rows = None if M <= 64 else np.arange(0, M, 7)
        _check_linear(oracle, x, S.stream_ids(wl), L, bits, 0, rows=rows)


# ------------------------------------------------------------------ GEMM-only entry point

@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (300, 512, 384), (520, 256, 2048),
                                   (33, 1024, 144), (4288, 2048, 2048)])
def test_gemm_w4ax_against_oracle(oracle, M, K, N, bits):
    """wq_gemm_w4ax on the oracle's codes and token scales: int8 codes, or packed
    int4 codes (the packed-activation mainloop, which unpacks them per tile)."""
    rows_ = ((0, M - M // 4 - M // 8), (1, M // 8), (2, M // 4))
    wl = S.custom(f"gemm{M}x{K}x{N}", K, N, tuple(r for r in rows_ if r[1] > 0), act_bits=bits,
                  T=3)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0, step=1)
    sid = S.stream_ids(wl)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    qx, s_tok = oracle.act_quant(x, cinv, sid, L.alpha, 1, bits)
    y = gpu_gemm_w4ax(qx, s_tok, bits, K, sid, L.beta, 1, qw, s_w, L.bias)
    rows = np.arange(M) if M <= 600 else _sample_rows(wl, 24)
    acc = oracle.gemm_s32(qx[rows], bits, qw, K)
    y_ref = oracle.epilogue(acc, s_tok[rows], s_w, L.bias, L.beta, sid[rows], 1)
    ok, worst = within_tolerance(y[rows], y_ref)
    assert ok, worst



@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("M,K,N", [(16, 4096, 512), (40, 8192, 256), (64, 4096, 384),
                                   (1, 256, 16), (300, 8192, 384)])
def test_gemm_w4ax_ws_split_matches(oracle, M, K, N, bits):
    """wq_gemm_w4ax_ws: few tokens split K over every SM through the workspace (a
    garbage-filled one: the call clears it); y bit-identical to wq_gemm_w4ax (int32
    sums are exact in any order) and within tolerance of the oracle.  300 tokens at
    K = 8192 split on single-CTA 256-token tiles; one token with K = 256 does not split
    (no workspace needed)."""
    rows_ = ((0, M - M // 4 - M // 8), (1, M // 8), (2, M // 4))
    wl = S.custom(f"gemmws{M}x{K}x{N}", K, N, tuple(r for r in rows_ if r[1] > 0),
                  act_bits=bits, T=3)
    L = S.layer_inputs(wl, 0)
    x = S.activations(wl, 0, step=1)
    sid = S.stream_ids(wl)
    c, cinv = oracle.channel_scale(L.x_cal, L.W)
    qw, s_w = oracle.pack_int4(L.W, c)
    qx, s_tok = oracle.act_quant(x, cinv, sid, L.alpha, 1, bits)
    y_ws, nbytes = gpu_gemm_w4ax_ws(qx, s_tok, bits, K, sid, L.beta, 1, qw, s_w, L.bias)
    assert (nbytes > 0) == (M != 1)  # the 1-token shape (K = 256) does not split
    y = gpu_gemm_w4ax(qx, s_tok, bits, K, sid, L.beta, 1, qw, s_w, L.bias)
    assert np.array_equal(y_ws, y)
    acc = oracle.gemm_s32(qx, bits, qw, K)
    y_ref = oracle.epilogue(acc, s_tok, s_w, L.bias, L.beta, sid, 1)
    ok, worst = within_tolerance(y_ws, y_ref)
    assert ok, worst


@pytest.mark.parametrize("M", [16, 256])
@pytest.mark.parametrize("parent,layer", [(p, i) for p in (S.BLOCK2048_A8, S.BLOCK4096_A8)
                                          for i in range(4)],
                         ids=[f"{p}_{n}" for p in ("h2048", "h4096")
                              for n in ("qkv", "attn_out", "mlp_up", "mlp_down")])
def test_small_m_every_weight_shape(oracle, parent, layer, M):
    """Every small-M weight shape at 16 and 256 action tokens: the split of K over
    CTAs (int32 partial tiles summed through the workspace) gives the exact sums."""
    wl = S.small_m(parent, M, "action", 8)
    L = S.layer_inputs(wl, layer)
    x = S.activations(wl, layer, 0)
    _check_linear(oracle, x, S.stream_ids(wl), L, 8, 0,
                  rows=None if M <= 16 else np.arange(0, M, 5))
