"""Which GEMM instances the GPU parity tests run, checked on the CPU.

The library's plan query (host arithmetic, no device) names the kernel instance a call
runs for a shape: the activation-code format of the mainloop, the epilogue, the token
tile, CTAs per tile and the stage depth.  The GPU tests' shapes are read from their
parameter lists here, mapped to instances, and compared with

  * the instances the configured workloads run (tiny, both blocks at full size with
    int8 and int4 codes, the small token counts, the FFN pair): every one of them must
    be among those the GPU tests run, so a change of the dispatch rules that moves a
    configured shape onto an untested instance fails here;
  * every instance the dispatch can choose: the ones no GPU test runs yet are listed
    below, so that list cannot grow unnoticed.
"""
import activation_quantized_gemm_wq_b200 as wq
from activation_quantized_gemm_wq_b200 import synth as S

import test_gpu_gelu as G
import test_gpu_parity as P

# (code bits of the mainloop, epilogue: 0 = y, 8 / 4 = GELU then codes of that width,
#  token tile, CTAs per tile, K depth per stage)
KNOWN_UNTESTED = {
    (4, 0, 32, 1, 128), (8, 0, 32, 1, 128),
    (8, 8, 16, 1, 128), (8, 8, 32, 1, 128), (8, 8, 32, 1, 256), (8, 8, 64, 1, 128),
    (8, 8, 128, 1, 128), (8, 8, 256, 1, 128),
    (8, 4, 16, 1, 128), (8, 4, 32, 1, 128), (8, 4, 32, 1, 256), (8, 4, 64, 1, 128),
    (8, 4, 128, 1, 128), (8, 4, 256, 1, 128),
}


# One small shape per untested instance: (call, M, K, N, code bits of the GEMM call, or
# the next linear's code width for gelu_quant); K % 256 == 128 selects the 128-deep
# stages at <= 64 tokens, and 200 tokens with K = 16384 on 256 channels split K.
SHAPE_FOR_UNTESTED = {
    (4, 0, 32, 1, 128): ("gemm", 32, 384, 256, 4),
    (8, 0, 32, 1, 128): ("gemm", 32, 384, 256, 8),
}
for _e in (8, 4):
    SHAPE_FOR_UNTESTED.update({
        (8, _e, 16, 1, 128): ("gelu_quant", 16, 384, 256, _e),
        (8, _e, 32, 1, 128): ("gelu_quant", 32, 384, 256, _e),
        (8, _e, 32, 1, 256): ("gelu_quant", 32, 512, 256, _e),
        (8, _e, 64, 1, 128): ("gelu_quant", 64, 384, 256, _e),
        (8, _e, 128, 1, 128): ("gelu_quant", 100, 512, 256, _e),
        (8, _e, 256, 1, 128): ("gelu_quant", 200, 16384, 256, _e),
    })


def instance(M, K, N, bits, call, epi=0):
    """The instance `call` runs for (M, K, N), or None for an empty batch.  The fused
    calls keep one code per byte, so their mainloop takes int8 codes at either width."""
    p = wq.wq_gemm_plan_query(M, K, N, bits, call)
    if p["tile_tokens"] == 0:
        return None
    code_bits = bits if call in ("gemm", "gemm_ws") else 8
    return (code_bits, epi, p["tile_tokens"], p["ctas_per_tile"], p["k_stage"])


def params(fn, names):
    """The values of one parametrize mark of a test function, as tuples."""
    for m in getattr(fn, "pytestmark", []):
        if m.name == "parametrize" and m.args[0].replace(" ", "") == names:
            return [v if isinstance(v, tuple) else (v,) for v in m.args[1]]
    raise KeyError(f"{fn.__name__} has no parametrize mark for {names}")


def dispatchable():
    out = set()
    for bits in (8, 4):
        for t in (16, 32, 64):
            out |= {(bits, 0, t, 1, 128), (bits, 0, t, 1, 256)}
        out |= {(bits, 0, 128, 1, 128), (bits, 0, 256, 1, 128)}
    out |= {(8, 0, 224, 2, 128), (8, 0, 256, 2, 128)}
    for epi in (8, 4):
        for t in (16, 32, 64):
            out |= {(8, epi, t, 1, 128), (8, epi, t, 1, 256)}
        out |= {(8, epi, 128, 1, 128), (8, epi, 256, 1, 128), (8, epi, 256, 2, 128)}
    return out


def covered():
    cov = set()
    bits_both = params(P.test_gemm_s32_bit_exact, "bits")
    for (M, N, K) in params(P.test_gemm_s32_bit_exact, "M,N,K"):
        for (b,) in bits_both:
            cov.add(instance(M, K, N, b, "gemm_ws"))
    for (M, K, N) in params(P.test_linear_ragged_all_elements, "M,K,N"):
        cov.add(instance(M, K, N, 8, "linear"))
    for wl, _step in params(P.test_block2048_full_size_sampled_rows, "wl,step"):
        cov |= {instance(wl.M, lin.K, lin.N, 8, "linear") for lin in wl.linears}
    for (wl,) in params(P.test_block4096_full_size_sampled_rows, "wl"):
        cov |= {instance(wl.M, lin.K, lin.N, 8, "linear") for lin in wl.linears}
    # the body of test_small_m_weight_streaming: hidden-2048 qkv, hidden-4096 mlp_up
    for (M,) in params(P.test_small_m_weight_streaming, "M"):
        for parent, layer in ((S.BLOCK2048_A8, 0), (S.BLOCK4096_A8, 2)):
            lin = parent.linears[layer]
            cov.add(instance(M, lin.K, lin.N, 8, "linear"))
    for (M,) in params(P.test_small_m_every_weight_shape, "M"):
        for parent, layer in params(P.test_small_m_every_weight_shape, "parent,layer"):
            lin = parent.linears[layer]
            cov.add(instance(M, lin.K, lin.N, 8, "linear"))
    for (M, K, N) in params(P.test_gemm_w4ax_against_oracle, "M,K,N"):
        for (b,) in params(P.test_gemm_w4ax_against_oracle, "bits"):
            cov.add(instance(M, K, N, b, "gemm"))
    for (M, K, N) in params(P.test_gemm_w4ax_ws_split_matches, "M,K,N"):
        for (b,) in params(P.test_gemm_w4ax_ws_split_matches, "bits"):
            cov |= {instance(M, K, N, b, "gemm_ws"), instance(M, K, N, b, "gemm")}
    for (M, K, N, _wide) in params(G.test_gelu_quant_against_oracle, "M,K,N,wide"):
        for _bits_up, bits_next in params(G.test_gelu_quant_against_oracle,
                                          "bits_up,bits_next"):
            cov.add(instance(M, K, N, 8, "gelu_quant", bits_next))
            cov.add(instance(M, K, N, 8, "linear"))
        # the down-projection on those codes: 256 output channels, K = N
        cov |= {instance(M, N, 256, 8, "gemm_ws"), instance(M, N, 256, 8, "gemm")}
    cov.discard(None)
    return cov


def configured():
    need = set()
    for wl in (S.TINY, S.BLOCK2048_A8, S.BLOCK2048_A4, S.BLOCK4096_A8, S.BLOCK4096_A4):
        for lin in wl.linears:
            need.add(instance(wl.M, lin.K, lin.N, 8, "linear"))
            need.add(instance(wl.M, lin.K, lin.N, wl.act_bits, "gemm_ws"))
    for parent in (S.BLOCK2048_A8, S.BLOCK4096_A8):
        for M in S.SMALL_M:
            for lin in parent.linears:
                need.add(instance(M, lin.K, lin.N, 8, "linear"))
                need |= {instance(M, lin.K, lin.N, b, "gemm_ws") for b in (8, 4)}
        up, down = parent.linears[2], parent.linears[3]
        need |= {instance(parent.M, up.K, up.N, 8, "gelu_quant", e) for e in (8, 4)}
        need.add(instance(parent.M, down.K, down.N, 8, "gemm_ws"))
    return need


def test_every_configured_instance_runs_in_a_gpu_test():
    missing = configured() - covered()
    assert not missing, f"configured shapes on instances no GPU test runs: {sorted(missing)}"


def test_the_untested_instances_are_the_known_ones():
    cov = covered()
    assert cov <= dispatchable(), sorted(cov - dispatchable())
    assert dispatchable() - cov == KNOWN_UNTESTED


def test_both_pair_widths_and_the_split_path_are_covered():
    cov = covered()
    assert {(8, 0, 224, 2, 128), (8, 0, 256, 2, 128), (8, 0, 256, 1, 128),
            (8, 8, 256, 2, 128), (8, 4, 256, 2, 128)} <= cov


def test_each_untested_instance_has_a_shape_that_reaches_it():
    """The parity shapes to add next: each reaches its instance."""
    assert set(SHAPE_FOR_UNTESTED) == KNOWN_UNTESTED
    for inst, (call, M, K, N, bits) in SHAPE_FOR_UNTESTED.items():
        if call == "gelu_quant":
            assert instance(M, K, N, 8, call, bits) == inst
        else:
            assert instance(M, K, N, bits, call) == inst
