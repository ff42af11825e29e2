"""Seeded synthetic inputs: determinism, layout and the stated distributions."""
import numpy as np

from activation_quantized_gemm_wq_b200 import synth as S


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_deterministic_and_distinct():
    wl = S.TINY
    a, b = S.layer_inputs(wl, 0), S.layer_inputs(wl, 0)
    assert np.array_equal(a.W, b.W) and np.array_equal(a.x_cal, b.x_cal)
    assert np.array_equal(S.activations(wl, 0), S.activations(wl, 0))
    assert not np.array_equal(S.activations(wl, 0, seed=0), S.activations(wl, 0, seed=1))
    w2 = S.BLOCK2048_A4
    assert not np.array_equal(S.activations(w2, 1, 0)[:64], S.activations(w2, 1, 1)[:64])


def test_tiny_layout_and_tables():
    wl = S.TINY
    sid = S.stream_ids(wl)
    assert sid.shape == (64,)
    assert (sid[:48] == 0).all() and (sid[48:56] == 1).all() and (sid[56:] == 2).all()
    L = S.layer_inputs(wl, 0)
    assert L.W.shape == (256, 256) and L.x_cal.shape == (256, 256)
    np.testing.assert_array_equal(L.alpha, np.float32([[1.0, 0.95, 0.9]]))
    assert L.beta.shape == (1, 3, 256)


def test_stream_stds_and_outliers():
    wl = S.custom("stats", 1024, 16, ((0, 512), (1, 256), (2, 256)), outlier_frac=0.01,
                  outlier_range=(20.0, 50.0))
    x = _f(S.activations(wl, 0))
    mult_cols = np.abs(x).max(axis=0) > 15  # outlier channels stand out in every stream
    assert mult_cols.sum() == round(0.01 * 1024)
    plain = ~mult_cols
    for s, lo, hi, std in ((0, 0, 512, 1.0), (1, 512, 768, 3.0), (2, 768, 1024, 0.5)):
        got = x[lo:hi][:, plain].std()
        assert abs(got - std) < 0.05 * std
    assert S.small_m(S.BLOCK4096_A8, 32, "proprio_action", 4).rows == ((1, 8), (2, 24))


def test_block_workloads():
    assert S.BLOCK2048_A8.M == 4288 and S.BLOCK4096_A8.M == 8512
    assert [(l.K, l.N) for l in S.BLOCK2048_A8.linears] == [(2048, 6144), (2048, 2048),
                                                             (2048, 8192), (8192, 2048)]
    assert S.BLOCK4096_A4.T == 10 and S.BLOCK4096_A4.act_bits == 4
    L = S.layer_inputs(S.BLOCK2048_A4, 1)
    assert L.alpha.shape == (10, 3) and (L.alpha >= 0.85).all() and (L.alpha <= 1.0).all()
    cal = S._cal_rows(S.BLOCK2048_A8)
    assert cal.shape == (256,) and set(np.unique(cal)) == {0, 1, 2}
