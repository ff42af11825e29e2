"""The GELU-and-quantize GEMM epilogue takes bf16(GELU(y)) from a table for
2^-10 <= |y| < 16 and, outside it, from two closed forms instead of evaluating erfc:

  * a normal y with |y| < 2^-10 gives h = y/2 (the exponent field minus one), since
    GELU(y) = y/2 (1 + erf(y/sqrt 2)) and |erf(y/sqrt 2)| < 0.0008 is below half of
    bf16's relative spacing;
  * finite y >= 16 gives h = y, since 1 - Phi(16) < 2^-60;
  * finite y <= -16 gives h = -0, since |GELU(y)| < 2^-180 there, far below bf16's
    smallest subnormal (2^-133).

Zeros, subnormals, infinities and NaN stay with the evaluation.

Both are statements about the correctly rounded GELU (SteerQuant App. D keeps GELU in
BF16), so they are checked here against the oracle's fp64 GELU over every bf16
pattern they claim; the patterns they leave to the evaluation are listed too.
"""
import numpy as np

TAB_EXP0, TAB_EXPS = 117, 14
TAB_END = TAB_EXP0 + TAB_EXPS


def _all_patterns():
    return np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)


def test_tiny_normal_values_halve_exactly(oracle):
    y = _all_patterns()
    e = (y.astype(np.uint32) >> 7) & 0xFF
    sel = (e >= 2) & (e < TAB_EXP0)
    assert sel.sum() == 2 * (TAB_EXP0 - 2) * 128
    h = oracle.gelu_bf16(y[sel])
    assert np.array_equal(h, (y[sel].astype(np.uint32) - 0x80).astype(np.uint16))


def test_large_positive_values_pass_through(oracle):
    y = _all_patterns().astype(np.uint32)
    sel = (y >= TAB_END << 7) & (y < 0x7F80)  # 16 <= y <= the largest finite bf16
    assert sel.sum() == 0x7F80 - (TAB_END << 7)
    h = oracle.gelu_bf16(y[sel].astype(np.uint16))
    assert np.array_equal(h, y[sel].astype(np.uint16))


def test_large_negative_values_give_negative_zero(oracle):
    y = _all_patterns().astype(np.uint32)
    sel = (y >= 0x8000 | (TAB_END << 7)) & (y < 0xFF80)  # the largest finite bf16 <= y <= -16
    assert sel.sum() == 0x7F80 - (TAB_END << 7)
    h = oracle.gelu_bf16(y[sel].astype(np.uint16))
    assert np.all(h == 0x8000)


def test_the_rules_do_not_hold_past_their_ranges(oracle):
    """Just inside the table the closed forms would be wrong, which is why it starts and
    ends where it does."""
    # somewhere in 2^-10 <= |y| < 16 each shortcut gives a wrong h
    y = _all_patterns().astype(np.uint32)
    e = (y >> 7) & 0xFF
    inside = (e >= TAB_EXP0) & (e < TAB_END)
    h = oracle.gelu_bf16(y[inside].astype(np.uint16)).astype(np.uint32)
    assert np.any(h != y[inside] - 0x80)
    assert np.any(h != y[inside])
    # inside the table's negative half GELU(y) is not yet -0 (from about -14 on it is)
    y_neg = np.array([0xC100], np.uint16)  # -8
    assert oracle.gelu_bf16(y_neg)[0] != 0x8000
