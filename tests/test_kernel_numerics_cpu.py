"""Numerical claims of the prefill attention kernel, checked on the CPU.

Six of every sixteen key pairs of attn_tc.cu's softmax take 2^x from a cubic on
the FMA pipe instead of the transcendental unit.  These tests read that
function's constants from the kernel source and evaluate its steps in fp32 (an
emulation of the device arithmetic: fp32 adds, fused multiply-adds, and the
integer add of round(x) into the exponent field), then check what the kernel's
comments state: the rounding step gives round(x), the relative error stays
within 7.5e-5 over the arguments the kernel can see, masked keys underflow to
about 2^-126, and the polynomial pairs are spread evenly over a 32-key store.
"""
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "routed_sparse_attention_chunk_b200", "csrc", "attn_tc.cu")


def _kernel_constants():
    src = open(SRC).read()
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    magic = float(re.search(r"kMagic = ([0-9.]+)f", body).group(1))
    # the cubic's coefficients, highest degree first, as the fma chain uses them
    coef = [float(c) for c in re.findall(r"f2_pack\(([-+0-9.eE]+)f, \1f\)", body) if float(c) != -1.0]
    assert len(coef) == 4, coef
    polys = int(re.search(r"constexpr int kPolyPairs = (\d+);", src).group(1))
    return np.float32(magic), [np.float32(c) for c in coef], polys


def _fma32(a, b, c):
    # a * b is exact in fp64 for fp32 operands; one fp64 add, then the fp32 rounding
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(np.float32)


def _poly_exp2(x):
    """The kernel's exp2_poly2 on fp32 arguments; returns (2^x, round(x) as a float)."""
    magic, (c3, c2, c1, c0), _ = _kernel_constants()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    t = (x + magic).astype(np.float32)  # round(x) in the low mantissa bits
    jf = (t - magic).astype(np.float32)  # round(x) as a float
    f = _fma32(jf, -1.0, x)              # x - round(x)
    q = _fma32(f, c3, c2)
    q = _fma32(q, f, c1)
    q = _fma32(q, f, c0)
    bits = (q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32), jf


def test_rounding_step_is_round_to_nearest_even():
    x = np.concatenate([np.linspace(-126, 8, 200_001), np.arange(-126, 9) + 0.5]).astype(np.float32)
    _, jf = _poly_exp2(x)
    np.testing.assert_array_equal(jf, np.rint(x))


def test_relative_error_within_the_stated_bound():
    # softmax arguments are x = s * scale * log2(e) - m_run <= 8 (the running max moves once it is
    # exceeded by 2^8); below -125 the result leaves the normal range and is covered by the next test
    x = np.linspace(-125, 8, 2_000_001).astype(np.float32)
    e, _ = _poly_exp2(x)
    rel = np.abs(e.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.5e-5
    # and the error is that of a fitted cubic, not of the fp32 evaluation: it is not far below the bound
    assert rel.max() > 5e-5


def test_masked_and_far_below_max_keys_underflow():
    x = np.array([-np.inf, -1e30, -300.0, -126.0], dtype=np.float32)
    e, _ = _poly_exp2(x)
    assert np.all(e >= 0) and np.all(e <= np.float32(2.0 ** -125))


def test_polynomial_pairs_spread_evenly():
    _, _, polys = _kernel_constants()
    # the kernel's rule: pair i of 16 is a polynomial pair when i * n / 16 steps to the next integer
    pick = [(i * polys) // 16 != ((i + 1) * polys) // 16 for i in range(16)]
    assert sum(pick) == polys
    idx = [i for i, p in enumerate(pick) if p]
    gaps = np.diff(idx + [idx[0] + 16])
    assert gaps.max() - gaps.min() <= 1  # evenly spread, cyclically over consecutive stores


@pytest.mark.parametrize("x", [0.0, 1.0, -1.0, 0.5, -0.5, 7.0, -100.25])
def test_a_few_points_against_exp2(x):
    e, _ = _poly_exp2(np.array([x], dtype=np.float32))
    assert e[0] == pytest.approx(2.0 ** x, rel=7.5e-5)
