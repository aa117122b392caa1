"""The tile softmax's exponential on the FMA pipe (attn_tile.cu, exp2_fma_x2).

The kernel evaluates a quarter of its exponentials as 2^x = 2^n * p(f), with
n the nearest integer to x (rounded by adding 1.5 * 2^23), |f| <= 1/2 and p
a cubic fitted to 2^f.  This test takes the cubic's coefficients from the
kernel source, replays the same fp32 steps on the CPU (each FMA rounded once,
as the hardware does) and checks the result against 2^x in float64 over the
arguments the kernel meets (masked scores are -inf; visible ones are at most
8 above the reference maximum).  No GPU is needed.
"""
from __future__ import annotations

import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(__file__), "..", "block_sparse_gqa_indexer_b200", "csrc", "attn_tile.cu")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("exp2_fma_x2("):]
    m = re.search(r"c0 = ([0-9.eE+-]+)f, c1 = ([0-9.eE+-]+)f, c2 = ([0-9.eE+-]+)f, c3 = ([0-9.eE+-]+)f", body)
    assert m, "coefficients of exp2_fma_x2 not found"
    return [np.float32(float(v)) for v in m.groups()]


def _fma32(a, b, c):
    # a * b is exact in float64 for float32 operands; one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma(x: np.ndarray) -> np.ndarray:
    c0, c1, c2, c3 = _coefficients()
    rnd = np.float32(12582912.0)  # 1.5 * 2^23
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + rnd).astype(np.float32)
    n = (t - rnd).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    q = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    q = _fma32(q, f, np.full_like(f, c0))
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(
        0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_fraction_is_exact_and_bounded():
    x = np.linspace(-125.0, 8.0, 400_001).astype(np.float32)
    rnd = np.float32(12582912.0)
    n = ((x + rnd).astype(np.float32) - rnd).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    assert np.all(n == np.rint(x))  # nearest integer (ties to even)
    assert np.all(f.astype(np.float64) == x.astype(np.float64) - n.astype(np.float64))
    assert np.abs(f).max() <= 0.5


def test_relative_error_over_the_argument_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001), rng.uniform(-20.0, 8.0, 200_000),
                        np.arange(-125, 9, dtype=np.float64), np.arange(-125, 9) + 0.5]).astype(np.float32)
    got = exp2_fma(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    # the fit's bound (7.5e-5 in fp32) is far below the bf16 rounding of P (2^-9)
    assert rel.max() < 8e-5, rel.max()


def test_masked_and_zero_arguments():
    got = exp2_fma(np.array([-np.inf, -1e30, -125.0, 0.0, 1.0, 8.0], dtype=np.float32)).astype(np.float64)
    assert got[0] == got[1] == got[2] == pytest.approx(2.0 ** -125, rel=1e-4)  # masked: 2^-125, not 0
    assert got[3] == pytest.approx(1.0, rel=8e-5)
    assert got[4] == pytest.approx(2.0, rel=8e-5)
    assert got[5] == pytest.approx(256.0, rel=8e-5)


def test_a_wrong_coefficient_breaks_the_bound():
    # the bound is tight enough to notice a perturbed coefficient
    c0, c1, c2, c3 = _coefficients()
    f = np.linspace(-0.5, 0.5, 10_001)
    p = ((c3 * 1.01 * f + c2) * f + c1) * f + c0
    assert np.abs(p / np.exp2(f) - 1.0).max() > 8e-5
