"""Host check of the FMA-pipe 2^x used for a share of the softmax exponentials
(ex2_fma2 in the attention kernel): the cubic's coefficients, read from the
source, and the float32 steps of the function emulated here, stay within the
stated relative error of 2^x over the range where the softmax keeps its
results (x = s * scale * log2 e - m <= 8, m the max in use), give 2^8 (within
the fit's error) above it, far above the 2^7 at which the softmax's sum test
recomputes the max,
and give 0 below -125 and for a masked score (-inf)."""
import os
import re

import numpy as np

from tests.conftest import ROOT

SRC = os.path.join(ROOT, "spacetime_attention_vdit_b200", "csrc", "attn_tcgen05.cuh")


def coefficients():
    with open(SRC) as fh:
        text = fh.read()
    body = text[text.index("float2 ex2_fma2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    c3 = float(re.search(r"make_float2\(([0-9.e+-]+)f, \1f\), f, make_float2\(([0-9.e+-]+)f", body).group(1))
    c2 = float(re.search(r"make_float2\(([0-9.e+-]+)f, \1f\), f, make_float2\(([0-9.e+-]+)f", body).group(2))
    rest = re.findall(r"q = ffma2\(q, f, make_float2\(([0-9.e+-]+)f", body)
    return np.float32(c3), np.float32(c2), np.float32(rest[0]), np.float32(rest[1])


def ex2_fma_emulated(x):
    """The kernel's steps in float32 (fma rounded once, as the hardware does)."""
    c3, c2, c1, c0 = coefficients()
    x = np.asarray(x, dtype=np.float32)
    xc = np.minimum(np.maximum(x, np.float32(-125.0)), np.float32(8.0))
    rnd = np.float32(12582912.0)
    t = (xc + rnd).astype(np.float32)
    f = (xc.astype(np.float64) + (rnd.astype(np.float64) - t.astype(np.float64))).astype(np.float32)

    def fma(a, b, c):
        return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)

    q = fma(np.full_like(f, c3), f, np.full_like(f, c2))
    q = fma(q, f, np.full_like(f, c1))
    q = fma(q, f, np.full_like(f, c0))
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    out = bits.astype(np.uint32).view(np.float32)
    return np.where(x < -125.0, np.float32(0.0), out)


def test_cubic_fits_2_to_the_f():
    c3, c2, c1, c0 = (float(c) for c in coefficients())
    f = np.linspace(-0.5, 0.5, 200001)
    rel = (((c3 * f + c2) * f + c1) * f + c0) / np.exp2(f) - 1.0
    assert np.abs(rel).max() < 8e-5          # below half a bf16 ulp (2^-9) by a wide margin


def test_emulated_function_matches_exp2_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), -np.arange(0, 126, dtype=np.float64),
                        np.arange(0, 9, dtype=np.float64), [-0.5, 0.5, -124.5, 7.5]]).astype(np.float32)
    got = ex2_fma_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert np.abs(got / ref - 1.0).max() < 1.2e-4


def test_below_range_and_masked_scores_give_zero():
    x = np.array([-125.001, -126.0, -300.0, -1e30, -np.inf], dtype=np.float32)
    assert np.all(ex2_fma_emulated(x) == 0.0)


def test_above_eight_saturates_at_two_to_the_eight():
    """A score above the max in use by more than 8 (log2 units) comes out as 2^8
    (within the fit's error), so the tile's sum of P reaches the softmax's 2^7
    test and the max is recomputed: such a value is never kept."""
    x = np.array([8.0, 8.0001, 9.0, 20.0, 127.0, 1e30, np.inf], dtype=np.float32)
    got = ex2_fma_emulated(x).astype(np.float64)
    assert np.abs(got[0] / 256.0 - 1.0) < 1.2e-4
    assert np.all(got[1:] == got[0]) and got[0] > 2.0 * 128.0 * (1.0 - 1e-3)

