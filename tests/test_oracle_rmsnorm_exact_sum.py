"""The fused norm's row factor comes from the exact sum of squares.

"Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", Summary
and idea I2 (the quantiser folded into the RMS norm), fixes no precision for
the norm.  The oracle's reading: sum the squares exactly, round the sum once
to fp64, then r = 1/sqrt(ss/K + eps) in IEEE fp64 steps, so that r does not
depend on the order of the additions.  These tests pin that reading against
an independent exact summation, Python's math.fsum (the correctly rounded
sum of the fp64 squares, each exact for an fp16 value):

* on rows built so that an fp64 sum in plain order (sequential, or reversed)
  rounds away the many small squares between two large ones, and with an
  eps dialled so that this changes the stored fp32 scale, the oracle gives
  the exactly summed scale bit for bit (an oracle that summed in fp64 in
  either order fails here);
* on rows spanning the whole fp16 range (subnormals to 65504) likewise, for
  the scales and the FP16 outliers;
* a row holding a non-finite value has no norm: the oracle refuses it.
"""
import math

import numpy as np
import pytest


def _factor(ss, K, eps):
    return 1.0 / math.sqrt(ss / K + eps)


def _base_scale(h, gamma, k_o):
    """fl32(max|z| / 7) over the INT4 part of z = h * gamma (exact in fp32)."""
    z = (h.astype(np.float64) * gamma.astype(np.float64)).astype(np.float32)
    return np.float32(np.abs(z[:h.size - k_o]).max()) / np.float32(7), z


def _expected(h, gamma, eps, k_o, ss):
    """Stored per-token scale and FP16 outliers of one row from a given sum of
    squares (identity permutation)."""
    s, z = _base_scale(h, gamma, k_o)
    r = _factor(ss, h.size, float(np.float32(eps)))
    return np.float32(float(s) * r), (z[h.size - k_o:].astype(np.float64) * r).astype(np.float16)


def _sequential_sums(sq):
    return [float(np.add.accumulate(sq)[-1]), float(np.add.accumulate(sq[::-1])[-1])]


def _f32_step(e32, k):
    """The fp32 value k ulps away from the positive fp32 e32."""
    return float((np.array([e32], np.float32).view(np.int32) + k).view(np.float32)[0])


def _dialled_row(rng, K):
    """Two values near 65504 at the ends of the row, every other square below
    half an ulp of their sum, and an fp32 eps for which the scale from the
    exactly summed squares differs from both sequential orders' scales."""
    f = 1.0 + rng.integers(0, 400, K) / 1024.0
    h = (2.0 ** -11 * f * rng.choice([-1.0, 1.0], K)).astype(np.float16)
    h[0], h[-1] = np.float16(65504.0), np.float16(-61440.0)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float16)
    sq = h.astype(np.float64) ** 2
    exact = math.fsum(sq)
    naive = _sequential_sums(sq)
    assert all(n != exact for n in naive)
    s = float(_base_scale(h, gamma, 0)[0])
    p = np.float32(s * _factor(exact, K, 0.125))
    for nb in (np.nextafter(p, np.float32(np.inf)), np.nextafter(p, np.float32(-np.inf))):
        mid = (float(p) + float(nb)) / 2.0  # an fp32 rounding boundary
        r_mid = mid / s
        e32 = np.float32(1.0 / (r_mid * r_mid) - exact / K)
        for k in range(-400, 401):
            e = _f32_step(e32, k)
            if not e > 0:
                continue
            want = _expected(h, gamma, e, 0, exact)[0]
            if all(_expected(h, gamma, e, 0, n)[0] != want for n in naive):
                return h, gamma, e
    raise AssertionError("no eps separates the exact and the sequential sums")


@pytest.mark.parametrize("seed", range(4))
def test_order_sensitive_rows_take_the_exact_sum(oracle_mod, seed):
    K = 4096
    h, gamma, eps = _dialled_row(np.random.default_rng(100 + seed), K)
    perm = np.arange(K, dtype=np.int32)
    _, scale, _, _ = oracle_mod.rmsnorm_quantize_rows(h[None], gamma, eps, perm, 0, 0, False)
    want = _expected(h, gamma, eps, 0, math.fsum(h.astype(np.float64) ** 2))[0]
    assert scale[0].view(np.uint32) == want.view(np.uint32)


def test_full_range_rows_take_the_exact_sum(oracle_mod):
    rng = np.random.default_rng(5)
    R, K, k_o, eps = 64, 2048, 64, 1e-6
    X = rng.standard_normal((R, K)) * 2.0 ** rng.uniform(-22, 15, (R, K))
    X = np.clip(X, -65504, 65504).astype(np.float16)
    X[0, :] = np.float16(2.0 ** -24)      # all subnormal: the smallest squares
    X[1, :] = np.float16(65504.0)         # all at the maximum: the largest sum
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float16)
    perm = np.arange(K, dtype=np.int32)
    _, scale, O, _ = oracle_mod.rmsnorm_quantize_rows(X, gamma, eps, perm, k_o, 0, False)
    for i, h in enumerate(X):
        s_ref, o_ref = _expected(h, gamma, eps, k_o, math.fsum(h.astype(np.float64) ** 2))
        assert scale[i].view(np.uint32) == s_ref.view(np.uint32), i
        np.testing.assert_array_equal(O[i].view(np.uint16), o_ref.view(np.uint16))


def test_non_finite_row_is_refused(oracle_mod):
    X = np.ones((2, 256), np.float16)
    X[1, 7] = np.float16(np.inf)
    with pytest.raises(Exception):
        oracle_mod.rmsnorm_quantize_rows(X, np.ones(256, np.float16), 1e-6,
                                         np.arange(256, dtype=np.int32), 32, 0, False)
