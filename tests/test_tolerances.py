"""The fused norm's GPU tolerances follow from its arithmetic.

The kernel and the oracle take the norm's row factor r = 1/sqrt(ss/K + eps)
with the same IEEE fp64 steps from exact squares, and differ only in the
order in which ss is summed.  The GPU tests therefore allow one fp32 ulp on
the stored scales fl32(s * r) and one fp16 ulp on the FP16 outliers
fl16(z * r).  This test checks that claim on heavy-tailed rows: sequential,
pairwise and reversed fp64 sums give factors within a few fp64 ulps of the
exactly summed one, and the rounded scales and outliers agree to the stated
tolerance (almost always bit for bit).
"""
import math

import numpy as np


def _factor(ss, K, eps):
    return 1.0 / math.sqrt(ss / K + eps)


def _sums(sq):
    seq = 0.0
    for v in sq:
        seq += v
    rev = 0.0
    for v in sq[::-1]:
        rev += v
    return {"exact": math.fsum(sq), "sequential": seq, "reversed": rev,
            "pairwise": float(np.sum(sq))}


def test_summation_order_moves_scales_by_at_most_one_ulp():
    rng = np.random.default_rng(17)
    K, eps = 4096, np.float32(1e-5)
    differing_scales = differing_outliers = 0
    rows = 300
    for _ in range(rows):
        h = rng.standard_normal(K) * 2.0 ** rng.uniform(-2, 3)
        h[rng.integers(0, K, 128)] *= 30.0
        h = h.astype(np.float16).astype(np.float64)
        sq = [float(v) * float(v) for v in h]          # exact in fp64
        g = rng.uniform(0.5, 1.5, K).astype(np.float16).astype(np.float64)
        z = np.float32(h[:64] * g[:64])                 # exact in fp32
        s = np.float32(np.float32(np.abs(z).max()) / np.float32(7))
        sums = _sums(sq)
        r_ref = _factor(sums["exact"], K, float(eps))
        sx_ref = np.float32(float(s) * r_ref)
        o_ref = (z.astype(np.float64) * r_ref).astype(np.float16)
        for name, ss in sums.items():
            r = _factor(ss, K, float(eps))
            assert abs(r - r_ref) <= 8 * np.spacing(r_ref), name
            sx = np.float32(float(s) * r)
            assert abs(float(sx) - float(sx_ref)) <= float(np.spacing(sx_ref)), name
            differing_scales += int(sx != sx_ref)
            o = (z.astype(np.float64) * r).astype(np.float16)
            ulp = np.spacing(np.abs(o_ref).astype(np.float16)).astype(np.float64)
            assert np.all(np.abs(o.astype(np.float64) - o_ref.astype(np.float64)) <= ulp), name
            differing_outliers += int(np.count_nonzero(o != o_ref))
    # the tolerance is a margin, not the common case
    assert differing_scales <= rows // 50
    assert differing_outliers <= rows
