"""Pins of the oracle's RMS-norm-fused quantiser (``rmsnorm_quantize_rows``).

"Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", Summary
and idea I2: the dynamic quantisation and reordering are folded into the
operator that runs before the projection, which in Llama is the RMS norm
  y[k] = h[k] * gamma[k] / sqrt(mean_k(h[k]^2) + eps).

None of these tests re-types the oracle's arithmetic.  Each checks a fact
fixed by the definition of the norm and of the (separately pinned) unfused
quantiser:

* an exactly representable case, built so that mean(h^2) + eps = 64 and the
  row factor is exactly 1/8: the fused result must equal the unfused oracle
  applied to the normalised row, bit for bit (codes, scales, outliers);
* the norm's invariances (h -> 2^k h leaves everything unchanged when
  eps = 0; gamma -> 2^k gamma scales the scales and outliers by 2^k);
* a constant row, whose factor has a closed form;
* general inputs against numpy's fp64 norm: every code is a nearest code of
  y / scale and the scale is max|y| / 7 to fp32 rounding;
* the layer on lossless inputs equals numpy's fp64 product of the
  normalised activations and the weights.

A slip in the oracle (the sum taken over the INT4 channels only, a mean over
K_i instead of K, eps outside the root, gamma not reordered with the row, the
factor applied to the codes, a missing factor on the INT8 outlier scale)
breaks at least one of them.
"""
import numpy as np
import pytest


def exact_case(rng, R, K, lo_bits=False):
    """Rows h of integers in [-7, 7], gamma = k / 64 (k in +-[1, 255]), and eps
    with mean(h^2) + eps == 64 for every row, so r = 1/8 exactly and
    y = h * gamma / 8 is exact in fp16.  One eps serves all rows: every row
    gets the same sum of squares (a shuffled copy of one multiset)."""
    base = rng.integers(-7, 8, size=K)
    base[rng.integers(0, K)] = 7
    h = np.stack([rng.permutation(base) * rng.choice([-1, 1], size=K) for _ in range(R)])
    S = int((base.astype(np.int64) ** 2).sum())
    assert K & (K - 1) == 0, "K a power of two keeps S / K exact"
    eps = 64.0 - S / K
    assert eps >= 0 and np.float32(eps) == eps
    k = rng.integers(1, 256, size=K) * rng.choice([-1, 1], size=K)
    gamma = k / 64.0
    y = h * gamma / 8.0
    h16, g16, y16 = h.astype(np.float16), gamma.astype(np.float16), y.astype(np.float16)
    assert np.array_equal(h16.astype(np.float64), h)
    assert np.array_equal(g16.astype(np.float64), gamma)
    assert np.array_equal(y16.astype(np.float64), y), "normalised row not exact in fp16"
    return h16, g16, float(eps), y16


CASES = [  # K, k_o, group, int8 outliers, bits
    (256, 32, 0, False, 4),
    (256, 32, 0, True, 4),
    (256, 0, 0, False, 4),
    (256, 256, 0, False, 4),
    (256, 256, 0, True, 4),
    (512, 128, 128, False, 4),
    (512, 128, 128, True, 4),
    (256, 32, 0, False, 8),
    (256, 64, 0, True, 8),
]


@pytest.mark.parametrize("K,k_o,group,int8,bits", CASES)
def test_exact_case_equals_unfused(oracle_mod, K, k_o, group, int8, bits):
    rng = np.random.default_rng(11 + K + k_o + group + 2 * int8 + bits)
    h16, g16, eps, y16 = exact_case(rng, 6, K)
    perm = rng.permutation(K).astype(np.int32)
    fused = oracle_mod.rmsnorm_quantize_rows(h16, g16, eps, perm, k_o, group, int8, bits)
    unfused = oracle_mod.quantize_rows(y16, perm, k_o, group, int8, bits)
    names = ("codes", "scales", "outliers", "outlier scales")
    for name, a, b in zip(names, fused, unfused):
        if a is None and b is None:
            continue
        assert a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8)), name


def test_row_scaling_invariance(oracle_mod):
    rng = np.random.default_rng(3)
    K, k_o = 384, 32
    h = rng.standard_normal((5, K)).astype(np.float16)
    g = rng.uniform(0.2, 2.0, K).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    for int8 in (False, True):
        ref = oracle_mod.rmsnorm_quantize_rows(h, g, 0.0, perm, k_o, 0, int8)
        for e in (-3, 4):
            got = oracle_mod.rmsnorm_quantize_rows((h * 2.0 ** e).astype(np.float16), g, 0.0,
                                                  perm, k_o, 0, int8)
            for a, b in zip(ref, got):
                if a is not None:
                    assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_gamma_scaling_covariance(oracle_mod):
    rng = np.random.default_rng(4)
    K, k_o = 512, 128
    h = rng.standard_normal((4, K)).astype(np.float16)
    g = rng.uniform(0.5, 1.5, K).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    for group, int8 in ((0, False), (128, True)):
        q0, s0, o0, os0 = oracle_mod.rmsnorm_quantize_rows(h, g, 1e-5, perm, k_o, group, int8)
        q1, s1, o1, os1 = oracle_mod.rmsnorm_quantize_rows(h, (g * 4).astype(np.float16), 1e-5,
                                                          perm, k_o, group, int8)
        assert np.array_equal(q0, q1)
        assert np.array_equal(s1, s0 * np.float32(4))
        if int8:
            assert np.array_equal(o0, o1) and np.array_equal(os1, os0 * np.float32(4))
        else:
            assert np.array_equal(o1, (o0.astype(np.float32) * 4).astype(np.float16))


def test_constant_row_closed_form(oracle_mod):
    K, k_o = 128, 32
    perm = np.random.default_rng(5).permutation(K).astype(np.int32)
    for c, eps in ((0.75, 1e-6), (-3.0, 0.25), (2.0 ** -10, 1e-5)):
        h = np.full((1, K), c, np.float16)
        g = np.ones(K, np.float16)
        q, s, o, _ = oracle_mod.rmsnorm_quantize_rows(h, g, eps, perm, k_o)
        r = 1.0 / np.sqrt(float(c) ** 2 + float(np.float32(eps)))  # eps is an fp32 parameter
        code = 7 if c > 0 else -7
        nib = code & 0xF
        assert np.all(q == (nib | (nib << 4)))
        s_z = np.float32(abs(c)) / np.float32(7)
        assert s[0] == np.float32(float(s_z) * r)
        assert np.array_equal(o[0], np.full(k_o, c * r).astype(np.float16))


def decode(Q):
    lo = (Q & 0x0F).astype(np.int64)
    hi = (Q >> 4).astype(np.int64)
    out = np.empty((Q.shape[0], 2 * Q.shape[1]), np.int64)
    out[:, 0::2], out[:, 1::2] = lo, hi
    return np.where(out >= 8, out - 16, out)


@pytest.mark.parametrize("group,bits", [(0, 4), (128, 4), (0, 8)])
def test_general_inputs_against_numpy_norm(oracle_mod, group, bits):
    rng = np.random.default_rng(6 + group + bits)
    R, K, k_o = 8, 1024, 128
    Ki = K - k_o
    h = rng.standard_normal((R, K)) * rng.choice([1.0, 0.1, 20.0], size=(R, 1))
    h[:, rng.integers(0, K, 8)] *= 30.0
    h16 = h.astype(np.float16)
    g16 = rng.uniform(0.05, 3.0, K).astype(np.float16)
    eps = 1e-6
    perm = rng.permutation(K).astype(np.int32)
    q, s, o, _ = oracle_mod.rmsnorm_quantize_rows(h16, g16, eps, perm, k_o, group, False, bits)
    hd = h16.astype(np.float64)
    y = hd / np.sqrt((hd ** 2).mean(axis=1, keepdims=True) + eps) * g16.astype(np.float64)
    y = y[:, perm]
    codes = q.astype(np.int64) if bits == 8 else decode(q)
    qmax = 127 if bits == 8 else 7
    gs = group or Ki
    sx = np.repeat(s.reshape(R, -1).astype(np.float64), gs, axis=1)
    amax = np.abs(y[:, :Ki]).reshape(R, -1, gs).max(axis=2)
    assert np.allclose(s.reshape(R, -1), amax / qmax, rtol=3e-7, atol=0)
    # each code is a nearest integer of y / scale (slack for the fp32 roundings)
    assert np.all(np.abs(y[:, :Ki] / sx - codes) <= 0.5 + 1e-5)
    assert np.abs(codes).max() == qmax
    # FP16 outliers: the normalised values, rounded once to fp16
    ref = y[:, Ki:]
    assert np.all(np.abs(o.astype(np.float64) - ref) <= np.abs(ref) * 2.0 ** -11 * (1 + 1e-6) + 2.0 ** -25)


def lossless_block_rows(rng, R, perm, Ki, int8):
    """Rows of integers laid out through perm: the INT4 positions hold codes
    in [-7, 7] with a +-7, the outlier positions codes in [-127, 127] with a
    +-127 (INT8 outliers; the INT8 rule is then lossless too) or in [-7, 7]
    (FP16 outliers).  Every row is a signed shuffle of one base row inside
    each block, so all rows share one sum of squares."""
    K = len(perm)
    omax = 127 if int8 else 7
    b4 = rng.integers(-7, 8, size=Ki)
    b4[rng.integers(0, Ki)] = 7
    bo = rng.integers(-omax, omax + 1, size=K - Ki)
    if K > Ki:
        bo[rng.integers(0, K - Ki)] = omax
    rows = np.zeros((R, K))
    for r in range(R):
        rows[r, perm[:Ki]] = rng.permutation(b4) * rng.choice([-1, 1], size=Ki)
        rows[r, perm[Ki:]] = rng.permutation(bo) * rng.choice([-1, 1], size=K - Ki)
    return rows, int((b4 ** 2).sum() + (bo ** 2).sum())


@pytest.mark.parametrize("int8", [False, True])
def test_layer_lossless_equals_fp64_matmul(oracle_mod, int8):
    """h of integer codes (lossless per block), gamma = 2^-3 everywhere, and
    eps with mean(h^2) + eps = 4^b: the normalised row is h * 2^-(3+b),
    quantised without loss; with lossless weights the output equals numpy's
    fp64 product of the normalised row and W (plus bias)."""
    rng = np.random.default_rng(7 + int8)
    M, N, K, k_o = 6, 40, 256, 32
    Ki = K - k_o
    perm = rng.permutation(K).astype(np.int32)
    h, S = lossless_block_rows(rng, M, perm, Ki, int8)
    b = 0
    while 4.0 ** b < S / K:
        b += 1
    eps = 4.0 ** b - S / K
    assert np.float32(eps) == eps
    gamma = np.full(K, 2.0 ** -3)
    y = h * gamma * 2.0 ** -b
    Wc, _ = lossless_block_rows(rng, N, perm, Ki, int8)
    W = Wc * (2.0 ** rng.integers(-12, -6, size=(N, 1)))
    bias = rng.integers(-8, 8, size=N) * 2.0 ** -6
    for a in (h, y, W, bias):
        assert np.array_equal(a.astype(np.float16).astype(np.float64), a)
    out = oracle_mod.rmsnorm_layer(h.astype(np.float16), gamma.astype(np.float16), eps,
                                   W.astype(np.float16), perm, bias.astype(np.float16), k_o,
                                   0, int8)
    assert np.array_equal(out["Y"], y @ W.T + bias)
