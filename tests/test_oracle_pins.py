"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests re-types the oracle's formulas: each checks a property
that a plausible slip in the oracle (a dropped term, a wrong divisor, sign,
index, nibble order, a transposed operand, an outlier channel counted in the
INT4 scale, round-half-away instead of half-even) would break:

* hand-derived byte layout and tie-rounding fixtures (tests/golden);
* brute-force nearest-code search instead of rint;
* lossless inputs (values = code * 2^e) whose output must equal the fp64
  matrix product computed by numpy;
* the degenerate cases k_o = 0, k_o = K and one group per row;
* invariances (joint channel permutation, power-of-two scaling, negation);
* the integer sums against numpy's int64 matrix product of decoded codes.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers
def decode(Q: np.ndarray) -> np.ndarray:
    """Test-side nibble decoder: [R, B] bytes -> [R, 2B] signed codes."""
    lo = (Q & 0x0F).astype(np.int64)
    hi = (Q >> 4).astype(np.int64)
    out = np.empty((Q.shape[0], 2 * Q.shape[1]), np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return np.where(out >= 8, out - 16, out)


def lossless_rows(rng, R, n, group=0, exp_lo=-6, exp_hi=3):
    """Rows of values code * 2^e with a +-7 in every row (or group)."""
    codes = rng.integers(-7, 8, size=(R, n))
    gs = group if group else n
    scales = np.zeros((R, n // gs if n else 1))
    for r in range(R):
        for g in range(n // gs if n else 0):
            codes[r, g * gs + rng.integers(0, gs)] = rng.choice([-7, 7])
            scales[r, g] = 2.0 ** rng.integers(exp_lo, exp_hi)
    vals = codes * (np.repeat(scales, gs, axis=1) if n else 0)
    return codes, scales, vals


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, vals = line.split(":", 1)
                rows.append((key.strip(), vals.split()))
    return rows


def nearest_code(v: np.float32, s: np.float32, qmax: int) -> int:
    """Exhaustive search: the code whose value is nearest to fl32(v / s), ties to even."""
    if s == 0:
        return 0
    t = float(np.float32(v) / np.float32(s))
    best, bestd = None, None
    for q in range(-qmax, qmax + 1):
        d = abs(t - q)
        if best is None or d < bestd or (d == bestd and q % 2 == 0):
            best, bestd = q, d
    return best


# ----------------------------------------------------------------- golden fixtures
def test_pack_layout_golden(oracle_mod):
    g = dict(read_golden("pack_layout.txt"))
    codes = np.array([int(c) for c in g["codes"]])
    expect = np.array([int(b, 16) for b in g["bytes"]], np.uint8)
    X = codes.astype(np.float16)[None, :]
    perm = np.arange(len(codes), dtype=np.int32)
    Q, s, _, _ = oracle_mod.quantize_rows(X, perm, 0)
    assert s[0] == np.float32(1.0)
    np.testing.assert_array_equal(Q[0], expect)


def test_ties_golden(oracle_mod):
    rows = read_golden("ties.txt")
    for (kx, xs), (kq, qs) in zip(rows[0::2], rows[1::2]):
        x = np.array([float(v) for v in xs], np.float16)[None, :]
        q = np.array([int(v) for v in qs])
        n = x.shape[1]
        if kx.startswith("int4"):
            Q, _, _, _ = oracle_mod.quantize_rows(x, np.arange(n, dtype=np.int32), 0)
            np.testing.assert_array_equal(decode(Q)[0], q)
        else:
            # the whole row is the INT8 outlier block (k_o = K)
            _, _, O, so = oracle_mod.quantize_rows(x, np.arange(n, dtype=np.int32), n,
                                                   outlier_int8=True)
            assert so[0] == np.float32(1.0)
            np.testing.assert_array_equal(O[0].astype(np.int64), q)


# ----------------------------------------------------------------- rounding / scale
@pytest.mark.parametrize("group", [0, 32])
def test_codes_are_nearest_brute_force(oracle_mod, group):
    rng = np.random.default_rng(11)
    R, K = 5, 64
    X = (rng.standard_normal((R, K)) * rng.uniform(0.01, 10, size=(R, 1))).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    Q, s, _, _ = oracle_mod.quantize_rows(X, perm, 0, group)
    codes = decode(Q)
    Xr = X[:, perm].astype(np.float32)
    gs = group or K
    s = s.reshape(R, -1)
    for r in range(R):
        for j in range(K):
            sc = s[r, j // gs]
            assert codes[r, j] == nearest_code(Xr[r, j], sc, 7), (r, j)
        for g in range(K // gs):
            amax = np.abs(Xr[r, g * gs:(g + 1) * gs]).max()
            # divisor 7: 7 * s reproduces the absmax to within one fp32 rounding
            assert abs(np.float64(s[r, g]) * 7 - amax) <= np.spacing(np.float32(amax))


def test_int8_outlier_codes_are_nearest_brute_force(oracle_mod):
    rng = np.random.default_rng(12)
    R, K, k_o = 4, 48, 16
    X = (rng.standard_normal((R, K)) * 3).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    _, _, O, so = oracle_mod.quantize_rows(X, perm, k_o, outlier_int8=True)
    Xo = X[:, perm[K - k_o:]].astype(np.float32)
    for r in range(R):
        amax = np.abs(Xo[r]).max()
        assert abs(np.float64(so[r]) * 127 - amax) <= np.spacing(np.float32(amax))
        for i in range(k_o):
            assert int(O[r, i]) == nearest_code(Xo[r, i], so[r], 127)


def test_zero_row(oracle_mod):
    X = np.zeros((2, 32), np.float16)
    X[1, 5] = 3.0
    perm = np.arange(32, dtype=np.int32)
    Q, s, _, _ = oracle_mod.quantize_rows(X, perm, 0)
    assert s[0] == 0.0 and not np.isnan(s).any()
    assert (Q[0] == 0).all()
    Qg, sg, _, _ = oracle_mod.quantize_rows(X, perm, 0, group=16)
    assert sg[0, 0] == 0 and sg[0, 1] == 0 and sg[1, 1] == 0
    assert (decode(Qg)[1, 16:] == 0).all() and decode(Qg)[1, 5] == 7


# ----------------------------------------------------------------- lossless special cases
def _fp64_ref(X, W, bias):
    Y = X.astype(np.float64) @ W.astype(np.float64).T
    return Y if bias is None else Y + bias.astype(np.float64)[None, :]


@pytest.mark.parametrize("M,N,K,k_o,group,int8", [
    (7, 5, 64, 16, 0, False),
    (6, 9, 96, 32, 0, False),
    (5, 4, 288, 32, 128, False),
    (4, 6, 160, 32, 0, True),
    (3, 7, 272, 16, 128, True),
])
def test_lossless_equals_fp64_matmul(oracle_mod, M, N, K, k_o, group, int8):
    rng = np.random.default_rng(M * 100 + K)
    Ki = K - k_o
    perm = rng.permutation(K).astype(np.int32)
    cx, sx_true, vx = lossless_rows(rng, M, Ki, group)
    cw, sw_true, vw = lossless_rows(rng, N, Ki, group)
    X = np.zeros((M, K), np.float64)
    W = np.zeros((N, K), np.float64)
    X[:, perm[:Ki]] = vx
    W[:, perm[:Ki]] = vw
    if int8:
        ox, sxo, vxo = lossless_rows(rng, M, k_o, 0)
        ox = np.clip(ox * 18, -127, 127)
        ox[:, 0] = 127
        vxo = ox * sxo
        ow, swo, vwo = lossless_rows(rng, N, k_o, 0)
        ow = np.clip(ow * 18, -127, 127)
        ow[:, 1] = -127
        vwo = ow * swo
    else:
        # arbitrary fp16 values, larger than the INT4 part (outliers)
        vxo = rng.standard_normal((M, k_o)) * 40
        vwo = rng.standard_normal((N, k_o)) * 0.05
    X[:, perm[Ki:]] = vxo
    W[:, perm[Ki:]] = vwo
    X16, W16 = X.astype(np.float16), W.astype(np.float16)
    assert (X16.astype(np.float64)[:, perm[:Ki]] == vx).all()
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)

    r = oracle_mod.layer(X16, W16, perm, bias, k_o, group, int8)
    # codes and scales recovered exactly, outlier channels excluded from the scale
    np.testing.assert_array_equal(decode(r["Xq"]), cx)
    np.testing.assert_array_equal(decode(r["Wq"]), cw)
    np.testing.assert_array_equal(r["sx"].reshape(M, -1), sx_true.astype(np.float32))
    np.testing.assert_array_equal(r["sw"].reshape(N, -1), sw_true.astype(np.float32))
    if int8:
        np.testing.assert_array_equal(r["Xo"].astype(np.int64), ox)
        np.testing.assert_array_equal(r["sxo"], sxo[:, 0].astype(np.float32))
    else:
        np.testing.assert_array_equal(r["Xo"], X16[:, perm[Ki:]])
        np.testing.assert_array_equal(r["Wo"], W16[:, perm[Ki:]])
    ref = _fp64_ref(X16, W16, bias)
    np.testing.assert_allclose(r["Y"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_k_o_zero_is_pure_w4a4(oracle_mod):
    rng = np.random.default_rng(3)
    M, N, K = 6, 5, 64
    perm = rng.permutation(K).astype(np.int32)
    _, _, vx = lossless_rows(rng, M, K)
    _, _, vw = lossless_rows(rng, N, K)
    X = np.zeros((M, K)); W = np.zeros((N, K))
    X[:, perm] = vx; W[:, perm] = vw
    X16, W16 = X.astype(np.float16), W.astype(np.float16)
    r = oracle_mod.layer(X16, W16, perm, None, 0)
    assert r["Xo"].shape == (M, 0)
    np.testing.assert_allclose(r["Y"], _fp64_ref(X16, W16, None), rtol=1e-12, atol=1e-12)
    # with general (lossy) inputs the output is exactly the dequantised integer sums
    Xg = rng.standard_normal((M, K)).astype(np.float16)
    Wg = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    r = oracle_mod.layer(Xg, Wg, perm, None, 0)
    A = decode(r["Xq"]) @ decode(r["Wq"]).T
    np.testing.assert_allclose(r["Y"], A * r["sx"][:, None].astype(np.float64)
                               * r["sw"][None, :].astype(np.float64), rtol=1e-15, atol=0)


@pytest.mark.parametrize("int8", [False, True])
def test_k_o_equals_K(oracle_mod, int8):
    rng = np.random.default_rng(4)
    M, N, K = 5, 7, 48
    X16 = rng.standard_normal((M, K)).astype(np.float16)
    W16 = (rng.standard_normal((N, K)) * 0.1).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)
    r = oracle_mod.layer(X16, W16, perm, bias, K, 0, int8)
    assert r["Xq"].shape == (M, 0)
    if not int8:
        # the whole layer is an FP16 GEMM: exact products summed in fp64
        ref = _fp64_ref(X16, W16, bias)
        np.testing.assert_allclose(r["Y"], ref, rtol=1e-12, atol=1e-13)
    else:
        A8 = r["Xo"].astype(np.int64) @ r["Wo"].astype(np.int64).T
        ref = A8 * r["sxo"][:, None].astype(np.float64) * r["swo"][None, :].astype(np.float64)
        np.testing.assert_allclose(r["Y"], ref + bias.astype(np.float64), rtol=1e-14, atol=1e-14)


def test_single_group_equals_per_token(oracle_mod):
    rng = np.random.default_rng(5)
    M, N, K, k_o = 6, 4, 160, 32
    X16 = rng.standard_normal((M, K)).astype(np.float16)
    W16 = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    a = oracle_mod.layer(X16, W16, perm, None, k_o, 0)
    b = oracle_mod.layer(X16, W16, perm, None, k_o, 128)
    np.testing.assert_array_equal(a["Xq"], b["Xq"])
    np.testing.assert_array_equal(a["sx"], b["sx"][:, 0])
    np.testing.assert_array_equal(a["Y"], b["Y"])


# ----------------------------------------------------------------- invariances
def test_joint_channel_permutation(oracle_mod):
    rng = np.random.default_rng(6)
    M, N, K, k_o = 5, 6, 96, 32
    Ki = K - k_o
    X16 = rng.standard_normal((M, K)).astype(np.float16)
    W16 = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    base = oracle_mod.layer(X16, W16, perm, None, k_o)
    # (1) move the physical channels of X and W together and relabel perm
    sigma = rng.permutation(K)
    Xs, Ws = np.empty_like(X16), np.empty_like(W16)
    Xs[:, sigma] = X16
    Ws[:, sigma] = W16
    moved = oracle_mod.layer(Xs, Ws, sigma[perm].astype(np.int32), None, k_o)
    for k in ("Xq", "sx", "Wq", "sw", "Xo", "Wo", "Y"):
        np.testing.assert_array_equal(base[k], moved[k])
    # (2) shuffle the order inside the INT4 block and inside the outlier block
    tau = np.concatenate([rng.permutation(Ki), Ki + rng.permutation(k_o)])
    shuf = oracle_mod.layer(X16, W16, perm[tau].astype(np.int32), None, k_o)
    np.testing.assert_array_equal(base["sx"], shuf["sx"])
    np.testing.assert_array_equal(np.sort(decode(base["Xq"]), 1), np.sort(decode(shuf["Xq"]), 1))
    np.testing.assert_array_equal(oracle_mod.int_gemm(base["Xq"], base["Wq"]),
                                  oracle_mod.int_gemm(shuf["Xq"], shuf["Wq"]))
    np.testing.assert_allclose(base["Y"], shuf["Y"], rtol=1e-12, atol=1e-12)


def test_power_of_two_scale_covariance(oracle_mod):
    rng = np.random.default_rng(7)
    M, K, k_o = 6, 64, 16
    X16 = rng.standard_normal((M, K)).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    Q, s, _, _ = oracle_mod.quantize_rows(X16, perm, k_o)
    for k in (-3, 2):
        Q2, s2, _, _ = oracle_mod.quantize_rows((X16.astype(np.float32) * 2.0 ** k).astype(np.float16),
                                                perm, k_o)
        np.testing.assert_array_equal(Q, Q2)
        np.testing.assert_array_equal(s2, s * np.float32(2.0 ** k))


def test_sign_symmetry(oracle_mod):
    rng = np.random.default_rng(8)
    M, N, K = 5, 4, 64
    X16 = rng.standard_normal((M, K)).astype(np.float16)
    W16 = rng.standard_normal((N, K)).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    a = oracle_mod.quantize_rows(X16, perm, 0)
    b = oracle_mod.quantize_rows(-X16, perm, 0)
    np.testing.assert_array_equal(decode(a[0]), -decode(b[0]))
    np.testing.assert_array_equal(a[1], b[1])
    Wq = oracle_mod.quantize_rows(W16, perm, 0)[0]
    np.testing.assert_array_equal(oracle_mod.int_gemm(a[0], Wq), -oracle_mod.int_gemm(b[0], Wq))


# ----------------------------------------------------------------- integer sums
@pytest.mark.parametrize("group", [0, 128])
def test_int_gemm_equals_int64_matmul(oracle_mod, group):
    rng = np.random.default_rng(9)
    M, N, Ki = 9, 7, 256
    Xq = rng.integers(0, 256, size=(M, Ki // 2), dtype=np.uint8)
    Wq = rng.integers(0, 256, size=(N, Ki // 2), dtype=np.uint8)
    acc = oracle_mod.int_gemm(Xq, Wq, group)
    cx, cw = decode(Xq), decode(Wq)
    if group == 0:
        np.testing.assert_array_equal(acc, cx @ cw.T)
    else:
        for g in range(Ki // group):
            sl = slice(g * group, (g + 1) * group)
            np.testing.assert_array_equal(acc[g], cx[:, sl] @ cw[:, sl].T)


def test_sampled_agrees_with_full(oracle_mod):
    rng = np.random.default_rng(10)
    M, N, K, k_o, group = 7, 9, 288, 32, 128
    X16 = rng.standard_normal((M, K)).astype(np.float16)
    W16 = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)
    r = oracle_mod.layer(X16, W16, perm, bias, k_o, group, True)
    ms = rng.integers(0, M, 20)
    ns = rng.integers(0, N, 20)
    Y, acc = oracle_mod.linear_sampled(r["Xq"], r["sx"], r["Xo"], r["sxo"], r["Wq"], r["sw"],
                                       r["Wo"], r["swo"], bias, K, k_o, group, ms, ns)
    np.testing.assert_array_equal(Y, r["Y"][ms, ns])
    full = oracle_mod.int_gemm(r["Xq"], r["Wq"], group)
    np.testing.assert_array_equal(acc, full[:, ms, ns].T)


# ----------------------------------------------------------------- 8-bit activations (W4A8)
# The W4A8 reading: the INT8 rule of the outlier block (divisor and clamp 127)
# applied per token to the non-outlier positions, one signed byte per code.
def lossless_rows8(rng, R, n, exp_lo=-6, exp_hi=3):
    """Rows of values code * 2^e, codes in [-127, 127] with a +-127 in every row."""
    codes = rng.integers(-127, 128, size=(R, n))
    scales = np.zeros((R, 1))
    for r in range(R):
        codes[r, rng.integers(0, n)] = rng.choice([-127, 127])
        scales[r, 0] = 2.0 ** rng.integers(exp_lo, exp_hi)
    return codes, scales, codes * scales


def test_a8_codes_are_nearest_brute_force(oracle_mod):
    rng = np.random.default_rng(21)
    R, K, k_o = 5, 80, 16
    X = (rng.standard_normal((R, K)) * rng.uniform(0.01, 10, size=(R, 1))).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    Q, s, _, _ = oracle_mod.quantize_rows(X, perm, k_o, 0, False, bits=8)
    assert Q.dtype == np.int8 and Q.shape == (R, K - k_o)
    Xr = X[:, perm[:K - k_o]].astype(np.float32)
    for r in range(R):
        amax = np.abs(Xr[r]).max()
        # divisor 127 over the non-outlier positions only
        assert abs(np.float64(s[r]) * 127 - amax) <= np.spacing(np.float32(amax))
        for j in range(K - k_o):
            assert int(Q[r, j]) == nearest_code(Xr[r, j], s[r], 127), (r, j)


def test_a8_zero_row(oracle_mod):
    X = np.zeros((2, 48), np.float16)
    X[1, 7] = -2.0
    Q, s, _, _ = oracle_mod.quantize_rows(X, np.arange(48, dtype=np.int32), 16, 0, False, bits=8)
    assert s[0] == 0.0 and (Q[0] == 0).all()
    assert Q[1, 7] == -127 and np.count_nonzero(Q[1]) == 1


@pytest.mark.parametrize("M,N,K,k_o,int8", [
    (6, 5, 96, 32, False),
    (4, 7, 160, 32, True),
    (5, 3, 64, 0, False),
])
def test_a8_lossless_equals_fp64_matmul(oracle_mod, M, N, K, k_o, int8):
    rng = np.random.default_rng(M * 31 + K)
    Ki = K - k_o
    perm = rng.permutation(K).astype(np.int32)
    cx, sx_true, vx = lossless_rows8(rng, M, Ki)
    cw, sw_true, vw = lossless_rows(rng, N, Ki)
    X = np.zeros((M, K)); W = np.zeros((N, K))
    X[:, perm[:Ki]] = vx
    W[:, perm[:Ki]] = vw
    if int8:
        ox, sxo, vxo = lossless_rows8(rng, M, k_o)
        ow, swo, vwo = lossless_rows8(rng, N, k_o)
    else:
        vxo = rng.standard_normal((M, k_o)) * 40
        vwo = rng.standard_normal((N, k_o)) * 0.05
    X[:, perm[Ki:]] = vxo
    W[:, perm[Ki:]] = vwo
    X16, W16 = X.astype(np.float16), W.astype(np.float16)
    assert (X16.astype(np.float64)[:, perm[:Ki]] == vx).all()
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)
    r = oracle_mod.layer(X16, W16, perm, bias, k_o, 0, int8, act_bits=8)
    np.testing.assert_array_equal(r["Xq"].astype(np.int64), cx)
    np.testing.assert_array_equal(decode(r["Wq"]), cw)
    np.testing.assert_array_equal(r["sx"], sx_true[:, 0].astype(np.float32))
    ref = _fp64_ref(X16, W16, bias)
    np.testing.assert_allclose(r["Y"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_a8_int_gemm_equals_int64_matmul(oracle_mod):
    rng = np.random.default_rng(22)
    M, N, Ki = 8, 6, 192
    Xq = rng.integers(-127, 128, size=(M, Ki)).astype(np.int8)
    Wq = rng.integers(0, 256, size=(N, Ki // 2), dtype=np.uint8)
    acc = oracle_mod.int_gemm(Xq, Wq, 0)
    np.testing.assert_array_equal(acc, Xq.astype(np.int64) @ decode(Wq).T)
    # the sampled path reads the same codes
    sx = rng.uniform(0.1, 1, M).astype(np.float32)
    sw = rng.uniform(0.1, 1, N).astype(np.float32)
    ms, ns = rng.integers(0, M, 10), rng.integers(0, N, 10)
    Y, a = oracle_mod.linear_sampled(Xq, sx, None, None, Wq, sw, None, None, None, Ki, 0, 0, ms, ns)
    np.testing.assert_array_equal(a[:, 0], acc[ms, ns])
    np.testing.assert_allclose(Y, acc[ms, ns] * sx[ms].astype(np.float64) * sw[ns].astype(np.float64),
                               rtol=1e-15, atol=0)


# ----------------------------------------------------------------- 8-bit weights too (W8A8)
@pytest.mark.parametrize("M,N,K,k_o,int8", [
    (5, 6, 96, 32, False),
    (4, 5, 160, 32, True),
])
def test_w8a8_lossless_equals_fp64_matmul(oracle_mod, M, N, K, k_o, int8):
    rng = np.random.default_rng(M * 57 + K)
    Ki = K - k_o
    perm = rng.permutation(K).astype(np.int32)
    cx, sx_true, vx = lossless_rows8(rng, M, Ki)
    cw, sw_true, vw = lossless_rows8(rng, N, Ki)
    X = np.zeros((M, K)); W = np.zeros((N, K))
    X[:, perm[:Ki]] = vx
    W[:, perm[:Ki]] = vw
    if int8:
        _, _, vxo = lossless_rows8(rng, M, k_o)
        _, _, vwo = lossless_rows8(rng, N, k_o)
    else:
        vxo = rng.standard_normal((M, k_o)) * 40
        vwo = rng.standard_normal((N, k_o)) * 0.05
    X[:, perm[Ki:]] = vxo
    W[:, perm[Ki:]] = vwo
    X16, W16 = X.astype(np.float16), W.astype(np.float16)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)
    r = oracle_mod.layer(X16, W16, perm, bias, k_o, 0, int8, act_bits=8, weight_bits=8)
    np.testing.assert_array_equal(r["Xq"].astype(np.int64), cx)
    np.testing.assert_array_equal(r["Wq"].astype(np.int64), cw)
    np.testing.assert_array_equal(r["sw"], sw_true[:, 0].astype(np.float32))
    ref = _fp64_ref(X16, W16, bias)
    np.testing.assert_allclose(r["Y"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_w8a8_int_gemm_equals_int64_matmul(oracle_mod):
    rng = np.random.default_rng(23)
    M, N, Ki = 7, 9, 160
    Xq = rng.integers(-127, 128, size=(M, Ki)).astype(np.int8)
    Wq = rng.integers(-127, 128, size=(N, Ki)).astype(np.int8)
    np.testing.assert_array_equal(oracle_mod.int_gemm(Xq, Wq, 0),
                                  Xq.astype(np.int64) @ Wq.astype(np.int64).T)
