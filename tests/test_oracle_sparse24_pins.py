"""Pins of the oracle's 2:4-sparse INT4 weights (``prune24_quantize_rows``,
``unpack24``).

"QUIK: Towards End-to-End 4-Bit Inference on Generative Large Language
Models" (codewithpapers page, abstract): inference with quantisation plus
2:4 sparsity.  Reading: aligned groups of four reordered INT4 positions keep
their two values of largest magnitude (lower position on ties); the row's
scale and codes follow the dense quantiser; the outlier block stays dense.

None of these re-types the oracle's arithmetic:
* hand-derived rows (tests/golden/sparse24.txt): bytes, metadata, scale;
* structure: every metadata nibble names a valid pair, every group keeps at
  most two nonzero codes, and no pruned value is larger in magnitude than a
  kept one of its group (checked on the fp16 inputs);
* the dense, separately pinned quantiser applied to the pruned rows gives the
  same codes and scales as unpacking the sparse rows;
* a layer whose weights are already 2:4 and lossless equals numpy's fp64
  product, and the sparse layer equals the dense oracle layer on the pruned
  weights exactly.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
VALID = {0b0100, 0b1000, 0b1100, 0b1001, 0b1101, 0b1110}  # i0 | i1 << 2, i0 < i1


def read_cases():
    cases, cur = [], {}
    with open(os.path.join(GOLDEN, "sparse24.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, vals = line.split(":", 1)
            cur[key.strip()] = vals.split()
            if key.strip() == "scale":
                cases.append(cur)
                cur = {}
    return cases


@pytest.mark.parametrize("case", read_cases())
def test_golden_rows(oracle_mod, case):
    W = np.array([[float(v) for v in case["values"]]], np.float16)
    Qs, meta, s, _, _ = oracle_mod.prune24_quantize_rows(W, np.arange(8, dtype=np.int32), 0)
    assert [int(b) for b in Qs[0]] == [int(h, 16) for h in case["qs"]]
    assert [int(b) for b in meta[0]] == [int(h, 16) for h in case["meta"]]
    assert s[0] == np.float32(case["scale"][0])


def decode(Q):
    lo = (Q & 0x0F).astype(np.int64)
    hi = (Q >> 4).astype(np.int64)
    out = np.empty((Q.shape[0], 2 * Q.shape[1]), np.int64)
    out[:, 0::2], out[:, 1::2] = lo, hi
    return np.where(out >= 8, out - 16, out)


def _weights(rng, N, K, heavy=True):
    W = rng.standard_normal((N, K)) * 0.02
    if heavy:
        W[:, rng.integers(0, K, 5)] *= 20
    W = W.astype(np.float16)
    W[0, :8] = 0  # a zero group (equal magnitudes)
    W[1, :8] = np.float16(0.01)
    return W


@pytest.mark.parametrize("k_o,int8", [(0, False), (32, False), (64, True)])
def test_structure(oracle_mod, k_o, int8):
    rng = np.random.default_rng(1 + k_o)
    N, K = 40, 512
    Ki = K - k_o
    W = _weights(rng, N, K)
    perm = rng.permutation(K).astype(np.int32)
    Qs, meta, s, O, so = oracle_mod.prune24_quantize_rows(W, perm, k_o, int8)
    nib = np.stack([meta & 0xF, meta >> 4], axis=2).reshape(N, Ki // 4)
    assert set(np.unique(nib).tolist()) <= VALID
    codes = decode(oracle_mod.unpack24(Qs, meta)).reshape(N, Ki // 4, 4)
    assert ((codes != 0).sum(axis=2) <= 2).all()
    # magnitudes: every kept value is at least as large as every pruned one
    v = np.abs(W.astype(np.float64)[:, perm[:Ki]]).reshape(N, Ki // 4, 4)
    i0, i1 = nib & 3, nib >> 2
    kept = np.zeros_like(v, bool)
    np.put_along_axis(kept, i0[..., None], True, axis=2)
    np.put_along_axis(kept, i1[..., None], True, axis=2)
    assert (kept.sum(axis=2) == 2).all()
    min_kept = np.where(kept, v, np.inf).min(axis=2)
    max_pruned = np.where(kept, -np.inf, v).max(axis=2)
    assert (min_kept >= max_pruned).all()
    # on equal magnitudes the lower positions are kept: a pruned value equal
    # to a kept one lies above it
    eq = (max_pruned == min_kept)
    for n, t in zip(*np.nonzero(eq)):
        kpos = np.nonzero(kept[n, t] & (v[n, t] == min_kept[n, t]))[0]
        ppos = np.nonzero(~kept[n, t] & (v[n, t] == min_kept[n, t]))[0]
        assert kpos.max() < ppos.min()


@pytest.mark.parametrize("k_o,int8", [(0, False), (32, False), (64, True)])
def test_unpacked_equals_dense_quantiser_on_pruned_rows(oracle_mod, k_o, int8):
    rng = np.random.default_rng(5 + k_o)
    N, K = 24, 384
    Ki = K - k_o
    W = _weights(rng, N, K)
    perm = rng.permutation(K).astype(np.int32)
    Qs, meta, s, O, so = oracle_mod.prune24_quantize_rows(W, perm, k_o, int8)
    # the pruned rows in source channel order: zero the positions the
    # metadata drops (this reads only the pattern, not the codes)
    nib = np.stack([meta & 0xF, meta >> 4], axis=2).reshape(N, Ki // 4)
    keep = np.zeros((N, Ki // 4, 4), bool)
    np.put_along_axis(keep, (nib & 3)[..., None], True, axis=2)
    np.put_along_axis(keep, (nib >> 2)[..., None], True, axis=2)
    Wp = W.copy()
    drop_src = perm[:Ki][None, :].repeat(N, 0)[~keep.reshape(N, Ki)]
    rows = np.nonzero(~keep.reshape(N, Ki))[0]
    Wp[rows, drop_src] = 0
    Q, sd, Od, sod = oracle_mod.quantize_rows(Wp, perm, k_o, 0, int8)
    assert np.array_equal(oracle_mod.unpack24(Qs, meta), Q)
    assert np.array_equal(s, sd)
    assert np.array_equal(O, Od)
    if int8:
        assert np.array_equal(so, sod)


def test_lossless_sparse_layer_equals_fp64_matmul(oracle_mod):
    """Weights already 2:4 with values code * 2^e (a +-7 per row), lossless
    activations: the layer output equals numpy's fp64 product."""
    rng = np.random.default_rng(9)
    M, N, K, k_o = 8, 48, 256, 32
    Ki = K - k_o
    perm = rng.permutation(K).astype(np.int32)
    Wc = np.zeros((N, K))
    for n in range(N):
        row = np.zeros(Ki)
        for t in range(Ki // 4):
            pos = rng.choice(4, 2, replace=False)
            row[4 * t + pos] = rng.integers(-7, 8, 2)
        row[4 * rng.integers(0, Ki // 4) + rng.integers(0, 4)] = 0
        t = rng.integers(0, Ki // 4)
        row[4 * t:4 * t + 4] = [7, 0, 0, -3]
        Wc[n, perm[:Ki]] = row
        Wc[n, perm[Ki:]] = rng.integers(-7, 8, k_o)
    W = Wc * 2.0 ** rng.integers(-9, -5, size=(N, 1))
    Xc = rng.integers(-7, 8, size=(M, K)).astype(np.float64)
    Xc[:, perm[rng.integers(0, Ki)]] = 7
    X = Xc * 2.0 ** rng.integers(-3, 1, size=(M, 1))
    assert np.array_equal(W.astype(np.float16).astype(np.float64), W)
    W16, X16 = W.astype(np.float16), X.astype(np.float16)
    Qs, meta, sw, Wo, swo = oracle_mod.prune24_quantize_rows(W16, perm, k_o)
    Wq = oracle_mod.unpack24(Qs, meta)
    Xq, sx, Xo, sxo = oracle_mod.quantize_rows(X16, perm, k_o)
    Y = oracle_mod.linear(Xq, sx, Xo, sxo, Wq, sw, Wo, swo, None, K, k_o)
    assert np.array_equal(Y, X @ W.T)
