"""Parity of the 2:4-sparse weight path with the CPU oracle.

"QUIK: Towards End-to-End 4-Bit Inference on Generative Large Language
Models", abstract: inference with quantisation plus 2:4 sparsity.  The
weight pack (kept codes, position pairs, scales, outlier block) and the
integer sums of the sparse tensor-core product are bit-exact; the layer
output meets |y - ref| / max(|ref|, 1e-2) <= 2e-3 (ref in fp64, from the
oracle's 2:4 weights expanded to dense codes).  All calls go through the C
ABI.  Shapes cover ragged N, a ragged last k-block (K_i = 3968: half of a
256-position k-block), several token tiles, FP16 and INT8 outliers, k_o = 0
and k_o = K, and long K (the rings wrap).
"""
import numpy as np
import pytest
import torch

import oracle
import mixed_precision_quantized_quantize_b200 as q
from mixed_precision_quantized_quantize_b200 import workloads as wl

from helpers import assert_quant_equal, assert_y_close, gpu_tuple_np, np16

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q.lib()
    oracle.build()
    yield
    assert q.quik_sync_check() == q.QUIK_OK


# (M, N, K, k_o, int8 outliers, bias)
SHAPES = [
    (16, 256, 256, 0, False, True),      # one k-block, no outliers
    (1, 128, 512, 0, False, True),       # one token
    (5, 300, 640, 128, True, True),      # ragged N, INT8 outliers
    (16, 256, 4096, 128, False, False),  # K_i = 3968: ragged last k-block
    (17, 520, 1152, 128, False, True),   # 17 tokens (N = 32 per tile)
    (32, 136, 4224, 128, False, True),   # 32 tokens, 16 k-blocks (the rings wrap)
    (8, 384, 4352, 256, True, True),     # the largest INT8 outlier block
    (4, 128, 128, 128, False, True),     # everything is outlier (K_i = 0)
    (64, 200, 1152, 128, False, True),   # two token tiles
    (200, 300, 2176, 128, True, False),  # seven token tiles, INT8 outliers
    (24, 264, 8320, 128, True, False),   # long K
]


def _case(M, N, K, k_o, int8, bias, seed):
    cfg = wl.custom_config(M, N, K, k_o, 0, int8, bias, outlier_mult=30.0,
                           student_t=(seed % 2 == 1))
    return cfg, wl.make_layer(cfg, seed_offset=seed)


def _oracle_w24(d, k_o, int8):
    return oracle.prune24_quantize_rows(np16(d["W"]), d["perm"].numpy(), k_o, int8)


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_pack24_bit_exact(shape):
    M, N, K, k_o, int8, bias = shape
    cfg, d = _case(*shape, seed=21)
    g = q.pack_weights_24(d["W"].to(DEV), d["perm"].to(DEV), k_o, int8)
    torch.cuda.synchronize()
    ref = _oracle_w24(d, k_o, int8)
    names = ("kept codes", "position pairs", "scales", "outliers", "outlier scales")
    for name, a, b in zip(names, gpu_tuple_np(g), ref):
        if b is None:
            continue
        a = np.asarray(a)
        assert a.shape == b.shape, (name, a.shape, b.shape)
        assert np.array_equal(a.view(np.uint8), np.ascontiguousarray(b).view(np.uint8)), name


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_expand24_bit_exact(shape):
    """The dense packed codes the 2:4 weights stand for (the prefill path)."""
    M, N, K, k_o, int8, bias = shape
    if K == k_o:
        pytest.skip("no INT4 part")
    cfg, d = _case(*shape, seed=24)
    g = q.pack_weights_24(d["W"].to(DEV), d["perm"].to(DEV), k_o, int8)
    Wd = q.expand_weights_24(g[0], g[1], K, k_o)
    torch.cuda.synchronize()
    ow = _oracle_w24(d, k_o, int8)
    np.testing.assert_array_equal(Wd.cpu().numpy(), oracle.unpack24(ow[0], ow[1]))


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_sums24_bit_exact(shape):
    M, N, K, k_o, int8, bias = shape
    cfg, d = _case(*shape, seed=22)
    perm_d = d["perm"].to(DEV)
    gx = q.quantize_reorder(d["X"].to(DEV), perm_d, k_o, 0, int8)
    gw = q.pack_weights_24(d["W"].to(DEV), perm_d, k_o, int8)
    acc, acc_o = q.gemm24_i32(gx[0], gw[0], gw[1], K, k_o, gx[2], gw[3])
    torch.cuda.synchronize()
    ox = oracle.quantize_rows(np16(d["X"]), d["perm"].numpy(), k_o, 0, int8)
    assert_quant_equal(gpu_tuple_np(gx), ox, "X")
    ow = _oracle_w24(d, k_o, int8)
    if K - k_o > 0:
        ref = oracle.int_gemm(ox[0], oracle.unpack24(ow[0], ow[1]))
        np.testing.assert_array_equal(acc.cpu().numpy(), ref)
    if int8 and k_o > 0:
        ref_o = ox[2].astype(np.int64) @ ow[3].astype(np.int64).T
        np.testing.assert_array_equal(acc_o.cpu().numpy(), ref_o)


def _oracle_y24(d, k_o, int8):
    ox = oracle.quantize_rows(np16(d["X"]), d["perm"].numpy(), k_o, 0, int8)
    Qs, meta, sw, Wo, swo = _oracle_w24(d, k_o, int8)
    K = d["X"].shape[1]
    bias = None if d["bias"] is None else np16(d["bias"])
    return oracle.linear(ox[0], ox[1], ox[2] if k_o else None, ox[3], oracle.unpack24(Qs, meta),
                         sw, Wo if k_o else None, swo, bias, K, k_o)


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_linear24_within_tolerance(shape):
    M, N, K, k_o, int8, bias = shape
    cfg, d = _case(*shape, seed=23)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    layer = q.QuikLinear24(d["W"].to(DEV), perm_d, k_o, int8, b)
    X = d["X"].to(DEV)
    Y = layer(X)
    gx = q.quantize_reorder(X, perm_d, k_o, 0, int8)
    if M <= 32:  # the layer runs the sparse kernel
        Y2 = q.gemm_24(gx, (layer.Wq24, layer.Wmeta, layer.w_scale, layer.Wo, layer.wo_scale), K, k_o, b)
    else:        # the dense kernel on the expanded weights
        Wd = q.expand_weights_24(layer.Wq24, layer.Wmeta, K, k_o) if K > k_o else \
            torch.empty((N, 0), dtype=torch.uint8, device=DEV)
        Y2 = q.gemm(gx, (Wd, layer.w_scale, layer.Wo, layer.wo_scale), K, k_o, 0, b)
    torch.cuda.synchronize()
    assert_y_close(Y.float().cpu().numpy(), _oracle_y24(d, k_o, int8), f"linear24 {shape}")
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))
    if M > 32 and K > k_o:  # the sparse kernel on the same inputs, within the criterion
        Y3 = q.gemm_24(gx, (layer.Wq24, layer.Wmeta, layer.w_scale, layer.Wo, layer.wo_scale), K, k_o, b)
        torch.cuda.synchronize()
        assert_y_close(Y3.float().cpu().numpy(), _oracle_y24(d, k_o, int8), f"gemm24 {shape}")


def _samples(M, N, count, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(0, M, count), rng.integers(0, N, count)


@pytest.mark.parametrize("name", ["llama7b_up_sparse24_16x11008x4096",
                                  "llama7b_attn_sparse24_2048x4096x4096"])
def test_full_size_sparse24(name):
    """The benchmark's 2:4 workloads at full size: every kept code, pair and
    scale of W, and the output at sampled positions."""
    cfg = wl.CONFIGS[name]
    d = wl.make_layer(cfg)
    perm_d = d["perm"].to(DEV)
    layer = q.QuikLinear24(d["W"].to(DEV), perm_d, cfg.k_o, cfg.outlier_int8)
    Y = layer(d["X"].to(DEV))
    torch.cuda.synchronize()
    ow = _oracle_w24(d, cfg.k_o, cfg.outlier_int8)
    got = gpu_tuple_np((layer.Wq24, layer.Wmeta, layer.w_scale, layer.Wo))
    for a, b in zip(got, ow[:4]):
        assert np.array_equal(np.asarray(a).view(np.uint8), np.ascontiguousarray(b).view(np.uint8))
    ox = oracle.quantize_rows(np16(d["X"]), d["perm"].numpy(), cfg.k_o)
    ms, ns = _samples(cfg.M, cfg.N, 3000, seed=3)
    ref, _ = oracle.linear_sampled(ox[0], ox[1], ox[2], None, oracle.unpack24(ow[0], ow[1]), ow[2],
                                   ow[3], None, None, cfg.K, cfg.k_o, 0, ms, ns)
    assert_y_close(Y.float().cpu().numpy()[ms, ns], ref, name)
