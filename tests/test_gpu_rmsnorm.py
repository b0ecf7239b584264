"""Parity of the RMS-norm-fused quantiser and layer with the CPU oracle.

"Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", Summary
and idea I2: the activation quantiser runs inside the RMS norm in front of
the projection.  All calls go through the C ABI.

What must match, and why: everything, bit for bit.
* codes (INT4, INT8 activations, INT8 outliers) depend only on z = h * gamma
  (exact in fp32) and the fp32 base scale, never on the norm's row factor r;
* stored scales (x_scale, xo_scale) = fl32(s_z * r) and FP16 outliers
  fl16(z * r): both sides take the sum of squares exactly (every fp16 square
  is an integer multiple of 2^-48), round it once to fp64 and take r with
  the same IEEE fp64 steps, so r is the same double on both sides whatever
  order each summed in;
* the layer output: the criterion of every other layer test,
  |y - ref| / max(|ref|, 1e-2) <= 2e-3 with ref in fp64;
* an exactly representable case (integer rows, mean(h^2) + eps = 64, so
  r = 1/8 and every fp32 step is exact on both sides).
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


def _case(M, N, K, k_o, group, int8, bias, seed, act_bits=4):
    cfg = wl.custom_config(M, N, K, k_o, group, int8, bias, outlier_mult=30.0,
                           student_t=(seed % 2 == 1), act_bits=act_bits, rmsnorm=True)
    return cfg, wl.make_layer(cfg, seed_offset=seed)


def _oracle_norm_quant(d, k_o, group, int8, bits=4):
    return oracle.rmsnorm_quantize_rows(np16(d["X"]), np16(d["gamma"]), d["eps"],
                                        d["perm"].numpy(), k_o, group, int8, bits)


# (M, N, K, k_o, group, int8 outliers, bias, act_bits)
SHAPES = [
    (16, 256, 256, 32, 0, False, True, 4),      # the tiny layer
    (200, 300, 640, 64, 0, False, True, 4),     # ragged M, N
    (70, 300, 544, 32, 0, True, True, 4),       # INT8 outliers
    (64, 100, 256, 0, 0, False, True, 4),       # no outliers
    (64, 256, 256, 256, 0, False, True, 4),     # everything is outlier (FP16)
    (48, 144, 256, 256, 0, True, False, 4),     # everything is outlier (INT8)
    (150, 260, 1152, 128, 128, True, True, 4),  # groups + INT8 outliers
    (100, 200, 640, 128, 128, False, False, 4), # groups + FP16 outliers
    (96, 136, 512, 0, 128, True, True, 4),      # groups, no outliers
    (257, 513, 2080, 32, 0, False, True, 4),    # 3 x 3 tiles, long K
    (33, 72, 20544, 64, 0, True, True, 4),      # the widest rows (uint16 perm table)
    (5, 300, 640, 64, 0, True, True, 4),        # decode-shaped
    (200, 300, 640, 64, 0, False, True, 8),     # INT8 activations (W4A8)
    (70, 300, 544, 32, 0, True, True, 8),       # W4A8 + INT8 outliers
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_rmsnorm_quantize_parity(shape):
    M, N, K, k_o, group, int8, bias, ab = shape
    cfg, d = _case(M, N, K, k_o, group, int8, bias, seed=3, act_bits=ab)
    g = q.rmsnorm_quantize_reorder(d["X"].to(DEV), d["gamma"].to(DEV), d["eps"],
                                   d["perm"].to(DEV), k_o, group, int8, act_bits=ab)
    torch.cuda.synchronize()
    assert_quant_equal(gpu_tuple_np(g), _oracle_norm_quant(d, k_o, group, int8, ab),
                            f"rmsnorm {shape}")


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_rmsnorm_linear_within_tolerance(shape):
    M, N, K, k_o, group, int8, bias, ab = shape
    cfg, d = _case(M, N, K, k_o, group, int8, bias, seed=4, act_bits=ab)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    gamma = d["gamma"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, group, int8, b, act_bits=ab,
                         norm_weight=gamma, norm_eps=d["eps"])
    X = d["X"].to(DEV)
    Y = layer(X)
    # the same through the fused quantiser and the GEMM as two calls
    gx = q.rmsnorm_quantize_reorder(X, gamma, d["eps"], perm_d, k_o, group, int8, act_bits=ab)
    Y2 = q.gemm(gx, (layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale), K, k_o, group, b)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm_layer(np16(d["X"]), np16(d["gamma"]), d["eps"], np16(d["W"]),
                               d["perm"].numpy(), None if d["bias"] is None else np16(d["bias"]),
                               k_o, group, int8, ab)["Y"]
    assert_y_close(Y.float().cpu().numpy(), ref, f"rmsnorm linear {shape}")
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))


def _exact_rows(rng, R, K):
    """Integer rows in [-7, 7] sharing one sum of squares S, gamma = k/64,
    and eps = 64 - S/K (K a power of two): r = 1/8 exactly, on both sides."""
    base = rng.integers(-7, 8, size=K)
    base[0] = 7
    h = np.stack([rng.permutation(base) * rng.choice([-1, 1], size=K) for _ in range(R)])
    eps = 64.0 - float((base.astype(np.int64) ** 2).sum()) / K
    gamma = rng.integers(1, 256, size=K) * rng.choice([-1, 1], size=K) / 64.0
    return h.astype(np.float16), gamma.astype(np.float16), eps


@pytest.mark.parametrize("K,k_o,group,int8,ab", [(256, 32, 0, False, 4), (512, 128, 128, True, 4),
                                                 (1024, 64, 0, True, 8), (4096, 128, 0, False, 4)])
def test_rmsnorm_exact_case_bit_exact(K, k_o, group, int8, ab):
    rng = np.random.default_rng(K + k_o)
    h, gamma, eps = _exact_rows(rng, 300, K)
    perm = rng.permutation(K).astype(np.int32)
    g = q.rmsnorm_quantize_reorder(torch.from_numpy(h).to(DEV), torch.from_numpy(gamma).to(DEV),
                                   eps, torch.from_numpy(perm).to(DEV), k_o, group, int8,
                                   act_bits=ab)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm_quantize_rows(h, gamma, eps, perm, k_o, group, int8, ab)
    assert_quant_equal(gpu_tuple_np(g), ref, f"exact case K={K}")


def test_rmsnorm_zero_row():
    """A zero row: r = 1/sqrt(eps), every code and scale 0, outliers 0."""
    cfg, d = _case(8, 16, 640, 64, 0, True, False, seed=5)
    X = d["X"].clone()
    X[3] = 0
    d["X"] = X
    g = q.rmsnorm_quantize_reorder(X.to(DEV), d["gamma"].to(DEV), d["eps"], d["perm"].to(DEV),
                                   64, 0, True)
    torch.cuda.synchronize()
    gq = gpu_tuple_np(g)
    assert not gq[0][3].any() and gq[1][3] == 0 and not gq[2][3].any() and gq[3][3] == 0
    assert_quant_equal(gq, _oracle_norm_quant(d, 64, 0, True), "zero row")


def _samples(M, N, count, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(0, M, count), rng.integers(0, N, count)


def test_rmsnorm_full_size_layer():
    """The benchmark's norm-fused workload at full size: every code and scale
    of the 2048 x 4096 hidden state, and the output at sampled positions."""
    cfg = wl.CONFIGS["llama7b_attn_rmsnorm_2048x4096x4096"]
    d = wl.make_layer(cfg)
    perm_d = d["perm"].to(DEV)
    gamma = d["gamma"].to(DEV)
    X = d["X"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, cfg.k_o, cfg.group, cfg.outlier_int8,
                         norm_weight=gamma, norm_eps=d["eps"])
    Y = layer(X)
    gx = q.rmsnorm_quantize_reorder(X, gamma, d["eps"], perm_d, cfg.k_o)
    torch.cuda.synchronize()
    ox = _oracle_norm_quant(d, cfg.k_o, cfg.group, cfg.outlier_int8)
    assert_quant_equal(gpu_tuple_np(gx), ox, "full-size X")
    ow = oracle.quantize_rows(np16(d["W"]), d["perm"].numpy(), cfg.k_o)
    ms, ns = _samples(cfg.M, cfg.N, 3000, seed=2)
    ref, _ = oracle.linear_sampled(ox[0], ox[1], ox[2], None, ow[0], ow[1], ow[2], None, None,
                                   cfg.K, cfg.k_o, 0, ms, ns)
    assert_y_close(Y.float().cpu().numpy()[ms, ns], ref, "full-size rmsnorm layer")


def test_rmsnorm_extreme_magnitudes_bit_exact():
    """Rows whose squares span the whole fp16 range (subnormals up to 65504,
    so the exact sums pass 2^64 units of 2^-48): scales and outliers still
    bit-exact, per token and grouped."""
    rng = np.random.default_rng(23)
    R, K, k_o = 300, 4096, 128
    h = rng.standard_normal((R, K)) * 2.0 ** rng.uniform(-22, 15, (R, K))
    h = np.clip(h, -65504, 65504).astype(np.float16)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    eps = 1e-6
    for group, int8 in ((0, False), (0, True), (128, True)):
        g = q.rmsnorm_quantize_reorder(torch.from_numpy(h).to(DEV), torch.from_numpy(gamma).to(DEV),
                                       eps, torch.from_numpy(perm).to(DEV), k_o, group, int8)
        torch.cuda.synchronize()
        ref = oracle.rmsnorm_quantize_rows(h, gamma, eps, perm, k_o, group, int8)
        assert_quant_equal(gpu_tuple_np(g), ref, f"extreme rows group={group} int8={int8}")
