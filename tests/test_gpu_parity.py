"""Parity of the CUDA path with the CPU oracle, element by element.

Codes, scales, outlier blocks and INT32 sums must be bit-exact; fp16 outputs
must satisfy |y - ref| / max(|ref|, 1e-2) <= 2e-3 (ref in fp64).  Shapes span
several tiles with ragged tails in M, N and K; degenerate cases (k_o = 0,
k_o = K, zero rows, exact ties) are included.  All calls go through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
import mixed_precision_quantized_quantize_b200 as q
from mixed_precision_quantized_quantize_b200 import workloads as wl

from helpers import (assert_quant_equal, assert_y_close, gpu_tuple_np, np16, oracle_quant)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q.lib()
    oracle.build()
    yield
    assert q.quik_sync_check() == q.QUIK_OK


# (M, N, K, k_o, group, int8, bias)
SHAPES = [
    (16, 256, 256, 32, 0, False, True),      # the tiny layer
    (200, 300, 640, 64, 0, False, True),     # ragged M, N; K_i = 576 = 4.5 k-blocks
    (130, 520, 1056, 32, 0, False, False),   # 2 M tiles, 3 N tiles
    (64, 100, 256, 0, 0, False, True),       # no outliers; N % 8 != 0
    (64, 256, 256, 256, 0, False, True),     # everything is outlier (FP16 GEMM)
    (70, 300, 544, 32, 0, True, True),       # INT8 outliers, partial INT8 k-block
    (150, 260, 1152, 128, 128, True, True),  # groups + INT8 outliers
    (100, 200, 640, 128, 128, False, False), # groups + FP16 outliers
    (96, 136, 512, 0, 128, True, True),      # groups, no outliers
    (48, 144, 128, 128, 128, True, False),   # groups, everything outlier (INT8)
    (257, 513, 2080, 32, 0, False, True),    # 3 x 3 tiles, long K
    # long K: the operand ring wraps many times before the outlier k-blocks
    # (a producer running ahead must never alias a barrier phase)
    (200, 300, 8320, 128, 128, True, True),  # 64 groups + INT8 outliers
    (130, 260, 8256, 64, 0, False, True),    # 64 INT4 k-blocks + FP16 outliers
    # K_i = 20480: the quantiser's widest rows (8 words per thread, 10 warps)
    (33, 72, 20544, 64, 0, True, True),
    # decode-shaped products (M <= 32, per-channel scales): W as the MMA's rows
    (1, 128, 256, 32, 0, False, True),       # one token
    (5, 300, 640, 64, 0, True, True),        # 5 tokens, ragged N, INT8 outliers
    (17, 520, 1056, 32, 0, False, False),    # 17 tokens: the MMA's N = 32
    (32, 136, 4224, 128, 0, False, True),    # 32 tokens, the largest FP16 outlier block (k_o = 128)
    (32, 136, 4160, 256, 0, False, True),    # FP16 k_o = 256: past that block, the pair kernel
    (8, 384, 4352, 256, 0, True, True),      # the largest INT8 outlier block (k_o = 256)
    (4, 128, 128, 128, 0, False, True),      # everything is outlier
    (24, 264, 8320, 128, 0, True, False),    # long K (the W ring wraps 4 times), INT8 outliers
    (16, 130, 160, 0, 0, False, True),       # no outliers, partial k-block, ragged N
]


def _case(M, N, K, k_o, group, int8, bias, seed):
    cfg = wl.custom_config(M, N, K, k_o, group, int8, bias, outlier_mult=30.0,
                           student_t=(seed % 2 == 1))
    return cfg, wl.make_layer(cfg, seed_offset=seed)


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_quantize_and_pack_bit_exact(shape):
    M, N, K, k_o, group, int8, bias = shape
    cfg, d = _case(*shape, seed=7)
    perm_d = d["perm"].to(DEV)
    gx = q.quantize_reorder(d["X"].to(DEV), perm_d, k_o, group, int8)
    gw = q.pack_weights(d["W"].to(DEV), perm_d, k_o, group, int8)
    torch.cuda.synchronize()
    assert_quant_equal(gpu_tuple_np(gx), oracle_quant(d["X"], d["perm"], k_o, group, int8), "X")
    assert_quant_equal(gpu_tuple_np(gw), oracle_quant(d["W"], d["perm"], k_o, group, int8), "W")


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_int32_sums_bit_exact(shape):
    M, N, K, k_o, group, int8, bias = shape
    cfg, d = _case(*shape, seed=11)
    perm_d = d["perm"].to(DEV)
    gx = q.quantize_reorder(d["X"].to(DEV), perm_d, k_o, group, int8)
    gw = q.pack_weights(d["W"].to(DEV), perm_d, k_o, group, int8)
    acc, acc_o = q.gemm_i32(gx[0], gw[0], K, k_o, group, gx[2], gw[2])
    torch.cuda.synchronize()
    ox = oracle_quant(d["X"], d["perm"], k_o, group, int8)
    ow = oracle_quant(d["W"], d["perm"], k_o, group, int8)
    if K - k_o > 0:
        ref = oracle.int_gemm(ox[0], ow[0], group)
        np.testing.assert_array_equal(acc.cpu().numpy(), ref)
    if int8 and k_o > 0:
        ref_o = ox[2].astype(np.int64) @ ow[2].astype(np.int64).T
        np.testing.assert_array_equal(acc_o.cpu().numpy(), ref_o)


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_linear_output_within_tolerance(shape):
    M, N, K, k_o, group, int8, bias = shape
    cfg, d = _case(*shape, seed=13)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, group, int8, b)
    Y = layer(d["X"].to(DEV))
    # the same result through quantize + gemm as two calls
    gx = q.quantize_reorder(d["X"].to(DEV), perm_d, k_o, group, int8)
    Y2 = q.gemm(gx, (layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale), K, k_o, group, b)
    torch.cuda.synchronize()
    ref = oracle.layer(np16(d["X"]), np16(d["W"]), d["perm"].numpy(),
                       None if d["bias"] is None else np16(d["bias"]), k_o, group, int8)["Y"]
    y = Y.float().cpu().numpy()
    assert_y_close(y, ref, f"linear {shape}")
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))


def _wide_expected(Q, Ki):
    """The oracle's packed codes (code 2i in the low nibble of byte i) as the
    layer call's widened operand: per 32 positions the 16 even ones, then the
    16 odd ones, each as the signed byte 16 c."""
    lo = (Q & 0xF).astype(np.int16)
    hi = (Q >> 4).astype(np.int16)
    codes = np.empty((Q.shape[0], Ki), np.int16)
    codes[:, 0::2] = np.where(lo > 7, lo - 16, lo)
    codes[:, 1::2] = np.where(hi > 7, hi - 16, hi)
    blocks = codes.reshape(Q.shape[0], Ki // 32, 16, 2)     # [row, block, j, parity]
    wide = blocks.transpose(0, 1, 3, 2).reshape(Q.shape[0], Ki)  # [row, block, parity, j]
    return (wide * 16).astype(np.int8)


def _r256(n):
    return (n + 255) // 256 * 256


# (M, K, k_o): layer calls above 32 tokens with FP16 or no outliers, whose
# quantiser writes the widened codes: one to eight words per thread (K_i from
# 448 to 20480), a few rows per SM up to more than 16 (4101 rows), the
# attention projection's rows, no outliers
WIDE = [(64, 512, 64), (200, 640, 64), (2048, 4096, 128), (4101, 1024, 0), (300, 8256, 64),
        (130, 11008, 0), (40, 20544, 64)]


@pytest.mark.parametrize("shape", WIDE, ids=[str(s) for s in WIDE])
def test_wide_codes_bit_exact(shape):
    """The layer call's widened codes, scales and FP16 outliers (read from
    its workspace) against the oracle's, bit for bit."""
    M, K, k_o = shape
    Ki = K - k_o
    cfg, d = _case(M, 64, K, k_o, 0, False, False, seed=17)
    perm_d = d["perm"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, 0, False, None)
    shape_s = layer.shape(M)
    ws = torch.full((q.quik_workspace_size(shape_s),), 0x5A, dtype=torch.uint8, device=DEV)
    Y = torch.empty((M, 64), dtype=torch.float16, device=DEV)
    q.quik_linear(shape_s, d["X"].to(DEV), perm_d, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale,
                  None, Y, ws)
    torch.cuda.synchronize()
    w = ws.cpu().numpy()
    Q, sx, O, _ = oracle_quant(d["X"], d["perm"], k_o, 0, False)
    np.testing.assert_array_equal(w[:M * Ki].view(np.int8).reshape(M, Ki), _wide_expected(Q, Ki))
    o_sx = _r256(M * Ki)
    np.testing.assert_array_equal(w[o_sx:o_sx + 4 * M].view(np.uint32), sx.view(np.uint32))
    if k_o:
        o_xo = o_sx + _r256(4 * M)
        np.testing.assert_array_equal(w[o_xo:o_xo + 2 * M * k_o].view(np.uint16).reshape(M, k_o),
                                      O.view(np.uint16))


def test_wide_codes_bad_perm_reported():
    """Entries of perm outside [0, K) read channel 0 and are reported, in the
    widened quantiser too; its codes then equal the oracle's on that perm
    (channel 0 twice: a repeated channel)."""
    M, K, k_o = 100, 512, 64
    cfg, d = _case(M, 64, K, k_o, 0, False, False, seed=19)
    perm = d["perm"].clone()
    perm[7] = K + 5
    perm[K - 3] = -2
    perm_d = perm.to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), d["perm"].to(DEV), k_o, 0, False, None)
    shape_s = layer.shape(M)
    ws = torch.zeros((q.quik_workspace_size(shape_s),), dtype=torch.uint8, device=DEV)
    Y = torch.empty((M, 64), dtype=torch.float16, device=DEV)
    assert q.quik_sync_check() == q.QUIK_OK
    q.quik_linear(shape_s, d["X"].to(DEV), perm_d, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale,
                  None, Y, ws)
    torch.cuda.synchronize()
    assert q.quik_sync_check() == q.QUIK_ERR_INVALID_ARG
    assert q.quik_sync_check() == q.QUIK_OK
    p0 = perm.numpy().copy()
    p0[(p0 < 0) | (p0 >= K)] = 0
    Q, sx, O, _ = oracle.quantize_rows(np16(d["X"]), p0, k_o, 0, False)
    w = ws.cpu().numpy()
    Ki = K - k_o
    np.testing.assert_array_equal(w[:M * Ki].view(np.int8).reshape(M, Ki), _wide_expected(Q, Ki))
    o_sx = _r256(M * Ki)
    np.testing.assert_array_equal(w[o_sx:o_sx + 4 * M].view(np.uint32), sx.view(np.uint32))
    o_xo = o_sx + _r256(4 * M)
    np.testing.assert_array_equal(w[o_xo:o_xo + 2 * M * k_o].view(np.uint16).reshape(M, k_o), O.view(np.uint16))


def test_zero_rows_and_ties():
    """All-zero rows give zero scales and codes; exact half-way values round to even."""
    M, N, K, k_o = 40, 64, 256, 32
    rng = np.random.default_rng(3)
    X = rng.standard_normal((M, K)).astype(np.float16)
    X[3] = 0
    X[17] = 0
    # ties: with max|x| = 7 (s = 1), x in {k + 0.5} lands exactly between codes
    X[5] = np.resize(np.array([7, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5], np.float16), K)
    perm = np.arange(K, dtype=np.int32)
    perm_t = torch.from_numpy(perm)
    for group, int8 in [(0, False), (0, True), (128, True)]:
        Kq = K if group == 0 else 128 + k_o  # grouped needs K_i % 128 == 0
        Xk = np.ascontiguousarray(X[:, :Kq])
        pk = torch.from_numpy(np.arange(Kq, dtype=np.int32))
        g = q.quantize_reorder(torch.from_numpy(Xk).to(DEV), pk.to(DEV), k_o, group, int8)
        torch.cuda.synchronize()
        assert_quant_equal(gpu_tuple_np(g), oracle.quantize_rows(Xk, pk.numpy(), k_o, group, int8))
        sc = g[1].cpu().numpy().reshape(M, -1)
        assert (sc[3] == 0).all() and (sc[17] == 0).all()
    del perm_t


@pytest.mark.parametrize("group,int8", [(0, False), (0, True), (128, True)])
def test_quantize_many_rows_per_cta(group, int8):
    """8192 rows: every quantiser CTA walks several rows through its two-slot ring."""
    M, K, k_o = 8192, 1024 + 64, 64
    cfg, d = _case(M, 16, K, k_o, group, int8, False, seed=11)
    g = q.quantize_reorder(d["X"].to(DEV), d["perm"].to(DEV), k_o, group, int8)
    torch.cuda.synchronize()
    assert_quant_equal(gpu_tuple_np(g), oracle_quant(d["X"], d["perm"], k_o, group, int8))


@pytest.mark.parametrize("int8", [False, True])
def test_scales_for_every_fp16_absmax(int8):
    """Row r's absmax runs over every finite non-negative fp16 value: the scales are the
    IEEE fp32 quotients fl(m / 7) and fl(m / 127), and codes match the oracle bit for bit."""
    vals = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16)  # +0 .. 65504
    M, Ki, k_o = len(vals), 32, 16
    K = Ki + k_o
    X = np.zeros((M, K), np.float16)
    X[:, 0] = vals
    X[:, 1] = -vals
    X[:, 5] = (vals.astype(np.float32) * np.float32(0.3)).astype(np.float16)
    X[:, 9] = (vals.astype(np.float32) * np.float32(-0.77)).astype(np.float16)
    X[:, Ki] = vals
    X[:, Ki + 3] = (vals.astype(np.float32) * np.float32(0.51)).astype(np.float16)
    perm = torch.arange(K, dtype=torch.int32)
    g = q.quantize_reorder(torch.from_numpy(X).to(DEV), perm.to(DEV), k_o, 0, int8)
    torch.cuda.synchronize()
    got = gpu_tuple_np(g)
    m32 = vals.astype(np.float32)
    np.testing.assert_array_equal(got[1].reshape(-1).view(np.uint32), (m32 / np.float32(7)).view(np.uint32))
    if int8:
        np.testing.assert_array_equal(got[3].reshape(-1).view(np.uint32), (m32 / np.float32(127)).view(np.uint32))
    assert_quant_equal(got, oracle.quantize_rows(X, perm.numpy(), k_o, 0, int8))


def test_out_of_range_perm_is_reported():
    """perm entries outside [0, K) are never read out of bounds; sync_check reports them."""
    M, K, k_o = 8, 256, 32
    X = torch.randn((M, K), dtype=torch.float16, device=DEV)
    perm = torch.arange(K, dtype=torch.int32)
    perm[5] = K + 3
    perm[9] = -1
    assert q.quik_sync_check() == q.QUIK_OK
    q.quantize_reorder(X, perm.to(DEV), k_o)
    assert q.quik_sync_check() == q.QUIK_ERR_INVALID_ARG
    assert q.quik_sync_check() == q.QUIK_OK  # the count was cleared


def test_canary_guards_untouched():
    """Writes stay inside the output buffers: guard bytes around each are unchanged."""
    M, N, K, k_o = 130, 300, 640, 64
    cfg, d = _case(M, N, K, k_o, 0, False, True, seed=5)
    G = 4096
    pat = 0xA5

    def guarded(nbytes):
        buf = torch.full((G + nbytes + G,), pat, dtype=torch.uint8, device=DEV)
        return buf, buf[G:G + nbytes]

    Ki = K - k_o
    bq, Xq = guarded(M * Ki // 2)
    bs, sxb = guarded(M * 4)
    bo, Xob = guarded(M * k_o * 2)
    by, Yb = guarded(M * N * 2)
    perm_d = d["perm"].to(DEV)
    shape = q.make_shape(M, N, K, k_o)
    q.quik_quantize_reorder(shape, d["X"].to(DEV), perm_d, Xq, sxb.view(torch.float32),
                            Xob.view(torch.float16), None)
    gw = q.pack_weights(d["W"].to(DEV), perm_d, k_o)
    q.quik_gemm(shape, Xq, sxb.view(torch.float32), Xob.view(torch.float16), None, gw[0], gw[1],
                gw[2], None, d["bias"].to(DEV), Yb.view(torch.float16))
    torch.cuda.synchronize()
    for buf in (bq, bs, bo, by):
        h = buf.cpu().numpy()
        assert (h[:G] == pat).all() and (h[-G:] == pat).all()


def test_timeout_is_reported_without_fault():
    assert q.quik_sync_check() == q.QUIK_OK
    q.quik_selftest_timeout(2000)  # 2 ms limit on a barrier nothing completes
    assert q.quik_sync_check() == q.QUIK_ERR_TIMEOUT
    assert q.quik_sync_check() == q.QUIK_OK  # the word was cleared
    # the context is still usable
    x = torch.ones(4, device=DEV)
    assert float(x.sum()) == 4.0


def test_invalid_arguments_enqueue_nothing():
    X = torch.zeros((16, 256), dtype=torch.float16, device=DEV)
    perm = torch.arange(256, dtype=torch.int32, device=DEV)
    with pytest.raises(q.QuikError) as e:
        q.quantize_reorder(X, perm, 24)  # k_o not a multiple of 16
    assert e.value.status == q.QUIK_ERR_INVALID_ARG
    with pytest.raises(q.QuikError) as e:
        q.quik_quantize_reorder(q.make_shape(16, 1, 256, 32, 64), X, perm, None, None, None, None)
    assert e.value.status == q.QUIK_ERR_UNSUPPORTED


# ------------------------------------------------------------------ full-size layers
FULL = [
    ("tiny_16x256x256", None),
    ("llama7b_attn_2048x4096x4096", None),
    ("llama7b_up_16x11008x4096", None),
    ("llama7b_up_256x11008x4096", None),
    ("llama7b_up_2048x11008x4096", None),
    ("llama65b_mlp_grouped_1024x22016x8192", None),
    ("llama7b_down_fused_4096x4096x11008", None),
    ("llama7b_attn_w4a8_2048x4096x4096", None),
    ("llama7b_attn_w8a8_2048x4096x4096", None),
]


def _samples(M, N, count, seed):
    rng = np.random.default_rng(seed)
    ms = rng.integers(0, M, count)
    ns = rng.integers(0, N, count)
    # always include the corners and the last row / column
    extra_m = np.array([0, M - 1, 0, M - 1, M // 2])
    extra_n = np.array([0, N - 1, N - 1, 0, N // 2])
    return np.concatenate([ms, extra_m]), np.concatenate([ns, extra_n])


@pytest.mark.parametrize("name", [f[0] for f in FULL])
def test_full_size_layer(name):
    cfg = wl.CONFIGS[name]
    d = wl.make_layer(cfg)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    X = d["X"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, cfg.k_o, cfg.group, cfg.outlier_int8, b,
                         act_bits=cfg.act_bits, weight_bits=cfg.weight_bits)
    Y = layer(X)
    gx = q.quantize_reorder(X, perm_d, cfg.k_o, cfg.group, cfg.outlier_int8, act_bits=cfg.act_bits)
    torch.cuda.synchronize()
    ox = oracle.quantize_rows(np16(d["X"]), d["perm"].numpy(), cfg.k_o, cfg.group, cfg.outlier_int8,
                              cfg.act_bits)
    ow = oracle.quantize_rows(np16(d["W"]), d["perm"].numpy(), cfg.k_o, cfg.group, cfg.outlier_int8,
                              cfg.weight_bits)
    # every code, scale and outlier value, activations and weights
    assert_quant_equal(gpu_tuple_np(gx), ox, f"{name} X")
    assert_quant_equal(gpu_tuple_np((layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale)), ow,
                       f"{name} W")
    # outputs at sampled positions, each computed by the oracle one by one
    ms, ns = _samples(cfg.M, cfg.N, 3000, seed=1)
    bias_np = None if d["bias"] is None else np16(d["bias"])
    ref, ref_acc = oracle.linear_sampled(ox[0], ox[1], ox[2] if cfg.k_o else None, ox[3],
                                         ow[0], ow[1], ow[2] if cfg.k_o else None, ow[3], bias_np,
                                         cfg.K, cfg.k_o, cfg.group, ms, ns)
    y = Y.float().cpu().numpy()[ms, ns]
    assert_y_close(y, ref, name)
    # integer sums at sampled positions (one per group with groups), from a
    # row/column slice of the same kernel
    rows = np.unique(ms)[:256]
    cols = np.unique(ns)[:512]
    r_t = torch.from_numpy(rows).to(DEV)
    c_t = torch.from_numpy(cols).to(DEV)
    int8_o = cfg.outlier_int8 and cfg.k_o > 0
    acc, acc_o = q.gemm_i32(gx[0][r_t].contiguous(), layer.Wq[c_t].contiguous(), cfg.K, cfg.k_o,
                            cfg.group, gx[2][r_t].contiguous() if int8_o else None,
                            layer.Wo[c_t].contiguous() if int8_o else None)
    full = oracle.int_gemm(ox[0][rows], ow[0][cols], cfg.group)
    np.testing.assert_array_equal(acc.cpu().numpy(), full)
    if int8_o:  # the INT8 outlier block's sums, exact
        ref_o = ox[2][rows].astype(np.int64) @ ow[2][cols].astype(np.int64).T
        np.testing.assert_array_equal(acc_o.cpu().numpy(), ref_o)


# the layers small enough for the oracle to compute every output: the tiny
# layer, the Llama-7B attention projection at 2048 tokens and the up
# projection at 16 and 256 tokens
EVERY_ELEMENT = ["tiny_16x256x256", "llama7b_attn_2048x4096x4096", "llama7b_up_16x11008x4096",
                 "llama7b_up_256x11008x4096"]


@pytest.mark.parametrize("name", EVERY_ELEMENT)
def test_full_size_every_element(name):
    """At the full size, every output of the layer call (the kernels the bench
    times: the widened-operand persistent GEMM above 32 tokens, the decode
    kernel up to 32) against the oracle's fp64 layer; every INT32 sum of the
    same GEMM (its debug instantiation, fed the packed codes, writes all M x N
    sums) against the oracle's exact sums; and the two-call path
    (quik_quantize_reorder + quik_gemm) bit-identical to the layer call."""
    cfg = wl.CONFIGS[name]
    d = wl.make_layer(cfg, seed_offset=5)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    X = d["X"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, cfg.k_o, cfg.group, cfg.outlier_int8, b)
    Y = layer(X)
    gx = q.quantize_reorder(X, perm_d, cfg.k_o, cfg.group, cfg.outlier_int8)
    Y2 = q.gemm(gx, (layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale), cfg.K, cfg.k_o,
                cfg.group, b)
    acc, _ = q.gemm_i32(gx[0], layer.Wq, cfg.K, cfg.k_o, 0)
    torch.cuda.synchronize()
    ox = oracle.quantize_rows(np16(d["X"]), d["perm"].numpy(), cfg.k_o, 0, cfg.outlier_int8)
    ow = oracle.quantize_rows(np16(d["W"]), d["perm"].numpy(), cfg.k_o, 0, cfg.outlier_int8)
    assert_quant_equal(gpu_tuple_np(gx), ox, f"{name} X")
    assert_quant_equal(gpu_tuple_np((layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale)), ow,
                       f"{name} W")
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.int_gemm(ox[0], ow[0], 0))
    bias_np = None if d["bias"] is None else np16(d["bias"])
    ref = oracle.linear(ox[0], ox[1], ox[2] if cfg.k_o else None, ox[3], ow[0], ow[1],
                        ow[2] if cfg.k_o else None, ow[3], bias_np, cfg.K, cfg.k_o, 0)
    assert_y_close(Y.float().cpu().numpy(), ref, name)
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))


# ----------------------------------------------------------------- INT8 activations (W4A8)
# (M, N, K, k_o, int8 outliers, bias); per-token scales
SHAPES_A8 = [
    (16, 256, 256, 32, False, True),      # the tiny layer
    (200, 300, 640, 64, False, True),     # ragged M, N; K_i = 576 = 4.5 k-blocks
    (130, 520, 1056, 32, False, False),   # 2 M tiles, 3 N tiles
    (70, 300, 544, 32, True, True),       # INT8 outliers
    (64, 100, 256, 0, False, True),       # no outliers; N % 8 != 0
    (64, 256, 256, 256, True, True),      # everything is outlier
    (257, 513, 2080, 32, False, True),    # 3 x 3 tiles, long K
    (130, 260, 8256, 64, False, True),    # 64 k-blocks
    (33, 72, 20544, 64, True, True),      # the widest rows: sums past 2^24
    (5, 300, 640, 64, True, True),        # a few tokens
]


def _case_a8(M, N, K, k_o, int8, bias, seed, wb=4):
    cfg = wl.custom_config(M, N, K, k_o, 0, int8, bias, outlier_mult=30.0,
                           student_t=(seed % 2 == 1), act_bits=8, weight_bits=wb)
    return cfg, wl.make_layer(cfg, seed_offset=seed)


WB = [4, 8]  # INT4 weights (W4A8) and INT8 weights (W8A8)


@pytest.mark.parametrize("shape", SHAPES_A8, ids=[str(s) for s in SHAPES_A8])
def test_a8_quantize_bit_exact(shape):
    M, N, K, k_o, int8, bias = shape
    cfg, d = _case_a8(*shape, seed=7)
    gx = q.quantize_reorder(d["X"].to(DEV), d["perm"].to(DEV), k_o, 0, int8, act_bits=8)
    torch.cuda.synchronize()
    assert gx[0].dtype == torch.int8 and tuple(gx[0].shape) == (M, K - k_o)
    ref = oracle.quantize_rows(np16(d["X"]), d["perm"].numpy(), k_o, 0, int8, 8)
    assert_quant_equal(gpu_tuple_np(gx), ref, "X (INT8 codes)")


@pytest.mark.parametrize("wb", WB, ids=["w4a8", "w8a8"])
@pytest.mark.parametrize("shape", SHAPES_A8, ids=[str(s) for s in SHAPES_A8])
def test_a8_int32_sums_bit_exact(shape, wb):
    M, N, K, k_o, int8, bias = shape
    cfg, d = _case_a8(*shape, seed=11, wb=wb)
    perm_d = d["perm"].to(DEV)
    gx = q.quantize_reorder(d["X"].to(DEV), perm_d, k_o, 0, int8, act_bits=8)
    gw = q.pack_weights(d["W"].to(DEV), perm_d, k_o, 0, int8, weight_bits=wb)
    acc, acc_o = q.gemm_i32(gx[0], gw[0], K, k_o, 0, gx[2], gw[2])
    torch.cuda.synchronize()
    ox = oracle.quantize_rows(np16(d["X"]), d["perm"].numpy(), k_o, 0, int8, 8)
    ow = oracle.quantize_rows(np16(d["W"]), d["perm"].numpy(), k_o, 0, int8, wb)
    if wb == 8:  # the weights' INT8 codes and scales, bit-exact
        assert_quant_equal(gpu_tuple_np(gw), ow, "W (INT8 codes)")
    if K - k_o > 0:
        np.testing.assert_array_equal(acc.cpu().numpy(), oracle.int_gemm(ox[0], ow[0], 0))
    if int8 and k_o > 0:
        ref_o = ox[2].astype(np.int64) @ ow[2].astype(np.int64).T
        np.testing.assert_array_equal(acc_o.cpu().numpy(), ref_o)


@pytest.mark.parametrize("wb", WB, ids=["w4a8", "w8a8"])
@pytest.mark.parametrize("shape", SHAPES_A8, ids=[str(s) for s in SHAPES_A8])
def test_a8_linear_output_within_tolerance(shape, wb):
    M, N, K, k_o, int8, bias = shape
    cfg, d = _case_a8(*shape, seed=13, wb=wb)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, 0, int8, b, act_bits=8, weight_bits=wb)
    Y = layer(d["X"].to(DEV))
    gx = q.quantize_reorder(d["X"].to(DEV), perm_d, k_o, 0, int8, act_bits=8)
    Y2 = q.gemm(gx, (layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale), K, k_o, 0, b)
    torch.cuda.synchronize()
    ref = oracle.layer(np16(d["X"]), np16(d["W"]), d["perm"].numpy(),
                       None if d["bias"] is None else np16(d["bias"]), k_o, 0, int8, act_bits=8,
                       weight_bits=wb)["Y"]
    assert_y_close(Y.float().cpu().numpy(), ref, f"W{wb}A8 linear {shape}")
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))


def test_a8_grouped_is_unsupported():
    shape = q.make_shape(16, 256, 512, 0, 128, q.QUIK_OUTLIER_FP16, 8)
    X = torch.zeros((16, 512), dtype=torch.float16, device=DEV)
    perm = torch.arange(512, dtype=torch.int32, device=DEV)
    Xq = torch.empty((16, 512), dtype=torch.int8, device=DEV)
    sx = torch.empty((16, 4), dtype=torch.float32, device=DEV)
    with pytest.raises(q.QuikError) as e:
        q.quik_quantize_reorder(shape, X, perm, Xq, sx, None, None)
    assert e.value.status == q.QUIK_ERR_UNSUPPORTED


def test_w8_without_a8_is_unsupported():
    shape = q.make_shape(16, 256, 256, 0, 0, q.QUIK_OUTLIER_FP16, 4, 8)
    W = torch.zeros((256, 256), dtype=torch.float16, device=DEV)
    perm = torch.arange(256, dtype=torch.int32, device=DEV)
    Wq = torch.empty((256, 256), dtype=torch.int8, device=DEV)
    sw = torch.empty((256,), dtype=torch.float32, device=DEV)
    with pytest.raises(q.QuikError) as e:
        q.quik_pack_weights(shape, W, perm, Wq, sw, None, None)
    assert e.value.status == q.QUIK_ERR_UNSUPPORTED


@pytest.mark.parametrize("shape", [(257, 513, 2080, 32, 0, False, True),
                                   (16, 256, 256, 32, 0, False, True)])
def test_linear_timed_is_linear(shape):
    """quik_linear_timed (an event between the layer's two kernels) writes
    the same Y as quik_linear, bit for bit, and its event falls between the
    events around the call."""
    M, N, K, k_o, group, int8, bias = shape
    cfg, d = _case(*shape, seed=17)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    X = d["X"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, group, int8, b)
    Y = layer(X)
    shape_s = layer.shape(M)
    ws = torch.empty(q.quik_workspace_size(shape_s), dtype=torch.uint8, device=DEV)
    Y2 = torch.full_like(Y, float("nan"))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    q.quik_linear_timed(shape_s, X, perm_d, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale, b,
                        Y2, ws, ev[1])
    ev[2].record()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))
    assert ev[0].elapsed_time(ev[1]) > 0 and ev[1].elapsed_time(ev[2]) > 0


@pytest.mark.parametrize("site,shape", [(1, (64, 256, 512, 64)), (2, (257, 513, 2080, 32))],
                         ids=["quantiser", "persistent-gemm"])
def test_production_kernel_timeout_path(site, shape):
    """quik_test_stall: a production kernel (1: the quantiser's row wait, 2:
    the persistent GEMM's MMA issuer) first waits on a barrier that nothing
    completes.  The bounded wait runs out (2 s), the kernel leaves through
    its abort path without a fault, quik_sync_check reports
    QUIK_ERR_TIMEOUT once, and the next layer call is correct (bit-identical
    to the one before the stall)."""
    M, N, K, k_o = shape
    cfg, d = _case(M, N, K, k_o, 0, False, True, seed=21)
    perm_d = d["perm"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, 0, False, d["bias"].to(DEV))
    X = d["X"].to(DEV)
    Y_ref = layer(X)
    torch.cuda.synchronize()
    assert q.quik_sync_check() == q.QUIK_OK
    q.quik_test_stall(site)
    try:
        layer(X)
        torch.cuda.synchronize()
    finally:
        q.quik_test_stall(0)
    assert q.quik_sync_check() == q.QUIK_ERR_TIMEOUT
    assert q.quik_sync_check() == q.QUIK_OK
    Y = layer(X)
    torch.cuda.synchronize()
    assert q.quik_sync_check() == q.QUIK_OK
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y_ref.cpu().numpy().view(np.uint16))


# the layer calls the canary and self-checking tests run: (M, N, K, k_o, group, int8 outliers, act bits)
GUARDED = [
    (130, 300, 640, 64, 0, False, 4),     # persistent GEMM (packed X through quik_gemm; widened in the layer)
    (16, 520, 1056, 32, 0, False, 4),     # decode kernel
    (70, 300, 544, 32, 0, True, 4),       # pair kernel with INT8 outliers
    (150, 260, 1152, 128, 128, True, 4),  # grouped scales
    (200, 300, 640, 64, 0, False, 8),     # W4A8
]


@pytest.mark.parametrize("shape", GUARDED, ids=[str(s) for s in GUARDED])
def test_canary_guards_untouched_every_kernel(shape):
    """Guard bytes around the workspace and Y of a layer call, and around
    the outputs of the two-call path, stay untouched on every GEMM kernel
    (persistent, decode, pair, grouped, W4A8) and the quantiser."""
    M, N, K, k_o, group, int8, ab = shape
    cfg = wl.custom_config(M, N, K, k_o, group, int8, True, outlier_mult=30.0, act_bits=ab)
    d = wl.make_layer(cfg, seed_offset=3)
    G, pat = 4096, 0xA5

    def guarded(nbytes):
        buf = torch.full((G + nbytes + G,), pat, dtype=torch.uint8, device=DEV)
        return buf, buf[G:G + nbytes]

    perm_d = d["perm"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, group, int8, d["bias"].to(DEV), act_bits=ab)
    s = layer.shape(M)
    bw, ws = guarded(q.quik_workspace_size(s))
    by, Yb = guarded(M * N * 2)
    q.quik_linear(s, d["X"].to(DEV), perm_d, layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale,
                  d["bias"].to(DEV), Yb.view(torch.float16).view(M, N), ws)
    torch.cuda.synchronize()
    assert q.quik_sync_check() == q.QUIK_OK
    for buf in (bw, by):
        h = buf.cpu().numpy()
        assert (h[:G] == pat).all() and (h[-G:] == pat).all()


def test_sparse24_canary_guards_untouched():
    """The same for the 2:4 layer, at decode (sparse kernel) and prefill
    (expanded weights) token counts."""
    for M in (16, 130):
        cfg = wl.custom_config(M, 264, 1088, 64, 0, False, True, outlier_mult=30.0)
        d = wl.make_layer(cfg, seed_offset=4)
        G, pat = 4096, 0xA5
        perm_d = d["perm"].to(DEV)
        layer = q.QuikLinear24(d["W"].to(DEV), perm_d, 64, False, d["bias"].to(DEV))
        s = layer.shape(M)
        buf_w = torch.full((G + q.quik_workspace_size_24(s) + G,), pat, dtype=torch.uint8, device=DEV)
        buf_y = torch.full((G + M * 264 * 2 + G,), pat, dtype=torch.uint8, device=DEV)
        ws = buf_w[G:G + q.quik_workspace_size_24(s)]
        Yb = buf_y[G:G + M * 264 * 2].view(torch.float16).view(M, 264)
        q.quik_linear_24(s, d["X"].to(DEV), perm_d, layer.Wq24, layer.Wmeta, layer.w_scale, layer.Wo,
                         layer.wo_scale, d["bias"].to(DEV), Yb, ws)
        torch.cuda.synchronize()
        assert q.quik_sync_check() == q.QUIK_OK
        for b in (buf_w, buf_y):
            h = b.cpu().numpy()
            assert (h[:G] == pat).all() and (h[-G:] == pat).all(), M


_CHECKED_CHILD = r'''
import ctypes, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
import mixed_precision_quantized_quantize_b200._binding as B
B.LIB_PATH = sys.argv[2]
import mixed_precision_quantized_quantize_b200 as q
from mixed_precision_quantized_quantize_b200 import workloads as wl
out = {}
for i, (M, N, K, k_o, group, int8, ab) in enumerate(eval(sys.argv[3])):
    cfg = wl.custom_config(M, N, K, k_o, group, int8, True, outlier_mult=30.0, act_bits=ab)
    d = wl.make_layer(cfg, seed_offset=9)
    layer = q.QuikLinear(d["W"].cuda(), d["perm"].cuda(), k_o, group, int8, d["bias"].cuda(), act_bits=ab)
    out[f"y{i}"] = layer(d["X"].cuda()).cpu().numpy().view(np.uint16)
torch.cuda.synchronize()
L = q.lib()
for f in ("qchk_quantize_word", "qchk_gemm_word"):
    getattr(L, f).restype = ctypes.c_ulonglong
out["words"] = np.array([L.qchk_quantize_word(), L.qchk_gemm_word(), L.quik_sync_check(None)], np.uint64)
np.savez(sys.argv[4], **out)
'''


def test_self_checking_build_matches(tmp_path):
    """The self-checking build (-DQUIK_CHECKS: computed indices and
    alignments checked, the first violation recorded and the access
    skipped) runs the layer on every GEMM kernel with no violation and the
    same outputs, bit for bit, as the normal build (in a child process: one
    copy of the library per process)."""
    import os
    import subprocess
    import sys
    from mixed_precision_quantized_quantize_b200 import build as qbuild
    checked = qbuild.build(checks=True)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    npz = str(tmp_path / "checked.npz")
    subprocess.run([sys.executable, "-c", _CHECKED_CHILD, root, checked, repr(GUARDED), npz],
                   check=True, timeout=600)
    got = np.load(npz)
    assert got["words"].tolist() == [0, 0, q.QUIK_OK], got["words"]
    for i, (M, N, K, k_o, group, int8, ab) in enumerate(GUARDED):
        cfg = wl.custom_config(M, N, K, k_o, group, int8, True, outlier_mult=30.0, act_bits=ab)
        d = wl.make_layer(cfg, seed_offset=9)
        layer = q.QuikLinear(d["W"].to(DEV), d["perm"].to(DEV), k_o, group, int8, d["bias"].to(DEV),
                             act_bits=ab)
        y = layer(d["X"].to(DEV)).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(y, got[f"y{i}"], err_msg=str(GUARDED[i]))


# shapes whose layer call takes the 512-token tiles (two 256-token halves per
# widened weight unit): ragged tokens and channels, FP16 outliers or none,
# TMA or plain output stores
TWO_HALVES = [
    (1100, 4000, 1056, 32, True),   # 3 token tiles of 512 (the last one ragged), 16 weight tiles
    (1100, 4100, 1088, 0, False),   # no outliers; N % 8 != 0 (plain stores), a ragged weight tile
    (1536, 4096, 2176, 192, True),  # three outlier units (the most this form takes)
]


@pytest.mark.parametrize("shape", TWO_HALVES, ids=[str(s) for s in TWO_HALVES])
def test_two_halves_layer(shape):
    """The layer call on shapes that take the 512-token persistent tiles:
    every output against the oracle's fp64 layer, and bit-identical to the
    two-call path (quik_quantize_reorder + quik_gemm, 256-token tiles on the
    packed codes)."""
    M, N, K, k_o, bias = shape
    cfg, d = _case(M, N, K, k_o, 0, False, bias, seed=31)
    perm_d = d["perm"].to(DEV)
    b = d["bias"].to(DEV) if d["bias"] is not None else None
    X = d["X"].to(DEV)
    layer = q.QuikLinear(d["W"].to(DEV), perm_d, k_o, 0, False, b)
    Y = layer(X)
    gx = q.quantize_reorder(X, perm_d, k_o, 0, False)
    Y2 = q.gemm(gx, (layer.Wq, layer.w_scale, layer.Wo, layer.wo_scale), K, k_o, 0, b)
    torch.cuda.synchronize()
    assert q.quik_sync_check() == q.QUIK_OK
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))
    ref = oracle.layer(np16(d["X"]), np16(d["W"]), d["perm"].numpy(),
                       None if d["bias"] is None else np16(d["bias"]), k_o, 0, False)["Y"]
    assert_y_close(Y.float().cpu().numpy(), ref, f"two halves {shape}")
