"""Python handle on the CPU oracle (``quik_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this module, and this module imports nothing from the product.

Arrays cross the boundary as numpy arrays; fp16 data is passed as its uint16
bit pattern so that no conversion happens on the Python side.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "quik_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fno-fast-math",
                               "-ffp-contract=off", "-Wall", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        _C = ctypes.c_int
        lib.oracle_quantize_rows.argtypes = [_I, _I, _I, _I, _C, _C, _P, _P, _P, _P, _P, _P]
        lib.oracle_rmsnorm_quantize_rows.argtypes = [_I, _I, _I, _I, _C, _C, _P, _P,
                                                     ctypes.c_float, _P, _P, _P, _P, _P]
        lib.oracle_prune24_quantize_rows.argtypes = [_I, _I, _I, _C, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_unpack24.argtypes = [_I, _I, _P, _P, _P]
        lib.oracle_int_gemm.argtypes = [_I, _I, _I, _I, _C, _C, _P, _P, _P]
        lib.oracle_linear.argtypes = [_I, _I, _I, _I, _I, _C, _C, _C,
                                      _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_linear_sampled.argtypes = [_I, _I, _I, _I, _I, _C, _C, _C,
                                              _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                              _I, _P, _P, _P, _P]
        lib.oracle_num_threads.argtypes = []
        for f in (lib.oracle_quantize_rows, lib.oracle_rmsnorm_quantize_rows,
                  lib.oracle_prune24_quantize_rows, lib.oracle_unpack24,
                  lib.oracle_int_gemm, lib.oracle_linear,
                  lib.oracle_linear_sampled, lib.oracle_num_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def quantize_rows(X_f16: np.ndarray, perm: np.ndarray, k_o: int, group: int = 0,
                  outlier_int8: bool = False, bits: int = 4):
    """Reorder + quantise (+ pack) the rows of ``X_f16`` ([R, K] float16).

    Returns (Q, scale float32 [R] or [R,G], O float16 or int8 [R,k_o],
             o_scale float32 [R] or None); Q is uint8 [R,(K-k_o)/2] packed INT4
    (bits 4) or int8 [R,K-k_o] (bits 8).
    """
    X = np.ascontiguousarray(X_f16, dtype=np.float16)
    R, K = X.shape
    Ki = K - k_o
    G = Ki // group if group else 1
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    Q = np.zeros((R, Ki), np.int8) if bits == 8 else np.zeros((R, Ki // 2), np.uint8)
    scale = np.zeros((R, G) if group else (R,), np.float32)
    O = np.zeros((R, k_o), np.int8 if outlier_int8 else np.float16)
    o_scale = np.zeros((R,), np.float32) if outlier_int8 else None
    rc = _load().oracle_quantize_rows(R, K, k_o, group, int(outlier_int8), int(bits),
                                      _ptr(X.view(np.uint16)), _ptr(perm), _ptr(Q),
                                      _ptr(scale), _ptr(O), _ptr(o_scale))
    _check(rc, "quantize_rows")
    return Q, scale, O, o_scale


def rmsnorm_quantize_rows(X_f16: np.ndarray, gamma_f16: np.ndarray, eps: float,
                          perm: np.ndarray, k_o: int, group: int = 0,
                          outlier_int8: bool = False, bits: int = 4):
    """RMS-normalise each row of ``X_f16`` ([R, K] float16) with weight
    ``gamma_f16`` ([K], source channel order) and ``eps``, then reorder and
    quantise it ("Atom", idea I2: quantisation fused into the norm).

    Codes and base scales are those of z = X * gamma; the row factor
    r = 1/sqrt(mean(X^2) + eps) (fp64; eps is taken as fp32, the type of the
    norm's parameter) multiplies the stored scales, and FP16 outliers are
    fl16(z * r).  Returns the tuple of ``quantize_rows``.
    """
    X = np.ascontiguousarray(X_f16, dtype=np.float16)
    g = np.ascontiguousarray(gamma_f16, dtype=np.float16)
    R, K = X.shape
    assert g.shape == (K,)
    Ki = K - k_o
    G = Ki // group if group else 1
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    Q = np.zeros((R, Ki), np.int8) if bits == 8 else np.zeros((R, Ki // 2), np.uint8)
    scale = np.zeros((R, G) if group else (R,), np.float32)
    O = np.zeros((R, k_o), np.int8 if outlier_int8 else np.float16)
    o_scale = np.zeros((R,), np.float32) if outlier_int8 else None
    rc = _load().oracle_rmsnorm_quantize_rows(R, K, k_o, group, int(outlier_int8), int(bits),
                                              _ptr(X.view(np.uint16)), _ptr(g.view(np.uint16)),
                                              float(eps), _ptr(perm), _ptr(Q), _ptr(scale),
                                              _ptr(O), _ptr(o_scale))
    _check(rc, "rmsnorm_quantize_rows")
    return Q, scale, O, o_scale


def prune24_quantize_rows(W_f16: np.ndarray, perm: np.ndarray, k_o: int,
                          outlier_int8: bool = False):
    """2:4-sparse INT4 rows (QUIK abstract: quantisation plus 2:4 sparsity):
    each aligned group of four reordered INT4 positions keeps its two values of
    largest magnitude (lower position on ties), then the usual quantiser.

    Returns (Qs uint8 [R, K_i/4] two kept codes per byte, meta uint8
    [R, K_i/8] one nibble i0 | i1 << 2 per group, scale float32 [R],
    O, o_scale as quantize_rows).
    """
    X = np.ascontiguousarray(W_f16, dtype=np.float16)
    R, K = X.shape
    Ki = K - k_o
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    Qs = np.zeros((R, Ki // 4), np.uint8)
    meta = np.zeros((R, Ki // 8), np.uint8)
    scale = np.zeros((R,), np.float32)
    O = np.zeros((R, k_o), np.int8 if outlier_int8 else np.float16)
    o_scale = np.zeros((R,), np.float32) if outlier_int8 else None
    rc = _load().oracle_prune24_quantize_rows(R, K, k_o, int(outlier_int8),
                                              _ptr(X.view(np.uint16)), _ptr(perm), _ptr(Qs),
                                              _ptr(meta), _ptr(scale), _ptr(O), _ptr(o_scale))
    _check(rc, "prune24_quantize_rows")
    return Qs, meta, scale, O, o_scale


def unpack24(Qs: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """Dense packed INT4 rows [R, K_i/2] that 2:4 rows (Qs, meta) stand for."""
    Qs = np.ascontiguousarray(Qs, np.uint8)
    meta = np.ascontiguousarray(meta, np.uint8)
    R, Ki = Qs.shape[0], 4 * Qs.shape[1]
    Q = np.zeros((R, Ki // 2), np.uint8)
    _check(_load().oracle_unpack24(R, Ki, _ptr(Qs), _ptr(meta), _ptr(Q)), "unpack24")
    return Q


def _x_bits(Q) -> int:
    """8 for one signed byte per code (int8 array), 4 for packed nibbles."""
    return 8 if Q.dtype == np.int8 else 4


def int_gemm(Xq: np.ndarray, Wq: np.ndarray, group: int = 0) -> np.ndarray:
    """Exact INT32 sums of the codes (each operand packed INT4 uint8, or int8
    codes): [M,N], or [G,M,N] with groups."""
    xb, wb = _x_bits(Xq), _x_bits(Wq)
    Xq = np.ascontiguousarray(Xq.view(np.uint8))
    Wq = np.ascontiguousarray(Wq.view(np.uint8))
    M = Xq.shape[0]
    N = Wq.shape[0]
    Ki = Wq.shape[1] if wb == 8 else 2 * Wq.shape[1]
    G = Ki // group if group else 1
    acc = np.zeros((G, M, N), np.int32)
    _check(_load().oracle_int_gemm(M, N, Ki, group, xb, wb, _ptr(Xq), _ptr(Wq), _ptr(acc)),
           "int_gemm")
    return acc if group else acc[0]


def _linear_args(Xq, sx, Xo, sxo, Wq, sw, Wo, swo, bias):
    c = np.ascontiguousarray
    Xq, Wq = c(Xq.view(np.uint8)), c(Wq.view(np.uint8))
    sx, sw = c(sx, np.float32), c(sw, np.float32)
    int8 = Xo is not None and Xo.dtype == np.int8
    if Xo is not None:
        Xo = c(Xo.view(np.uint16)) if Xo.dtype == np.float16 else c(Xo, np.int8)
        Wo = c(Wo.view(np.uint16)) if Wo.dtype == np.float16 else c(Wo, np.int8)
    sxo = None if sxo is None else c(sxo, np.float32)
    swo = None if swo is None else c(swo, np.float32)
    b = None if bias is None else c(np.asarray(bias, np.float16).view(np.uint16))
    return Xq, sx, Xo, sxo, Wq, sw, Wo, swo, b, int8


def linear(Xq, sx, Xo, sxo, Wq, sw, Wo, swo, bias, K: int, k_o: int, group: int = 0):
    """fp64 Y [M,N] of the layer from quantised operands (no fp16 rounding)."""
    xb, wb = _x_bits(Xq), _x_bits(Wq)
    Xq, sx, Xo, sxo, Wq, sw, Wo, swo, b, int8 = _linear_args(Xq, sx, Xo, sxo, Wq, sw, Wo, swo, bias)
    M, N = Xq.shape[0], Wq.shape[0]
    Y = np.zeros((M, N), np.float64)
    rc = _load().oracle_linear(M, N, K, k_o, group, int(int8), xb, wb, _ptr(Xq), _ptr(sx), _ptr(Xo),
                               _ptr(sxo), _ptr(Wq), _ptr(sw), _ptr(Wo), _ptr(swo), _ptr(b), _ptr(Y))
    _check(rc, "linear")
    return Y


def linear_sampled(Xq, sx, Xo, sxo, Wq, sw, Wo, swo, bias, K: int, k_o: int, group: int,
                   ms: np.ndarray, ns: np.ndarray):
    """fp64 Y at the (ms[i], ns[i]) positions plus their integer sums [count, G]."""
    xb, wb = _x_bits(Xq), _x_bits(Wq)
    Xq, sx, Xo, sxo, Wq, sw, Wo, swo, b, int8 = _linear_args(Xq, sx, Xo, sxo, Wq, sw, Wo, swo, bias)
    M, N = Xq.shape[0], Wq.shape[0]
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    G = (K - k_o) // group if group else 1
    Y = np.zeros(len(ms), np.float64)
    acc = np.zeros((len(ms), max(G, 1)), np.int32)
    rc = _load().oracle_linear_sampled(M, N, K, k_o, group, int(int8), xb, wb, _ptr(Xq), _ptr(sx),
                                       _ptr(Xo), _ptr(sxo), _ptr(Wq), _ptr(sw), _ptr(Wo),
                                       _ptr(swo), _ptr(b), len(ms), _ptr(ms), _ptr(ns),
                                       _ptr(Y), _ptr(acc))
    _check(rc, "linear_sampled")
    return Y, acc


def layer(X_f16, W_f16, perm, bias, k_o: int, group: int = 0, outlier_int8: bool = False,
          act_bits: int = 4, weight_bits: int = 4):
    """The whole layer from fp16 inputs: quantise X and W (INT4, or INT8 when
    act_bits / weight_bits == 8), then the fp64 output.

    Returns a dict with every intermediate (codes, scales, outlier blocks, Y).
    """
    K = X_f16.shape[1]
    Xq, sx, Xo, sxo = quantize_rows(X_f16, perm, k_o, group, outlier_int8, act_bits)
    Wq, sw, Wo, swo = quantize_rows(W_f16, perm, k_o, group, outlier_int8, weight_bits)
    Y = linear(Xq, sx, Xo if k_o else None, sxo, Wq, sw, Wo if k_o else None, swo, bias,
               K, k_o, group)
    return dict(Xq=Xq, sx=sx, Xo=Xo, sxo=sxo, Wq=Wq, sw=sw, Wo=Wo, swo=swo, Y=Y)


def rmsnorm_layer(X_f16, gamma_f16, eps, W_f16, perm, bias, k_o: int, group: int = 0,
                  outlier_int8: bool = False, act_bits: int = 4, weight_bits: int = 4):
    """The layer behind an RMS norm: ``rmsnorm_quantize_rows`` on the
    activations, ``quantize_rows`` on the weights, then the fp64 output."""
    K = X_f16.shape[1]
    Xq, sx, Xo, sxo = rmsnorm_quantize_rows(X_f16, gamma_f16, eps, perm, k_o, group,
                                            outlier_int8, act_bits)
    Wq, sw, Wo, swo = quantize_rows(W_f16, perm, k_o, group, outlier_int8, weight_bits)
    Y = linear(Xq, sx, Xo if k_o else None, sxo, Wq, sw, Wo if k_o else None, swo, bias,
               K, k_o, group)
    return dict(Xq=Xq, sx=sx, Xo=Xo, sxo=sxo, Wq=Wq, sw=sw, Wo=Wo, swo=swo, Y=Y)
