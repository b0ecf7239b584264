"""ctypes binding of libquik_b200.so (the C ABI in include/quik.h).

Argument marshalling only: every function below checks dtypes / devices,
turns torch tensors into device pointers and calls the C entry point of the
same name on the current CUDA stream.  Convenience helpers allocate the
output tensors with torch (device memory is PyTorch's job here); all
arithmetic runs in the library's kernels.  There is no CPU fallback: if the
library is missing, or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QUIK_LIBRARY may name another build of the same library (e.g. the
# self-checking variant libquik_b200_checked.so); default: the in-tree build.
LIB_PATH = os.environ.get("QUIK_LIBRARY") or os.path.join(_HERE, "libquik_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "quik.h")

QUIK_OK, QUIK_ERR_INVALID_ARG, QUIK_ERR_UNSUPPORTED, QUIK_ERR_CUDA, QUIK_ERR_TIMEOUT = range(5)
QUIK_OUTLIER_FP16, QUIK_OUTLIER_INT8 = 0, 1
GROUP = 128


class QuikError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class quik_shape(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("k_o", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("outlier", ctypes.c_int32), ("act_bits", ctypes.c_int32),
                ("weight_bits", ctypes.c_int32)]


_P = ctypes.c_void_p
_S = ctypes.POINTER(quik_shape)
_SIGS = {
    "quik_workspace_size": (ctypes.c_size_t, [_S]),
    "quik_quantize_reorder": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P]),
    "quik_rmsnorm_quantize_reorder": (ctypes.c_int, [_S, _P, _P, ctypes.c_float, _P, _P, _P, _P,
                                                      _P, _P]),
    "quik_pack_weights": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P]),
    "quik_gemm": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "quik_linear": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "quik_rmsnorm_linear": (ctypes.c_int, [_S, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P, _P,
                                            _P, _P, ctypes.c_size_t, _P]),
    "quik_linear_noalloc": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "quik_linear_timed": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                         _P, _P]),
    "quik_gemm_i32_debug": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P]),
    "quik_pack_weights_24": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P]),
    "quik_gemm_24": (ctypes.c_int, [_S] + [_P] * 12),
    "quik_linear_24": (ctypes.c_int, [_S] + [_P] * 10 + [ctypes.c_size_t, _P]),
    "quik_gemm_24_i32_debug": (ctypes.c_int, [_S] + [_P] * 8),
    "quik_expand_weights_24": (ctypes.c_int, [_S, _P, _P, _P, _P]),
    "quik_workspace_size_24": (ctypes.c_size_t, [_S]),
    "quik_sync_check": (ctypes.c_int, [_P]),
    "quik_selftest_timeout": (ctypes.c_int, [ctypes.c_uint32, _P]),
    "quik_test_stall": (ctypes.c_int, [ctypes.c_int]),
    "quik_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}
_lib = None


def header_functions() -> list[str]:
    """Names of the functions include/quik.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(quik_[a-z0-9_]+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixed_precision_quantized_quantize_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().quik_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != QUIK_OK:
        raise QuikError(status, what)


def make_shape(M: int, N: int, K: int, k_o: int, group_size: int = 0,
               outlier: int = QUIK_OUTLIER_FP16, act_bits: int = 4,
               weight_bits: int = 4) -> quik_shape:
    return quik_shape(M, N, K, k_o, group_size, outlier, act_bits, weight_bits)


def _ptr(t, dtype=None, what="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{what} must live on a CUDA device")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t.data_ptr() if t.numel() > 0 else None


def _xq_dtype(shape: quik_shape):
    """Quantised activations: packed INT4 bytes, or INT8 codes when act_bits == 8."""
    return torch.int8 if shape.act_bits == 8 else torch.uint8


def _wq_dtype(shape: quik_shape):
    """Packed weights: INT4 bytes, or INT8 codes when weight_bits == 8."""
    return torch.int8 if shape.weight_bits == 8 else torch.uint8


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ------------------------------------------------------------------ raw entry points
def quik_workspace_size(shape: quik_shape) -> int:
    return int(lib().quik_workspace_size(ctypes.byref(shape)))


def quik_quantize_reorder(shape, X, perm, Xq, x_scale, Xo, xo_scale, stream=None):
    _check(lib().quik_quantize_reorder(
        ctypes.byref(shape), _ptr(X, torch.float16, "X"), _ptr(perm, torch.int32, "perm"),
        _ptr(Xq, _xq_dtype(shape), "Xq"), _ptr(x_scale, torch.float32, "x_scale"), _ptr(Xo, None, "Xo"),
        _ptr(xo_scale, torch.float32, "xo_scale"), _stream(stream)), "quik_quantize_reorder")


def quik_rmsnorm_quantize_reorder(shape, X, gamma, eps, perm, Xq, x_scale, Xo, xo_scale,
                                  stream=None):
    _check(lib().quik_rmsnorm_quantize_reorder(
        ctypes.byref(shape), _ptr(X, torch.float16, "X"), _ptr(gamma, torch.float16, "gamma"),
        float(eps), _ptr(perm, torch.int32, "perm"), _ptr(Xq, _xq_dtype(shape), "Xq"),
        _ptr(x_scale, torch.float32, "x_scale"), _ptr(Xo, None, "Xo"),
        _ptr(xo_scale, torch.float32, "xo_scale"), _stream(stream)),
        "quik_rmsnorm_quantize_reorder")


def quik_pack_weights(shape, W, perm, Wq, w_scale, Wo, wo_scale, stream=None):
    _check(lib().quik_pack_weights(
        ctypes.byref(shape), _ptr(W, torch.float16, "W"), _ptr(perm, torch.int32, "perm"),
        _ptr(Wq, _wq_dtype(shape), "Wq"), _ptr(w_scale, torch.float32, "w_scale"), _ptr(Wo, None, "Wo"),
        _ptr(wo_scale, torch.float32, "wo_scale"), _stream(stream)), "quik_pack_weights")


def quik_gemm(shape, Xq, x_scale, Xo, xo_scale, Wq, w_scale, Wo, wo_scale, bias, Y, stream=None):
    _check(lib().quik_gemm(
        ctypes.byref(shape), _ptr(Xq, _xq_dtype(shape), "Xq"), _ptr(x_scale, torch.float32, "x_scale"),
        _ptr(Xo, None, "Xo"), _ptr(xo_scale, torch.float32, "xo_scale"),
        _ptr(Wq, _wq_dtype(shape), "Wq"), _ptr(w_scale, torch.float32, "w_scale"),
        _ptr(Wo, None, "Wo"), _ptr(wo_scale, torch.float32, "wo_scale"),
        _ptr(bias, torch.float16, "bias"), _ptr(Y, torch.float16, "Y"), _stream(stream)), "quik_gemm")


def quik_linear(shape, X, perm, Wq, w_scale, Wo, wo_scale, bias, Y, workspace, stream=None):
    _check(lib().quik_linear(
        ctypes.byref(shape), _ptr(X, torch.float16, "X"), _ptr(perm, torch.int32, "perm"),
        _ptr(Wq, _wq_dtype(shape), "Wq"), _ptr(w_scale, torch.float32, "w_scale"),
        _ptr(Wo, None, "Wo"), _ptr(wo_scale, torch.float32, "wo_scale"),
        _ptr(bias, torch.float16, "bias"), _ptr(Y, torch.float16, "Y"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)), "quik_linear")


def quik_linear_timed(shape, X, perm, Wq, w_scale, Wo, wo_scale, bias, Y, workspace, between,
                      stream=None):
    """quik_linear with the torch.cuda.Event `between` recorded between its two
    kernels (the GEMM then waits for the quantiser to finish)."""
    if between.cuda_event == 0:
        between.record(stream)  # torch creates the CUDA event on its first record
    _check(lib().quik_linear_timed(
        ctypes.byref(shape), _ptr(X, torch.float16, "X"), _ptr(perm, torch.int32, "perm"),
        _ptr(Wq, _wq_dtype(shape), "Wq"), _ptr(w_scale, torch.float32, "w_scale"),
        _ptr(Wo, None, "Wo"), _ptr(wo_scale, torch.float32, "wo_scale"),
        _ptr(bias, torch.float16, "bias"), _ptr(Y, torch.float16, "Y"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), between.cuda_event,
        _stream(stream)), "quik_linear_timed")


def quik_rmsnorm_linear(shape, X, gamma, eps, perm, Wq, w_scale, Wo, wo_scale, bias, Y, workspace,
                        stream=None):
    _check(lib().quik_rmsnorm_linear(
        ctypes.byref(shape), _ptr(X, torch.float16, "X"), _ptr(gamma, torch.float16, "gamma"),
        float(eps), _ptr(perm, torch.int32, "perm"),
        _ptr(Wq, _wq_dtype(shape), "Wq"), _ptr(w_scale, torch.float32, "w_scale"),
        _ptr(Wo, None, "Wo"), _ptr(wo_scale, torch.float32, "wo_scale"),
        _ptr(bias, torch.float16, "bias"), _ptr(Y, torch.float16, "Y"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "quik_rmsnorm_linear")


def quik_linear_noalloc(shape, X, perm, Wq, w_scale, Wo, wo_scale, bias, Y, stream=None):
    """quik_linear on the library's own fixed workspace (for callers that cannot
    allocate device memory); see include/quik.h."""
    _check(lib().quik_linear_noalloc(
        ctypes.byref(shape), _ptr(X, torch.float16, "X"), _ptr(perm, torch.int32, "perm"),
        _ptr(Wq, _wq_dtype(shape), "Wq"), _ptr(w_scale, torch.float32, "w_scale"),
        _ptr(Wo, None, "Wo"), _ptr(wo_scale, torch.float32, "wo_scale"),
        _ptr(bias, torch.float16, "bias"), _ptr(Y, torch.float16, "Y"), _stream(stream)),
        "quik_linear_noalloc")


def quik_gemm_i32_debug(shape, Xq, Wq, Xo, Wo, acc, acc_outlier, stream=None):
    _check(lib().quik_gemm_i32_debug(
        ctypes.byref(shape), _ptr(Xq, _xq_dtype(shape), "Xq"), _ptr(Wq, _wq_dtype(shape), "Wq"),
        _ptr(Xo, None, "Xo"), _ptr(Wo, None, "Wo"), _ptr(acc, torch.int32, "acc"),
        _ptr(acc_outlier, torch.int32, "acc_outlier"), _stream(stream)), "quik_gemm_i32_debug")


def quik_pack_weights_24(shape, W, perm, Wq24, Wmeta, w_scale, Wo, wo_scale, stream=None):
    _check(lib().quik_pack_weights_24(
        ctypes.byref(shape), _ptr(W, torch.float16, "W"), _ptr(perm, torch.int32, "perm"),
        _ptr(Wq24, torch.uint8, "Wq24"), _ptr(Wmeta, torch.uint8, "Wmeta"),
        _ptr(w_scale, torch.float32, "w_scale"), _ptr(Wo, None, "Wo"),
        _ptr(wo_scale, torch.float32, "wo_scale"), _stream(stream)), "quik_pack_weights_24")


def quik_gemm_24(shape, Xq, x_scale, Xo, xo_scale, Wq24, Wmeta, w_scale, Wo, wo_scale, bias, Y,
                 stream=None):
    _check(lib().quik_gemm_24(
        ctypes.byref(shape), _ptr(Xq, torch.uint8, "Xq"), _ptr(x_scale, torch.float32, "x_scale"),
        _ptr(Xo, None, "Xo"), _ptr(xo_scale, torch.float32, "xo_scale"),
        _ptr(Wq24, torch.uint8, "Wq24"), _ptr(Wmeta, torch.uint8, "Wmeta"),
        _ptr(w_scale, torch.float32, "w_scale"), _ptr(Wo, None, "Wo"),
        _ptr(wo_scale, torch.float32, "wo_scale"), _ptr(bias, torch.float16, "bias"),
        _ptr(Y, torch.float16, "Y"), _stream(stream)), "quik_gemm_24")


def quik_linear_24(shape, X, perm, Wq24, Wmeta, w_scale, Wo, wo_scale, bias, Y, workspace,
                   stream=None):
    _check(lib().quik_linear_24(
        ctypes.byref(shape), _ptr(X, torch.float16, "X"), _ptr(perm, torch.int32, "perm"),
        _ptr(Wq24, torch.uint8, "Wq24"), _ptr(Wmeta, torch.uint8, "Wmeta"),
        _ptr(w_scale, torch.float32, "w_scale"), _ptr(Wo, None, "Wo"),
        _ptr(wo_scale, torch.float32, "wo_scale"), _ptr(bias, torch.float16, "bias"),
        _ptr(Y, torch.float16, "Y"), _ptr(workspace, torch.uint8, "workspace"), workspace.numel(),
        _stream(stream)), "quik_linear_24")


def quik_gemm_24_i32_debug(shape, Xq, Wq24, Wmeta, Xo, Wo, acc, acc_outlier, stream=None):
    _check(lib().quik_gemm_24_i32_debug(
        ctypes.byref(shape), _ptr(Xq, torch.uint8, "Xq"), _ptr(Wq24, torch.uint8, "Wq24"),
        _ptr(Wmeta, torch.uint8, "Wmeta"), _ptr(Xo, None, "Xo"), _ptr(Wo, None, "Wo"),
        _ptr(acc, torch.int32, "acc"), _ptr(acc_outlier, torch.int32, "acc_outlier"),
        _stream(stream)), "quik_gemm_24_i32_debug")


def quik_expand_weights_24(shape, Wq24, Wmeta, Wq, stream=None):
    _check(lib().quik_expand_weights_24(
        ctypes.byref(shape), _ptr(Wq24, torch.uint8, "Wq24"), _ptr(Wmeta, torch.uint8, "Wmeta"),
        _ptr(Wq, torch.uint8, "Wq"), _stream(stream)), "quik_expand_weights_24")


def quik_workspace_size_24(shape: quik_shape) -> int:
    return int(lib().quik_workspace_size_24(ctypes.byref(shape)))


def quik_sync_check(stream=None) -> int:
    return int(lib().quik_sync_check(_stream(stream)))


def quik_test_stall(site: int):
    """Test entry: 1 stalls the quantiser's first row wait, 2 the persistent
    GEMM's MMA issuer (each then times out and reports QUIK_ERR_TIMEOUT);
    0 restores normal operation."""
    _check(lib().quik_test_stall(int(site)), "quik_test_stall")


def quik_selftest_timeout(limit_us: int, stream=None):
    _check(lib().quik_selftest_timeout(int(limit_us), _stream(stream)), "quik_selftest_timeout")


def quik_status_string(status: int) -> str:
    return status_string(status)


# ------------------------------------------------------------------ allocating helpers
def _outlier_kind(int8: bool) -> int:
    return QUIK_OUTLIER_INT8 if int8 else QUIK_OUTLIER_FP16


def _quant_outputs(rows: int, K: int, k_o: int, group: int, int8: bool, device, bits: int = 4):
    Ki = K - k_o
    G = Ki // group if group else 1
    Q = (torch.empty((rows, Ki), dtype=torch.int8, device=device) if bits == 8 else
         torch.empty((rows, Ki // 2), dtype=torch.uint8, device=device))
    scale = torch.empty((rows, G) if group else (rows,), dtype=torch.float32, device=device)
    O = torch.empty((rows, k_o), dtype=torch.int8 if int8 else torch.float16, device=device)
    o_scale = torch.empty((rows,), dtype=torch.float32, device=device) if int8 else None
    return Q, scale, O, o_scale


def quantize_reorder(X: torch.Tensor, perm: torch.Tensor, k_o: int, group: int = 0,
                     outlier_int8: bool = False, stream=None, act_bits: int = 4):
    """Activations -> (Xq, x_scale, Xo, xo_scale), allocated on X's device.
    Xq is packed INT4 (uint8 [M, K_i/2]), or int8 [M, K_i] when act_bits == 8."""
    M, K = X.shape
    shape = make_shape(M, 1, K, k_o, group, _outlier_kind(outlier_int8), act_bits)
    out = _quant_outputs(M, K, k_o, group, outlier_int8, X.device, act_bits)
    quik_quantize_reorder(shape, X, perm, *out, stream=stream)
    return out


def rmsnorm_quantize_reorder(X: torch.Tensor, gamma: torch.Tensor, eps: float, perm: torch.Tensor,
                             k_o: int, group: int = 0, outlier_int8: bool = False, stream=None,
                             act_bits: int = 4):
    """RMS norm (weight gamma [K], eps) fused with quantize_reorder: the hidden
    state X -> (Xq, x_scale, Xo, xo_scale) of the normalised rows."""
    M, K = X.shape
    shape = make_shape(M, 1, K, k_o, group, _outlier_kind(outlier_int8), act_bits)
    out = _quant_outputs(M, K, k_o, group, outlier_int8, X.device, act_bits)
    quik_rmsnorm_quantize_reorder(shape, X, gamma, eps, perm, *out, stream=stream)
    return out


def pack_weights(W: torch.Tensor, perm: torch.Tensor, k_o: int, group: int = 0,
                 outlier_int8: bool = False, stream=None, weight_bits: int = 4):
    """Weights -> (Wq, w_scale, Wo, wo_scale), allocated on W's device.
    Wq is packed INT4 (uint8 [N, K_i/2]), or int8 [N, K_i] when weight_bits == 8."""
    N, K = W.shape
    shape = make_shape(1, N, K, k_o, group, _outlier_kind(outlier_int8),
                       8 if weight_bits == 8 else 4, weight_bits)
    out = _quant_outputs(N, K, k_o, group, outlier_int8, W.device, weight_bits)
    quik_pack_weights(shape, W, perm, *out, stream=stream)
    return out


def gemm(xq, wq, K: int, k_o: int, group: int = 0, bias=None, stream=None):
    """Y fp16 [M, N] from quantised activations xq and packed weights wq (4-tuples)."""
    Xq, sx, Xo, sxo = xq
    Wq, sw, Wo, swo = wq
    M, N = sx.shape[0], sw.shape[0]
    int8 = Xo.dtype == torch.int8
    shape = make_shape(M, N, K, k_o, group, _outlier_kind(int8), 8 if Xq.dtype == torch.int8 else 4,
                       8 if Wq.dtype == torch.int8 else 4)
    Y = torch.empty((M, N), dtype=torch.float16, device=sx.device)
    quik_gemm(shape, Xq, sx, Xo, sxo, Wq, sw, Wo, swo, bias, Y, stream=stream)
    return Y


def gemm_i32(Xq, Wq, K: int, k_o: int, group: int = 0, Xo=None, Wo=None, stream=None):
    """Raw integer sums: acc [M, N] (or [G, M, N]) and, for INT8 outliers, acc_o [M, N]."""
    M, N = Xq.shape[0], Wq.shape[0]
    Ki = K - k_o
    G = Ki // group if group else 1
    int8 = Xo is not None and Xo.dtype == torch.int8
    shape = make_shape(M, N, K, k_o, group, _outlier_kind(int8), 8 if Xq.dtype == torch.int8 else 4,
                       8 if Wq.dtype == torch.int8 else 4)
    acc = torch.empty((G, M, N) if group else (M, N), dtype=torch.int32, device=Xq.device)
    acc_o = torch.empty((M, N), dtype=torch.int32, device=Xq.device) if int8 and k_o else None
    quik_gemm_i32_debug(shape, Xq, Wq, Xo if int8 else None, Wo if int8 else None, acc, acc_o,
                        stream=stream)
    return acc, acc_o


def pack_weights_24(W: torch.Tensor, perm: torch.Tensor, k_o: int, outlier_int8: bool = False,
                    stream=None):
    """Weights -> 2:4-sparse (Wq24 uint8 [N, K_i/4], Wmeta uint8 [N, K_i/8],
    w_scale [N], Wo, wo_scale), allocated on W's device."""
    N, K = W.shape
    Ki = K - k_o
    shape = make_shape(1, N, K, k_o, 0, _outlier_kind(outlier_int8))
    dev = W.device
    Wq24 = torch.empty((N, Ki // 4), dtype=torch.uint8, device=dev)
    Wmeta = torch.empty((N, Ki // 8), dtype=torch.uint8, device=dev)
    _, w_scale, Wo, wo_scale = _quant_outputs(N, K, k_o, 0, outlier_int8, dev)
    quik_pack_weights_24(shape, W, perm, Wq24, Wmeta, w_scale, Wo, wo_scale, stream=stream)
    return Wq24, Wmeta, w_scale, Wo, wo_scale


def gemm_24(xq, w24, K: int, k_o: int, bias=None, stream=None):
    """Y fp16 [M, N] from quantised activations xq (4-tuple) and 2:4 weights w24 (5-tuple)."""
    Xq, sx, Xo, sxo = xq
    Wq24, Wmeta, sw, Wo, swo = w24
    M, N = sx.shape[0], sw.shape[0]
    shape = make_shape(M, N, K, k_o, 0, _outlier_kind(Xo.dtype == torch.int8))
    Y = torch.empty((M, N), dtype=torch.float16, device=sx.device)
    quik_gemm_24(shape, Xq, sx, Xo, sxo, Wq24, Wmeta, sw, Wo, swo, bias, Y, stream=stream)
    return Y


def gemm24_i32(Xq, Wq24, Wmeta, K: int, k_o: int, Xo=None, Wo=None, stream=None):
    """Integer sums of the 2:4 product: acc [M, N] and, for INT8 outliers, acc_o."""
    M, N = Xq.shape[0], Wq24.shape[0]
    int8 = Xo is not None and Xo.dtype == torch.int8
    shape = make_shape(M, N, K, k_o, 0, _outlier_kind(int8))
    acc = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    acc_o = torch.empty((M, N), dtype=torch.int32, device=Xq.device) if int8 and k_o else None
    quik_gemm_24_i32_debug(shape, Xq, Wq24, Wmeta, Xo if int8 else None, Wo if int8 else None, acc,
                           acc_o, stream=stream)
    return acc, acc_o


def expand_weights_24(Wq24: torch.Tensor, Wmeta: torch.Tensor, K: int, k_o: int, stream=None):
    """Dense packed INT4 weights uint8 [N, K_i/2] that 2:4 weights stand for."""
    N = Wq24.shape[0]
    shape = make_shape(1, N, K, k_o)
    Wq = torch.empty((N, (K - k_o) // 2), dtype=torch.uint8, device=Wq24.device)
    quik_expand_weights_24(shape, Wq24, Wmeta, Wq, stream=stream)
    return Wq


class QuikLinear24:
    """A W4A4 + outlier linear layer with 2:4-sparse INT4 weights.

    ``QuikLinear24(W, perm, k_o, outlier_int8, bias)`` prunes and packs W once
    (quik_pack_weights_24); calling it on fp16 activations runs quik_linear_24
    into a workspace it keeps (above 32 tokens the workspace also holds the
    weights expanded for the dense kernel).
    """

    def __init__(self, W: torch.Tensor, perm: torch.Tensor, k_o: int, outlier_int8: bool = False,
                 bias: torch.Tensor | None = None):
        self.N, self.K = W.shape
        self.k_o, self.outlier_int8, self.perm, self.bias = k_o, outlier_int8, perm, bias
        (self.Wq24, self.Wmeta, self.w_scale, self.Wo,
         self.wo_scale) = pack_weights_24(W, perm, k_o, outlier_int8)
        self._ws = None

    def shape(self, M: int) -> quik_shape:
        return make_shape(M, self.N, self.K, self.k_o, 0, _outlier_kind(self.outlier_int8))

    def __call__(self, X: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        M = X.shape[0]
        need = quik_workspace_size_24(self.shape(M))
        if need == 0:
            raise QuikError(QUIK_ERR_UNSUPPORTED, "quik_workspace_size_24")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty((need,), dtype=torch.uint8, device=X.device)
        Y = out if out is not None else torch.empty((M, self.N), dtype=torch.float16, device=X.device)
        quik_linear_24(self.shape(M), X, self.perm, self.Wq24, self.Wmeta, self.w_scale, self.Wo,
                       self.wo_scale, self.bias, Y, self._ws, stream=stream)
        return Y


class QuikLinear:
    """A hybrid W4A4 (or W4A8, W8A8) + outlier linear layer with packed weights on the GPU.

    ``QuikLinear(W, perm, k_o, group, outlier_int8, bias, act_bits, weight_bits)``
    packs W once (quik_pack_weights); calling it on fp16 activations runs
    quik_linear into a workspace it keeps.  act_bits / weight_bits 8 quantise
    the activations / weights to INT8.  With ``norm_weight`` (fp16 [K]) the
    layer takes the hidden state before an RMS norm (weight norm_weight,
    epsilon norm_eps) and runs quik_rmsnorm_linear: the norm is folded into
    the activation quantiser.
    """

    def __init__(self, W: torch.Tensor, perm: torch.Tensor, k_o: int, group: int = 0,
                 outlier_int8: bool = False, bias: torch.Tensor | None = None, act_bits: int = 4,
                 weight_bits: int = 4, norm_weight: torch.Tensor | None = None,
                 norm_eps: float = 1e-6):
        self.norm_weight, self.norm_eps = norm_weight, norm_eps
        self.N, self.K = W.shape
        self.k_o, self.group, self.outlier_int8 = k_o, group, outlier_int8
        self.act_bits, self.weight_bits = act_bits, weight_bits
        self.perm = perm
        self.bias = bias
        self.Wq, self.w_scale, self.Wo, self.wo_scale = pack_weights(W, perm, k_o, group, outlier_int8,
                                                                     weight_bits=weight_bits)
        self._ws = None

    def shape(self, M: int) -> quik_shape:
        return make_shape(M, self.N, self.K, self.k_o, self.group, _outlier_kind(self.outlier_int8),
                          self.act_bits, self.weight_bits)

    def workspace(self, M: int, device) -> torch.Tensor:
        need = quik_workspace_size(self.shape(M))
        if need == 0:
            raise QuikError(QUIK_ERR_INVALID_ARG, "quik_workspace_size")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty((need,), dtype=torch.uint8, device=device)
        return self._ws

    def __call__(self, X: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        M = X.shape[0]
        Y = out if out is not None else torch.empty((M, self.N), dtype=torch.float16, device=X.device)
        if self.norm_weight is not None:
            quik_rmsnorm_linear(self.shape(M), X, self.norm_weight, self.norm_eps, self.perm, self.Wq,
                                self.w_scale, self.Wo, self.wo_scale, self.bias, Y,
                                self.workspace(M, X.device), stream=stream)
        else:
            quik_linear(self.shape(M), X, self.perm, self.Wq, self.w_scale, self.Wo, self.wo_scale,
                        self.bias, Y, self.workspace(M, X.device), stream=stream)
        return Y
