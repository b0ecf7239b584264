"""B200-native (sm_100a) hybrid W4A4 + outlier linear layer (QUIK / Atom).

The compute path is the CUDA library ``libquik_b200.so`` (C ABI in
``include/quik.h``); this package is its Python binding.  Importing the
package does not load the library; the first call does, and raises if the
library has not been built (there is no CPU fallback).
"""
from ._binding import (  # noqa: F401
    GROUP,
    QUIK_ERR_CUDA,
    QUIK_ERR_INVALID_ARG,
    QUIK_ERR_TIMEOUT,
    QUIK_ERR_UNSUPPORTED,
    QUIK_OK,
    QUIK_OUTLIER_FP16,
    QUIK_OUTLIER_INT8,
    LIB_PATH,
    QuikError,
    QuikLinear,
    gemm,
    gemm_i32,
    header_functions,
    lib,
    make_shape,
    pack_weights,
    quantize_reorder,
    rmsnorm_quantize_reorder,
    quik_gemm,
    quik_gemm_i32_debug,
    quik_linear,
    quik_linear_noalloc,
    quik_pack_weights,
    quik_quantize_reorder,
    quik_rmsnorm_linear,
    quik_rmsnorm_quantize_reorder,
    quik_selftest_timeout,
    quik_shape,
    quik_status_string,
    quik_sync_check,
    quik_workspace_size,
    status_string,
)
