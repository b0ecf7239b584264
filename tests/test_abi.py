"""The C-ABI library without a GPU: it loads, exports every function that
include/quik.h declares, and its host-side logic (status strings, workspace
sizes, argument validation that returns before any CUDA call) behaves as the
header documents."""
import ctypes
import subprocess

import pytest

import mixed_precision_quantized_quantize_b200 as q
from mixed_precision_quantized_quantize_b200 import build as qbuild


@pytest.fixture(scope="module")
def L():
    qbuild.build()
    return q.lib()


def test_exports_every_header_function(L):
    names = q.header_functions()
    assert "quik_linear" in names and "quik_pack_weights" in names
    out = subprocess.run(["nm", "-D", "--defined-only", q.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)
    # nothing else of ours leaks out of the library
    assert {e for e in exported if e.startswith("quik")} == set(names)


def test_status_strings(L):
    for s, name in [(q.QUIK_OK, "QUIK_OK"), (q.QUIK_ERR_INVALID_ARG, "QUIK_ERR_INVALID_ARG"),
                    (q.QUIK_ERR_UNSUPPORTED, "QUIK_ERR_UNSUPPORTED"),
                    (q.QUIK_ERR_CUDA, "QUIK_ERR_CUDA"), (q.QUIK_ERR_TIMEOUT, "QUIK_ERR_TIMEOUT")]:
        assert q.status_string(s) == name


def _ws(M, N, K, k_o, group=0, outlier=0, act_bits=4, weight_bits=4):
    return q.quik_workspace_size(q.make_shape(M, N, K, k_o, group, outlier, act_bits, weight_bits))


def test_workspace_size(L):
    r = lambda b: (b + 255) // 256 * 256
    # FP16 outliers above 32 tokens: the codes widened to one byte each (the
    # persistent GEMM's operand), per-token scales, fp16 outlier block
    assert _ws(2048, 4096, 4096, 128) == r(2048 * 3968) + r(2048 * 4) + r(2048 * 128 * 2)
    # up to 32 tokens (the decode kernel) and with INT8 outliers: packed codes
    assert _ws(32, 4096, 4096, 128) == r(32 * 3968 // 2) + r(32 * 4) + r(32 * 128 * 2)
    assert _ws(64, 4096, 4096, 128, 0, 1) == r(64 * 3968 // 2) + r(64 * 4) + r(64 * 128) + r(64 * 4)
    # grouped + INT8 outliers: G scales per token, int8 block, one INT8 scale per token
    G = (8192 - 128) // 128
    assert _ws(1024, 22016, 8192, 128, 128, 1) == (r(1024 * 8064 // 2) + r(1024 * G * 4)
                                                   + r(1024 * 128) + r(1024 * 4))
    assert _ws(16, 256, 256, 0) == r(16 * 128) + r(16 * 4)
    # INT8 activations (W4A8): one byte per code; 0 is INT4 as well
    assert _ws(2048, 4096, 4096, 128, 0, 0, 8) == r(2048 * 3968) + r(2048 * 4) + r(2048 * 128 * 2)
    assert _ws(2048, 4096, 4096, 128, 0, 0, 0) == _ws(2048, 4096, 4096, 128)


@pytest.mark.parametrize("shape", [
    (0, 16, 256, 32, 0, 0),       # M < 1
    (16, 0, 256, 32, 0, 0),       # N < 1
    (16, 16, 256, 300, 0, 0),     # k_o > K
    (16, 16, 256, -16, 0, 0),     # k_o < 0
    (16, 16, 272, 32, 0, 0),      # K_i = 240 not a multiple of 32
    (16, 16, 264, 8, 0, 0),       # k_o not a multiple of 16
    (16, 16, 320, 32, 128, 0),    # grouped with K_i = 288, not a multiple of 128
    (16, 16, 256, 0, -1, 0),      # negative group size
    (16, 16, 256, 0, 0, 5),       # unknown outlier kind
    (16, 16, 65536, 0, 0, 0),     # K above the supported maximum
    (16, 16, 256, 0, 0, 0, 3),    # activation width neither 4 nor 8
    (16, 16, 256, 0, 0, 0, 16),
    (16, 16, 256, 0, 0, 0, 8, 2),  # weight width neither 4 nor 8
])
def test_invalid_shapes_rejected(L, shape):
    assert _ws(*shape) == 0
    s = q.make_shape(*shape)
    st = L.quik_quantize_reorder(ctypes.byref(s), None, None, None, None, None, None, None)
    assert st == q.QUIK_ERR_INVALID_ARG


def test_unsupported_group_size(L):
    s = q.make_shape(16, 16, 256, 0, 64, 0)
    assert L.quik_gemm(ctypes.byref(s), *([None] * 11)) == q.QUIK_ERR_UNSUPPORTED


def test_int8_weights_need_int8_activations(L):
    s = q.make_shape(16, 16, 256, 0, 0, 0, 4, 8)
    assert q.quik_workspace_size(s) == 0
    assert L.quik_gemm(ctypes.byref(s), *([None] * 11)) == q.QUIK_ERR_UNSUPPORTED
    # W8A8: the workspace holds the INT8 activations, as for W4A8
    assert q.quik_workspace_size(q.make_shape(64, 16, 256, 0, 0, 0, 8, 8)) == 64 * 256 + 256


def test_grouped_int8_activations_unsupported(L):
    s = q.make_shape(16, 16, 256, 0, 128, 0, 8)
    assert _ws(16, 16, 256, 0, 128, 0, 8) == 0
    assert L.quik_gemm(ctypes.byref(s), *([None] * 11)) == q.QUIK_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected(L):
    s = q.make_shape(16, 16, 256, 32, 0, 0)
    assert L.quik_quantize_reorder(ctypes.byref(s), None, None, None, None, None, None, None) \
        == q.QUIK_ERR_INVALID_ARG
    # misaligned (but otherwise fake, never dereferenced) addresses
    bad = ctypes.c_void_p(0x1001)
    good = ctypes.c_void_p(0x1000)
    assert L.quik_quantize_reorder(ctypes.byref(s), bad, good, good, good, good, None, None) \
        == q.QUIK_ERR_INVALID_ARG
    assert L.quik_linear(ctypes.byref(s), good, good, good, good, good, None, None, good, good,
                         1, None) == q.QUIK_ERR_INVALID_ARG  # workspace too small
    assert L.quik_selftest_timeout(0, None) == q.QUIK_ERR_INVALID_ARG
    assert L.quik_selftest_timeout(2000000, None) == q.QUIK_ERR_INVALID_ARG


def test_rmsnorm_arguments_rejected(L):
    """The fused norm needs an aligned gamma and a finite eps > 0; every case
    below is rejected before anything is launched (fake addresses, never
    dereferenced)."""
    s = q.make_shape(16, 16, 256, 32, 0, 0)
    good = ctypes.c_void_p(0x1000)
    bad = ctypes.c_void_p(0x1008)
    f = L.quik_rmsnorm_quantize_reorder
    for gamma, eps in ((None, 1e-6), (bad, 1e-6), (good, 0.0), (good, -1e-6),
                       (good, float("nan")), (good, float("inf"))):
        assert f(ctypes.byref(s), good, gamma, eps, good, good, good, good, None, None) \
            == q.QUIK_ERR_INVALID_ARG
        assert L.quik_rmsnorm_linear(ctypes.byref(s), good, gamma, eps, good, good, good, good,
                                     None, None, good, good, 1 << 30, None) \
            == q.QUIK_ERR_INVALID_ARG


def test_rmsnorm_widest_rows_unsupported(L):
    """K past 24576 does not fit the fused norm's two shared-memory tables."""
    s = q.make_shape(16, 16, 24576 + 64, 64, 0, 0)
    good = ctypes.c_void_p(0x1000)
    assert L.quik_rmsnorm_quantize_reorder(ctypes.byref(s), good, good, 1e-5, good, good, good,
                                           good, None, None) == q.QUIK_ERR_UNSUPPORTED
    assert L.quik_rmsnorm_linear(ctypes.byref(s), good, good, 1e-5, good, good, good, good, None,
                                 None, good, good, 1 << 30, None) == q.QUIK_ERR_UNSUPPORTED


def test_sparse24_shape_rules(L):
    """2:4 weights need per-channel scales, INT4 activations and weights,
    K_i % 128 == 0 and a small outlier block; anything else is unsupported
    (rejected before any pointer is looked at)."""
    good = ctypes.c_void_p(0x1000)
    for args in ((16, 16, 512, 0, 128, 0, 4, 4),    # groups
                 (16, 16, 512, 0, 0, 0, 8, 4),      # INT8 activations
                 (16, 16, 512, 64, 0, 0, 4, 4),     # K_i = 448
                 (16, 16, 1024, 256, 0, 0, 4, 4),   # 256 FP16 outlier channels
                 (16, 16, 1024, 384, 0, 1, 4, 4)):  # 384 INT8 outlier channels
        s = q.make_shape(*args)
        assert L.quik_pack_weights_24(ctypes.byref(s), good, good, good, good, good, good, good,
                                      None) == q.QUIK_ERR_UNSUPPORTED
        assert L.quik_gemm_24(ctypes.byref(s), *([good] * 11), None) == q.QUIK_ERR_UNSUPPORTED


def test_sparse24_workspace_size(L):
    """Up to 32 tokens the 2:4 layer needs the dense layer's workspace; with
    more it also holds the expanded weights (N x K_i / 2 bytes, 256-aligned)."""
    for M in (1, 16, 32, 33, 2048):
        s = q.make_shape(M, 4096, 4096, 128)
        base = L.quik_workspace_size(ctypes.byref(s))
        extra = 0 if M <= 32 else -(-(4096 * 3968 // 2) // 256) * 256
        assert L.quik_workspace_size_24(ctypes.byref(s)) == base + extra
    assert L.quik_workspace_size_24(ctypes.byref(q.make_shape(16, 16, 512, 64))) == 0  # K_i = 448


def test_header_is_plain_c(tmp_path):
    """include/quik.h compiles as C99 and a C program links against the
    library and calls it (size queries need no GPU)."""
    import os
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    libdir = os.path.dirname(q.LIB_PATH)
    src = tmp_path / "abi.c"
    src.write_text(
        '#include <stdio.h>\n#include "quik.h"\n'
        "int main(void) {\n"
        "    quik_shape s = {2048, 4096, 4096, 128, 0, QUIK_OUTLIER_FP16, 4, 4};\n"
        '    printf("%zu %zu %s\\n", quik_workspace_size(&s), quik_workspace_size_24(&s),\n'
        "           quik_status_string(QUIK_ERR_UNSUPPORTED));\n"
        "    return 0;\n}\n")
    exe = tmp_path / "abi"
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc,
                           str(src), "-o", str(exe), "-L", libdir, "-lquik_b200",
                           f"-Wl,-rpath,{libdir}"])
    out = subprocess.check_output([str(exe)], text=True).split()
    s = q.make_shape(2048, 4096, 4096, 128)
    assert int(out[0]) == q.quik_workspace_size(s)
    assert int(out[1]) == q.quik_workspace_size_24(s)
    assert out[2] == "QUIK_ERR_UNSUPPORTED"
