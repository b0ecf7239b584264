"""Host-side arithmetic of bench.py (no GPU): the layer call's path roofline
for every workload, against its definition written out for two of them."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixed_precision_quantized_quantize_b200 import workloads as wl  # noqa: E402

PEAKS = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}


@pytest.mark.parametrize("name", sorted(wl.CONFIGS))
def test_path_roofline_is_well_formed(name):
    cfg = wl.CONFIGS[name]
    r = bench.path_roofline(cfg, PEAKS, 100e-6)
    assert r["t_roof_us"] > 0 and r["gemm_roof_us"] > 0 and r["quantise_roof_us"] > 0
    assert r["t_roof_us"] == pytest.approx(r["gemm_roof_us"] + r["quantise_roof_us"], abs=0.02)
    assert r["frac"] == pytest.approx(r["t_roof_us"] / 100.0, abs=1e-4)


def test_path_roofline_attention_projection():
    """2048 x 4096 x 4096, 128 FP16 outliers: INT4 part at 3.2 POPS, outliers at 1.6 PFLOP/s."""
    cfg = wl.CONFIGS["llama7b_attn_2048x4096x4096"]
    r = bench.path_roofline(cfg, PEAKS, 68.8e-6)
    t_tensor = 2 * 2048 * 4096 * 3968 / 3.2e15 + 2 * 2048 * 4096 * 128 / 1.6e15
    quant = 2048 * 4096 * 2 + 2048 * 3968 // 2 + 2048 * 128 * 2 + 2048 * 4
    assert r["gemm_bound"] == "tensor"
    assert r["gemm_roof_us"] == pytest.approx(t_tensor * 1e6, abs=0.01)
    assert r["quantise_roof_us"] == pytest.approx(quant / 6.5e12 * 1e6, abs=0.01)


def test_path_roofline_decode_is_byte_bound():
    cfg = wl.CONFIGS["llama7b_up_16x11008x4096"]
    r = bench.path_roofline(cfg, PEAKS, 19.5e-6)
    assert r["gemm_bound"] == "hbm"
    assert r["gemm_roof_us"] == pytest.approx(cfg.gemm_bytes / 6.5e12 * 1e6, abs=0.01)


@pytest.mark.parametrize("M,N,K,k_o,rmsnorm,kernel", [
    # the attention projection: 128 tiles of 256 x 256 (two waves on 74
    # pairs), 64 of 256 x 512 (one wave) -> 512-token tiles, widened or
    # packed (the norm-fused workload's GEMM is timed on packed codes)
    (2048, 4096, 4096, 128, False, "w4a4_gemm_persistent2"),
    (2048, 4096, 4096, 128, True, "w4a4_gemm_persistent2"),
    # four FP16 outlier units: four operand stages with widened codes, three
    # with packed ones
    (2048, 4096, 4352, 256, False, "w4a4_gemm_persistent2"),
    (2048, 4096, 4352, 256, True, "w4a4_gemm_persistent "),
    # 172 tiles of 512 tokens: more than one wave either way
    (2048, 11008, 4096, 128, False, "w4a4_gemm_persistent "),
    # 43 tiles of 256: already one wave
    (256, 11008, 4096, 128, False, "w4a4_gemm_persistent "),
])
def test_gemm_kernel_names_the_tile_form(M, N, K, k_o, rmsnorm, kernel):
    """bench.py names the persistent GEMM's tile form by the library's
    dispatch rule (one wave of 512-token tiles where 256-token tiles need
    more, at most three or four outlier units)."""
    cfg = wl.custom_config(M, N, K, k_o, 0, False, False, rmsnorm=rmsnorm)
    name, profile = bench.gemm_kernel(cfg)
    assert name.startswith(kernel)
    assert profile.startswith(kernel.strip() + "_")
