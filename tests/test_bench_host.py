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
