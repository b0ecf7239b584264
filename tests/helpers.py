"""Shared test helpers: run the CPU oracle on the same seeded inputs the GPU
gets, and compare.  Only tests import this module."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixed_precision_quantized_quantize_b200 import workloads as wl

RTOL = 2e-3       # max relative error of fp16 outputs ...
DENOM_FLOOR = 1e-2  # ... with denominator max(|ref|, 1e-2)


def rel_err(y_gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    return np.abs(y_gpu.astype(np.float64) - ref) / np.maximum(np.abs(ref), DENOM_FLOOR)


def assert_y_close(y_gpu, ref, what=""):
    e = rel_err(np.asarray(y_gpu), np.asarray(ref))
    worst = np.unravel_index(np.argmax(e), e.shape) if e.size else None
    assert e.size == 0 or e.max() <= RTOL, (
        f"{what}: max rel err {e.max():.3e} at {worst}: gpu={np.asarray(y_gpu)[worst]} "
        f"ref={np.asarray(ref)[worst]}")
    return float(e.max()) if e.size else 0.0


def np16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def oracle_quant(t: torch.Tensor, perm: torch.Tensor, k_o: int, group: int, int8: bool):
    return oracle.quantize_rows(np16(t), perm.numpy(), k_o, group, int8)


def gpu_tuple_np(tup):
    return tuple(None if x is None else x.cpu().numpy() for x in tup)


def assert_quant_equal(gpu, ref, what=""):
    """Codes, scales, outlier block (and INT8 scales) bit-exact."""
    names = ("codes", "scales", "outliers", "outlier scales")
    for name, g, r in zip(names, gpu, ref):
        if r is None:
            continue
        g = np.asarray(g)
        if g.dtype == np.float32:
            g, r = g.view(np.uint32), np.asarray(r, np.float32).view(np.uint32)
        elif g.dtype == np.float16:
            g, r = g.view(np.uint16), np.asarray(r, np.float16).view(np.uint16)
        assert g.shape == r.shape, (what, name, g.shape, r.shape)
        bad = np.argwhere(g != r)
        assert bad.size == 0, f"{what}: {name} differ at {bad[:5].tolist()} ({len(bad)} total)"


def layer_inputs(cfg: wl.LayerConfig, M: int | None = None, seed_offset: int = 0):
    return wl.make_layer(cfg, M=M, seed_offset=seed_offset)
