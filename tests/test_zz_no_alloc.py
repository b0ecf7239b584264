"""quik_linear_noalloc: the layer for callers that cannot allocate device memory.

Some callers cannot give quik_linear a workspace: a host framework that owns
all device memory through a fixed plan and gives plugins none, or a
latency-critical path where cudaMalloc (which may synchronise the device) is
off limits.  For them the library keeps its own fixed workspace.  This test
calls that entry point through the C ABI twice in a row (the second call
reuses whatever the first left in the shared workspace) and checks each
output against quik_linear with a caller-provided workspace.  Both run the
same kernels on the same inputs, so the fp16 outputs must be bit-identical
(a looser check, the parity tests' 2e-3 relative tolerance, would hide a
workspace mix-up that perturbs a few values).  The device's free memory must
not change across the second call.  It must pass alone in a fresh process as
well as after the other tests; the file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixed_precision_quantized_quantize_b200 as q
from mixed_precision_quantized_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _run_both(cfg, seed):
    d = wl.make_layer(cfg, seed_offset=seed)
    dev = torch.device("cuda")
    perm = d["perm"].to(dev)
    X = d["X"].to(dev)
    bias = d["bias"].to(dev) if d["bias"] is not None else None
    layer = q.QuikLinear(d["W"].to(dev), perm, cfg.k_o, cfg.group, cfg.outlier_int8, bias)
    shape = layer.shape(cfg.M)
    ref = layer(X)  # quik_linear with a caller-provided workspace
    L = q.lib()
    outs = [torch.full((cfg.M, cfg.N), float("nan"), dtype=torch.float16, device=dev)
            for _ in range(2)]
    free = []
    for Y in outs:
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        st = L.quik_linear_noalloc(
            ctypes.byref(shape), X.data_ptr(), perm.data_ptr(), layer.Wq.data_ptr(),
            layer.w_scale.data_ptr(), layer.Wo.data_ptr() if cfg.k_o else None,
            layer.wo_scale.data_ptr() if layer.wo_scale is not None else None,
            bias.data_ptr() if bias is not None else None, Y.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert st == q.QUIK_OK, q.status_string(st)
    torch.cuda.synchronize()
    free.append(torch.cuda.mem_get_info()[0])
    assert q.quik_sync_check() == q.QUIK_OK
    # the second call allocates nothing (the first may load the module)
    assert free[2] == free[1]
    r = ref.cpu().numpy().view(np.uint16)
    for Y in outs:
        y = Y.cpu().numpy().view(np.uint16)
        bad = np.argwhere(y != r)
        assert bad.size == 0, f"{len(bad)} outputs differ from quik_linear, first at {bad[:3].tolist()}"


@pytest.mark.parametrize("name", ["tiny_16x256x256", "llama7b_attn_2048x4096x4096",
                                  "llama65b_mlp_grouped_1024x22016x8192",
                                  "llama7b_down_fused_4096x4096x11008"])
def test_noalloc_matches_linear_twice(name):
    _run_both(wl.CONFIGS[name], seed=0)


def test_noalloc_rejects_shapes_beyond_its_workspace():
    L = q.lib()
    # the widened codes alone (M x K_i bytes) exceed the fixed workspace:
    # refused before any launch
    s = q.make_shape(32768, 256, 4096, 0)
    assert q.quik_workspace_size(s) > (64 << 20)
    st = L.quik_linear_noalloc(ctypes.byref(s), None, None, None, None, None, None, None, None,
                               None)
    assert st == q.QUIK_ERR_UNSUPPORTED
