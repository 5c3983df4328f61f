"""The allocation-free global-statistics entry point (glga_global_stats_static).

Some callers may not allocate device memory where they enqueue work (plugin enqueue
callbacks, services that own all device memory through their own pool, latency-critical
paths that cannot take cudaMalloc's implicit synchronisation).  This entry point computes
the layer's S and z with its partial sums in a fixed array inside the library.  The test
calls it through the C ABI twice in a row and compares it with the S and z that
glga_forward computed on the same K and V, within the tolerance the other S/z checks use.
It lives in its own file, collected last, and also runs alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_workload
from tests.gpu_helpers import TOL, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,scale", [("citation", 1.0), ("arxiv", 0.05), ("packed", 0.02)])
def test_static_scratch_stats_match_forward_twice(name, scale):
    w = make_workload(name, scale=scale)
    out = run_gpu(w, keep_layer=True)
    layer = out["layer"]
    inter = layer.intermediates()
    torch.cuda.synchronize()
    KV = torch.cat([inter["K"], inter["V"]], dim=1).contiguous()
    H, r = w.H, w.r
    S_ref = inter["S"].cpu().numpy().astype(np.float64)
    z_ref = inter["z"].cpu().numpy().astype(np.float64)
    Sz = torch.empty(H * r * r + H * r, dtype=torch.float32, device=KV.device)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        Sz.fill_(float("nan"))           # every output must be written by the call
        st = glga.lib().glga_global_stats_static(
            ctypes.c_void_p(KV.data_ptr()), w.N, H, r,
            glga.GLGA_F32 if w.io == "f32" else glga.GLGA_BF16,
            ctypes.c_void_p(Sz.data_ptr()), ctypes.c_void_p(stream))
        assert st == 0, glga.lib().glga_last_error_message()
        torch.cuda.synchronize()
        got = Sz.cpu().numpy().astype(np.float64)
        S, z = got[: H * r * r].reshape(H, r, r), got[H * r * r:].reshape(H, r)
        tol = TOL[w.io]
        np.testing.assert_allclose(S, S_ref, rtol=0, atol=tol * np.abs(S_ref).max())
        np.testing.assert_allclose(z, z_ref, rtol=0, atol=tol * np.abs(z_ref).max())
    layer.close()


def test_static_scratch_rejects_shapes_beyond_its_size():
    KV = torch.zeros(4, 2 * 32 * 128, dtype=torch.bfloat16, device="cuda")
    Sz = torch.zeros(32 * 128 * 129, dtype=torch.float32, device="cuda")
    st = glga.lib().glga_global_stats_static(ctypes.c_void_p(KV.data_ptr()), 4, 32, 128,
                                             glga.GLGA_BF16, ctypes.c_void_p(Sz.data_ptr()), None)
    assert st == 3
    assert b"static scratch" in glga.lib().glga_last_error_message()
