"""The allocation-free global-statistics entry point (glga_global_stats_static).

Some callers may not allocate device memory where they enqueue work (plugin enqueue
callbacks, services that own all device memory through their own pool, latency-critical
paths that cannot take cudaMalloc's implicit synchronisation).  This entry point computes
the layer's S and z with its partial sums in a fixed array inside the library.  The tests
call it through the C ABI twice in a row and compare it with the float64 oracle's S and z
(method page "Gated Local-Global Graph Attention", Key formulas) computed on the very K and
V that were passed in, and on the oracle's own projections of X, within the tolerances of
the other parity tests; the S and z of glga_forward on the same graph are an extra check.
The call's error path (glga_global_stats_static_error) is exercised with the bounded-wait
probe, which times out without faulting the GPU.  This file is collected last and also
runs alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_workload
from tests.gpu_helpers import TOL, run_gpu

pytestmark = pytest.mark.gpu


def _static(KV, N, H, r, io, Sz):
    stream = torch.cuda.current_stream().cuda_stream
    st = glga.lib().glga_global_stats_static(
        ctypes.c_void_p(KV.data_ptr()), N, H, r, glga.GLGA_F32 if io == "f32" else glga.GLGA_BF16,
        ctypes.c_void_p(Sz.data_ptr()), ctypes.c_void_p(stream))
    assert st == 0, glga.lib().glga_last_error_message()
    torch.cuda.synchronize()
    got = Sz.cpu().numpy().astype(np.float64)
    return got[: H * r * r].reshape(H, r, r), got[H * r * r:].reshape(H, r)


def _close(got, ref, tol, what):
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert np.all(np.isfinite(got)) and err <= tol, f"{what}: {err:.3e} > {tol:g}"


@pytest.mark.parametrize("name,scale", [("citation", 1.0), ("arxiv", 0.05), ("packed", 0.02)])
def test_static_scratch_stats_match_oracle_twice(name, scale):
    w = make_workload(name, scale=scale)
    out = run_gpu(w, keep_layer=True)
    layer = out["layer"]
    inter = layer.intermediates()
    torch.cuda.synchronize()
    KV = torch.cat([inter["K"], inter["V"]], dim=1).contiguous()
    H, r = w.H, w.r
    # the oracle on exactly the K and V given to the call (widened to float64) ...
    K64 = inter["K"].float().cpu().numpy().astype(np.float64)
    V64 = inter["V"].float().cpu().numpy().astype(np.float64)
    S_in, z_in = oracle.global_stats(K64, V64, H, r)
    # ... and on the oracle's own projections of X
    S_or, z_or = oracle.global_stats(oracle.project(w.X, w.W_K), oracle.project(w.X, w.W_V), H, r)
    S_fw = inter["S"].cpu().numpy().astype(np.float64)
    z_fw = inter["z"].cpu().numpy().astype(np.float64)
    tol = TOL[w.io]
    Sz = torch.empty(H * r * r + H * r, dtype=torch.float32, device=KV.device)
    for _ in range(2):
        Sz.fill_(float("nan"))           # every output must be written by the call
        S, z = _static(KV, w.N, H, r, w.io, Sz)
        _close(S, S_in, tol, "S vs oracle on the given K, V")
        _close(z, z_in, tol, "z vs oracle on the given K, V")
        _close(S, S_or, tol, "S vs oracle forward")
        _close(z, z_or, tol, "z vs oracle forward")
        _close(S, S_fw, tol, "S vs glga_forward")
        _close(z, z_fw, tol, "z vs glga_forward")
        assert glga.global_stats_static_error() == 0
    layer.close()


def test_static_scratch_timeout_is_reported_then_cleared():
    # A bounded wait on the static calls' flag that nothing ends: it gives up after 20 ms
    # and raises the flag, as a timed-out statistics kernel would.  The report returns
    # GLGA_ERR_TIMEOUT once, then the flag is clear and the entry point still computes
    # correct statistics.
    w = make_workload("tiny")
    K = oracle.project(w.X, w.W_K)
    V = oracle.project(w.X, w.W_V)
    KV = torch.from_numpy(np.concatenate([K, V], axis=1).astype(np.float32)).cuda().contiguous()
    stream = torch.cuda.current_stream().cuda_stream
    assert glga.global_stats_static_error() == 0
    st = glga.lib().glga_debug_static_bounded_wait(20_000_000, ctypes.c_void_p(stream))
    assert st == 0, glga.lib().glga_last_error_message()
    assert glga.global_stats_static_error() == 6           # GLGA_ERR_TIMEOUT
    assert b"timed out" in glga.lib().glga_last_error_message()
    assert glga.global_stats_static_error() == 0           # read-and-clear
    Sz = torch.empty(w.H * w.r * w.r + w.H * w.r, dtype=torch.float32, device="cuda")
    S, z = _static(KV, w.N, w.H, w.r, "f32", Sz)
    S_ref, z_ref = oracle.global_stats(K.astype(np.float32).astype(np.float64),
                                       V.astype(np.float32).astype(np.float64), w.H, w.r)
    _close(S, S_ref, TOL["f32"], "S after the timeout")
    _close(z, z_ref, TOL["f32"], "z after the timeout")
    assert glga.global_stats_static_error() == 0
    assert glga.lib().glga_debug_static_bounded_wait(10, ctypes.c_void_p(stream)) == 1


def test_static_scratch_rejects_shapes_beyond_its_size():
    KV = torch.zeros(4, 2 * 32 * 128, dtype=torch.bfloat16, device="cuda")
    Sz = torch.zeros(32 * 128 * 129, dtype=torch.float32, device="cuda")
    st = glga.lib().glga_global_stats_static(ctypes.c_void_p(KV.data_ptr()), 4, 32, 128,
                                             glga.GLGA_BF16, ctypes.c_void_p(Sz.data_ptr()), None)
    assert st == 3
    assert b"static scratch" in glga.lib().glga_last_error_message()
