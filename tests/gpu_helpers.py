"""Helpers shared by the GPU tests: run the library on a seeded workload and compare it
with the float64 oracle on the same inputs."""
import functools

import numpy as np
import torch

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_workload

# Tolerances on max |Y_gpu - Y_oracle|, relative to max |Y_oracle| over the compared rows.
TOL = {"f32": 1e-4, "bf16": 2e-2}


@functools.lru_cache(maxsize=None)
def workload(name):
    return make_workload(name)


@functools.lru_cache(maxsize=None)
def oracle_csr(name):
    w = workload(name)
    return oracle.csr_from_coo(w.N, w.src, w.dst)


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(dtype) if dtype is not None else t


def run_gpu(w, options=None, csr=None, keep_layer=False):
    """CSR built on the GPU from the workload's COO, then one forward."""
    dt = glga.torch_dtype(w.io)
    if csr is None:
        row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    else:
        row_ptr, col_idx = to_dev(csr[0]), to_dev(csr[1])
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, options)
    args = [to_dev(a, dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    Y = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0
    out = {"Y": Y, "row_ptr": row_ptr, "col_idx": col_idx, "args": args}
    if keep_layer:
        out["layer"] = layer
    else:
        layer.close()
    return out


def sample_rows(w, row_ptr, n_random=2000, seed=1):
    """Random rows plus the heaviest rows, the lightest rows and both ends."""
    deg = np.diff(row_ptr)
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(w.N, size=min(n_random, w.N), replace=False).tolist())
    order = np.argsort(deg, kind="stable")
    rows.update(order[-48:].tolist())
    rows.update(order[:16].tolist())
    rows.update([0, w.N - 1])
    return np.array(sorted(rows), dtype=np.int64)


def assert_close_to_oracle(w, Y_gpu, ref, rows=None, tol=None):
    Yg = Y_gpu.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        Yg = Yg[rows]
    Yo = ref["Y"]
    scale = np.abs(Yo).max()
    err = np.abs(Yg - Yo).max()
    tol = TOL[w.io] if tol is None else tol
    assert np.all(np.isfinite(Yg))
    assert err <= tol * scale, f"max err {err:.3e} > {tol:g} * max|Y| ({scale:.3e})"
    return err / scale
