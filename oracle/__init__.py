"""float64 CPU oracle for the gated local-global graph-attention layer.

TEST INFRASTRUCTURE ONLY: imported by `tests/`, by `__graft_entry__.smoke()` and by the
CPU-baseline leg of `bench.py`, never by the library.  It shares no code with the CUDA
path.  The arithmetic lives in `glga_oracle.c` (plain C, double precision); this module
only compiles it with gcc, marshals numpy arrays and composes the steps in the order of
the method page ("Gated Local-Global Graph Attention", Key formulas): projections,
global statistics S and z, then per target the local softmax branch, the global readout,
the gate and the blend.

Parity status: every step here is pinned by `tests/test_oracle_pins.py` against page
witnesses, dense brute force, closed forms and invariants; no function is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "glga_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile glga_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_csr_from_coo.argtypes = [ctypes.c_int64, ctypes.c_int64, _i32p, _i32p, _i32p, _i32p]
        L.oracle_csr_from_coo.restype = ctypes.c_int
        L.oracle_degree_buckets.argtypes = [ctypes.c_int64, _i32p, ctypes.c_int32, ctypes.c_int32,
                                            _i64p] + [ctypes.c_void_p] * 5
        L.oracle_degree_buckets.restype = ctypes.c_int
        L.oracle_project.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _f32p, _f32p, _f64p]
        L.oracle_project.restype = None
        L.oracle_gate_logit.argtypes = [ctypes.c_int64, ctypes.c_int32, _f32p, _f32p, _f64p]
        L.oracle_gate_logit.restype = None
        L.oracle_phi.argtypes = [ctypes.c_double]
        L.oracle_phi.restype = ctypes.c_double
        L.oracle_global_stats.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _f64p, _f64p,
                                          _f64p, _f64p]
        L.oracle_global_stats.restype = None
        L.oracle_rows.argtypes = [ctypes.c_int64, _i64p, ctypes.c_int32, ctypes.c_int32, _i32p, _i32p,
                                  _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, ctypes.c_double,
                                  ctypes.c_double, _f64p, _f64p, _f64p, _f64p, _i64p]
        L.oracle_rows.restype = None
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def phi(x: float) -> float:
    return float(lib().oracle_phi(float(x)))


def csr_from_coo(N: int, src, dst):
    """Target-grouped CSR: row i lists the sources j of edges j -> i in ascending order."""
    src = np.ascontiguousarray(src, dtype=np.int32)
    dst = np.ascontiguousarray(dst, dtype=np.int32)
    row_ptr = np.zeros(N + 1, dtype=np.int32)
    col_idx = np.zeros(max(1, src.shape[0]), dtype=np.int32)
    rc = lib().oracle_csr_from_coo(N, src.shape[0], src, dst, row_ptr, col_idx)
    if rc != 0:
        raise ValueError(f"oracle_csr_from_coo failed ({rc})")
    return row_ptr, col_idx[: src.shape[0]]


def degree_buckets(row_ptr, warp_max: int, chunk_edges: int) -> dict:
    row_ptr = np.ascontiguousarray(row_ptr, dtype=np.int32)
    N = row_ptr.shape[0] - 1
    counts = np.zeros(4, dtype=np.int64)
    L = lib()
    if L.oracle_degree_buckets(N, row_ptr, warp_max, chunk_edges, counts, None, None, None, None, None):
        raise ValueError("bad bucket thresholds")
    out = {k: np.zeros(max(1, int(n)), dtype=np.int32) for k, n in
           (("warp_rows", counts[0]), ("cta_rows", counts[1]), ("split_rows", counts[2]),
            ("chunk_row", counts[3]), ("chunk_begin", counts[3]))}
    L.oracle_degree_buckets(N, row_ptr, warp_max, chunk_edges, counts,
                            *(out[k].ctypes.data for k in
                              ("warp_rows", "cta_rows", "split_rows", "chunk_row", "chunk_begin")))
    n = {"warp_rows": counts[0], "cta_rows": counts[1], "split_rows": counts[2],
         "chunk_row": counts[3], "chunk_begin": counts[3]}
    res = {k: out[k][: int(n[k])] for k in out}
    res["counts"] = counts.copy()
    return res


def project(X, W):
    X = np.ascontiguousarray(X, dtype=np.float32)
    W = np.ascontiguousarray(W, dtype=np.float32)
    n, d = X.shape
    D = W.shape[1]
    out = np.empty((n, D), dtype=np.float64)
    lib().oracle_project(n, d, D, X, W, out)
    return out


def gate_logit(X, w_g):
    X = np.ascontiguousarray(X, dtype=np.float32)
    w_g = np.ascontiguousarray(w_g, dtype=np.float32)
    t = np.empty(X.shape[0], dtype=np.float64)
    lib().oracle_gate_logit(X.shape[0], X.shape[1], X, w_g, t)
    return t


def global_stats(K, V, H: int, r: int):
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    S = np.empty((H, r, r), dtype=np.float64)
    z = np.empty((H, r), dtype=np.float64)
    lib().oracle_global_stats(K.shape[0], H, r, K, V, S, z)
    return S, z


def rows_output(rows, H, r, row_ptr, col_idx, Qrows, K, V, t_rows, S, z, b_g, eps):
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    D = H * r
    L = np.empty((n, D)); G = np.empty((n, D)); g = np.empty(n); Y = np.empty((n, D))
    ops = np.zeros(3, dtype=np.int64)
    col = np.ascontiguousarray(col_idx, dtype=np.int32)
    if col.shape[0] == 0:
        col = np.zeros(1, dtype=np.int32)
    lib().oracle_rows(n, rows, H, r, np.ascontiguousarray(row_ptr, dtype=np.int32), col,
                      np.ascontiguousarray(Qrows, dtype=np.float64),
                      np.ascontiguousarray(K, dtype=np.float64),
                      np.ascontiguousarray(V, dtype=np.float64),
                      np.ascontiguousarray(t_rows, dtype=np.float64),
                      np.ascontiguousarray(S, dtype=np.float64),
                      np.ascontiguousarray(z, dtype=np.float64), float(b_g), float(eps),
                      L, G, g, Y, ops)
    return {"L": L, "G": G, "g": g, "Y": Y, "ops": ops}


def forward(N, d, H, r, X, W_Q, W_K, W_V, w_g, b_g, eps, row_ptr, col_idx, rows=None,
            seg_ptr=None):
    """Full layer forward in float64 for the target rows `rows` (all rows if None).

    `seg_ptr` (optional, [n_seg + 1], 0 = seg_ptr[0] <= ... <= seg_ptr[n_seg] = N) splits
    the nodes into contiguous segments, the elements of a batch: the global statistics S,
    z are then summed over each segment's own nodes, and row i's readout uses the
    statistics of its segment (method page, "Implementation notes": the layer takes
    X [batch, N, d]; "Key formulas": the global sums run over the N nodes of one graph).
    None means one segment holding every node.

    Returns a dict with Y, L, G, g for those rows, S, z ([H, r, r] and [H, r]; with
    segments [n_seg, H, r, r] and [n_seg, H, r]), the row list, op counters and the
    seconds spent per stage (projection, global statistics, per-target outputs)."""
    t0 = time.perf_counter()
    X = np.ascontiguousarray(X, dtype=np.float32)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    K = project(X, W_K)
    V = project(X, W_V)
    Xr = np.ascontiguousarray(X[rows])
    Qr = project(Xr, W_Q)
    tr = gate_logit(Xr, w_g)
    t1 = time.perf_counter()
    if seg_ptr is None:
        S, z = global_stats(K, V, H, r)
        t2 = time.perf_counter()
        out = rows_output(rows, H, r, row_ptr, col_idx, Qr, K, V, tr, S, z, b_g, eps)
    else:
        seg_ptr = np.asarray(seg_ptr, dtype=np.int64)
        n_seg = seg_ptr.shape[0] - 1
        if n_seg < 1 or seg_ptr[0] != 0 or seg_ptr[-1] != N or np.any(np.diff(seg_ptr) < 0):
            raise ValueError("seg_ptr must run from 0 to N without decreasing")
        S = np.zeros((n_seg, H, r, r))
        z = np.zeros((n_seg, H, r))
        for k in range(n_seg):
            a, b = int(seg_ptr[k]), int(seg_ptr[k + 1])
            if b > a:
                S[k], z[k] = global_stats(K[a:b], V[a:b], H, r)
        t2 = time.perf_counter()
        # the segment of each listed row: the last segment starting at or before it
        seg = np.searchsorted(seg_ptr, rows, side="right") - 1
        D = H * r
        out = {"L": np.empty((rows.shape[0], D)), "G": np.empty((rows.shape[0], D)),
               "g": np.empty(rows.shape[0]), "Y": np.empty((rows.shape[0], D)),
               "ops": np.zeros(3, dtype=np.int64)}
        for k in np.unique(seg):
            idx = np.nonzero(seg == k)[0]
            part = rows_output(rows[idx], H, r, row_ptr, col_idx, Qr[idx], K, V, tr[idx],
                               S[k], z[k], b_g, eps)
            for key in ("L", "G", "g", "Y"):
                out[key][idx] = part[key]
            out["ops"] += part["ops"]
    t3 = time.perf_counter()
    out.update({"S": S, "z": z, "rows": rows, "t": tr, "Q": Qr,
                "seconds": {"project": t1 - t0, "global_stats": t2 - t1, "rows": t3 - t2}})
    return out


def block_output(X, Y, Wo, gamma, beta, ln_eps):
    """The block around the layer, in float64: Z = LayerNorm(X + Y Wo) with
    LayerNorm(u) = (u - mean(u)) / sqrt(var(u) + ln_eps) * gamma + beta over each row's d
    features (population variance).  Method page "Gated Local-Global Graph Attention",
    Implementation notes, item 2: "return LayerNorm(X + Wo(g*L+(1-g)*G))"; Wo is a plain
    [H*r, d] matrix (no bias), as the key formulas write the other projections."""
    X = np.asarray(X, dtype=np.float64)
    U = X + np.asarray(Y, dtype=np.float64) @ np.asarray(Wo, dtype=np.float64)
    mean = U.mean(axis=1, keepdims=True)
    var = ((U - mean) ** 2).mean(axis=1, keepdims=True)
    return (U - mean) / np.sqrt(var + ln_eps) * np.asarray(gamma, dtype=np.float64) + \
        np.asarray(beta, dtype=np.float64)


def forward_workload(w, rows=None, csr=None, seg_ptr=None):
    """Oracle forward of a `Workload` (see the package's workloads module)."""
    if csr is None:
        csr = csr_from_coo(w.N, w.src, w.dst)
    return forward(w.N, w.d, w.H, w.r, w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps,
                   csr[0], csr[1], rows, seg_ptr)
