"""Seeded synthetic workloads for the gated local-global graph-attention layer.

This module only draws inputs: a directed edge list (COO, self-loops included), node
features X and the layer parameters.  It holds none of the layer's arithmetic and no
CSR construction, so that the float64 oracle and the CUDA path both start from the same
draws and share nothing else.

Shapes follow the workloads described for the method ("Gated Local-Global Graph
Attention", Mathematical statement and Implementation notes): X [N, d], W_Q/W_K/W_V
[d, H*r], w_g [d], scalar b_g and eps.  An edge (src=j, dst=i) means A_ij = 1, i.e. j is
an in-neighbour of target i.

Every array is float32 or int32.  For bf16 workloads the float32 draws are rounded to the
nearest bf16 (ties to even) here, so the float32 arrays hold exactly the bf16 values that
both sides consume.

Draw order (one numpy PCG64 generator per workload): graph, X, W_Q, W_K, W_V, w_g, b_g.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = ["Workload", "CONFIGS", "make_workload", "round_to_bf16", "chung_lu_weights",
           "make_custom", "uniform_in_neighbours"]


@dataclasses.dataclass
class Workload:
    name: str
    N: int
    d: int
    H: int
    r: int
    io: str                 # "f32" or "bf16"
    src: np.ndarray         # int32 [E]   source node j of each edge
    dst: np.ndarray         # int32 [E]   target node i of each edge
    X: np.ndarray           # float32 [N, d]
    W_Q: np.ndarray         # float32 [d, H*r]
    W_K: np.ndarray
    W_V: np.ndarray
    w_g: np.ndarray         # float32 [d]
    b_g: float
    eps: float
    seed: int = 0

    @property
    def E(self) -> int:
        return int(self.src.shape[0])

    @property
    def D(self) -> int:
        return self.H * self.r

    def degree_stats(self) -> dict:
        deg = np.bincount(self.dst, minlength=self.N)
        return {"E": self.E, "max_in_degree": int(deg.max()) if self.N else 0,
                "mean_in_degree": float(deg.mean()) if self.N else 0.0}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    out = u.astype(np.uint32).view(np.float32)
    # NaN/Inf do not occur in these draws; keep them untouched anyway.
    bad = ~np.isfinite(a)
    if bad.any():
        out = out.copy()
        out[bad] = a[bad]
    return out


def chung_lu_weights(N: int, exponent: float, mean: float, cap: float | None,
                     rng: np.random.Generator) -> np.ndarray:
    """Expected-degree weights w_i proportional to (rank+1)^(-1/(exponent-1)).

    Scaled so that mean(w) == mean after capping at `cap` (a few fixed-point steps), then
    assigned to node ids through a random permutation so that hubs are spread over ids.
    """
    rank = np.arange(1, N + 1, dtype=np.float64)
    base = rank ** (-1.0 / (exponent - 1.0))
    scale = mean * N / base.sum()
    for _ in range(60):
        w = base * scale
        if cap is not None:
            w = np.minimum(w, cap)
        m = w.mean()
        if abs(m - mean) <= 1e-9 * mean:
            break
        scale *= mean / m
    perm = rng.permutation(N)
    out = np.empty(N, dtype=np.float64)
    out[perm] = w
    return out


def _sample_by_weight(rng: np.random.Generator, cdf: np.ndarray, n: int) -> np.ndarray:
    u = rng.random(n) * cdf[-1]
    return np.searchsorted(cdf, u, side="right").astype(np.int64)


def _sorted_unique(keys: np.ndarray) -> np.ndarray:
    """Sorted distinct values (sort-based; numpy's hash path is slow for large int64)."""
    k = np.sort(keys)
    if k.shape[0] == 0:
        return k
    keep = np.empty(k.shape[0], dtype=bool)
    keep[0] = True
    np.not_equal(k[1:], k[:-1], out=keep[1:])
    return k[keep]


def _first_distinct(keys: np.ndarray, want: int) -> np.ndarray:
    """First `want` distinct keys in draw order (or all of them if fewer)."""
    order = np.argsort(keys, kind="stable")
    k = keys[order]
    keep = np.ones(k.shape[0], dtype=bool)
    keep[1:] = k[1:] != k[:-1]
    first = np.sort(order[keep])
    return keys[first[:want]]


def _directed_chung_lu(rng, N, n_edges, w):
    """Distinct directed non-self edges u->v with u, v drawn independently in proportion to w."""
    cdf = np.cumsum(w)
    keys = np.empty(0, dtype=np.int64)
    batch = int(n_edges * 1.3) + 1024
    while True:
        u = _sample_by_weight(rng, cdf, batch)
        v = _sample_by_weight(rng, cdf, batch)
        keep = u != v
        keys = np.concatenate([keys, u[keep] * N + v[keep]])
        sel = _first_distinct(keys, n_edges)
        if sel.shape[0] >= n_edges:
            return sel // N, sel % N
        batch = max(1024, int((n_edges - sel.shape[0]) * 2))


def _undirected_chung_lu(rng, N, n_pairs, w):
    """Distinct undirected non-self pairs {u, v} drawn in proportion to w_u * w_v."""
    cdf = np.cumsum(w)
    keys = np.empty(0, dtype=np.int64)
    batch = int(n_pairs * 1.5) + 1024
    while True:
        u = _sample_by_weight(rng, cdf, batch)
        v = _sample_by_weight(rng, cdf, batch)
        keep = u != v
        a = np.minimum(u[keep], v[keep])
        b = np.maximum(u[keep], v[keep])
        keys = np.concatenate([keys, a * N + b])
        sel = _first_distinct(keys, n_pairs)
        if sel.shape[0] >= n_pairs:
            return sel // N, sel % N
        batch = max(1024, int((n_pairs - sel.shape[0]) * 3))


def _uniform_distinct_neighbours(rng, n_groups, group, k):
    """For every node of each group of `group` consecutive ids: k distinct uniform
    in-neighbours from its own group, excluding itself.  Returns (src, dst)."""
    n = n_groups * group
    keys = rng.random((n, group - 1))
    pick = np.argpartition(keys, k - 1, axis=1)[:, :k] if k < group - 1 else \
        np.tile(np.arange(group - 1), (n, 1))
    pick = np.sort(pick, axis=1)
    node = np.arange(n, dtype=np.int64)
    pos = (node % group)[:, None]
    off = np.where(pick < pos, pick, pick + 1)          # skip the node itself
    src = (node // group)[:, None] * group + off
    dst = np.broadcast_to(node[:, None], src.shape)
    return src.reshape(-1), dst.reshape(-1)


def _skewed_in_degree_graph(rng, N, exponent, mean, cap):
    """Per target i: deg_i ~ Poisson(w_i) capped at `cap`, sources distinct, != i, drawn in
    proportion to w (with-replacement draws, deduplicated, redrawn for the shortfall)."""
    w = chung_lu_weights(N, exponent, mean, cap, rng)
    deg = np.minimum(rng.poisson(w), int(cap)).astype(np.int64)
    cdf = np.cumsum(w)
    have = np.zeros(N, dtype=np.int64)
    keys = np.empty(0, dtype=np.int64)
    need = deg + (deg >> 3) + (deg > 0)
    for _ in range(6):
        tot = int(need.sum())
        if tot == 0:
            break
        dst = np.repeat(np.arange(N, dtype=np.int64), need)
        src = _sample_by_weight(rng, cdf, tot)
        keep = src != dst
        keys = _sorted_unique(np.concatenate([keys, dst[keep] * N + src[keep]]))
        have = np.bincount(keys // N, minlength=N)
        # rows with more distinct sources than asked for (cannot happen) are left as is
        need = np.maximum(deg - have, 0)
        need = np.where(need > 0, 2 * need + 1, 0)
    # trim rows that overshot their target degree (keep the smallest keys: deterministic)
    dst_all = keys // N
    start = np.searchsorted(dst_all, np.arange(N), side="left")
    rank = np.arange(keys.shape[0], dtype=np.int64) - start[dst_all]
    keys = keys[rank < deg[dst_all]]
    return keys % N, keys // N


CONFIGS = {
    # name: (description used in reports)
    "tiny": "N=256, d=32, H=1, r=16; 8 distinct uniform in-neighbours + self-loop; fp32",
    "citation": "N=2708, d=1433 binary BoW (1.27%), 5278 undirected Chung-Lu (gamma 2.5) "
                "edges both ways + self-loops, H=8, r=8; fp32",
    "arxiv": "N=169343, d=128, 1166243 directed Chung-Lu (gamma 2.3) edges symmetrised + "
             "self-loops, H=4, r=32, b_g~N(0,1); bf16",
    "packed": "512 sequences x 256 tokens, d=512, H=8, r=64; 16 uniform in-sequence "
              "in-neighbours + self-loop; bf16",
    "skewed": "N=2^20, d=256, H=8, r=32; Poisson(Chung-Lu gamma 2.1, mean 32, cap 50000) "
              "in-degree + self-loops; bf16",
}


def _params(rng, N, d, D, io, b_g_random, x_kind="normal", x_density=None):
    if x_kind == "bernoulli":
        X = (rng.random((N, d)) < x_density).astype(np.float32)
    else:
        X = rng.standard_normal((N, d), dtype=np.float32)
    std = np.float32(1.0 / np.sqrt(d))
    W_Q = rng.standard_normal((d, D), dtype=np.float32) * std
    W_K = rng.standard_normal((d, D), dtype=np.float32) * std
    W_V = rng.standard_normal((d, D), dtype=np.float32) * std
    w_g = rng.standard_normal((d,), dtype=np.float32) * std
    b_g = float(np.float32(rng.standard_normal())) if b_g_random else 0.0
    if io == "bf16":
        X, W_Q, W_K, W_V, w_g = (round_to_bf16(a) for a in (X, W_Q, W_K, W_V, w_g))
    return X, W_Q, W_K, W_V, w_g, b_g


def _with_self_loops(N, src, dst):
    loop = np.arange(N, dtype=np.int64)
    return (np.concatenate([np.asarray(src, np.int64), loop]).astype(np.int32),
            np.concatenate([np.asarray(dst, np.int64), loop]).astype(np.int32))


def make_workload(name: str, seed: int = 0, scale: float = 1.0) -> Workload:
    """Build one of the named workloads.  `scale` < 1 shrinks N (and the edge count in
    proportion) while keeping the degree distribution's shape; it is used for bounded
    CPU samples and for small ncu captures, never for reported full-size numbers."""
    rng = np.random.default_rng(np.random.PCG64(seed))
    if name == "tiny":
        N, d, H, r, io = max(2, int(256 * scale)), 32, 1, 16, "f32"
        k = min(8, N - 1)
        s, t = _uniform_distinct_neighbours(rng, 1, N, k)
        src, dst = _with_self_loops(N, s, t)
        X, WQ, WK, WV, wg, bg = _params(rng, N, d, H * r, io, False)
    elif name == "citation":
        N, d, H, r, io = max(8, int(2708 * scale)), 1433, 8, 8, "f32"
        pairs = int(round(5278 * N / 2708))
        w = chung_lu_weights(N, 2.5, 3.9, None, rng)
        a, b = _undirected_chung_lu(rng, N, pairs, w)
        src, dst = _with_self_loops(N, np.concatenate([a, b]), np.concatenate([b, a]))
        X, WQ, WK, WV, wg, bg = _params(rng, N, d, H * r, io, False,
                                        x_kind="bernoulli", x_density=0.0127)
    elif name == "arxiv":
        N, d, H, r, io = max(8, int(169343 * scale)), 128, 4, 32, "bf16"
        n_dir = int(round(1166243 * N / 169343))
        w = chung_lu_weights(N, 2.3, 1.0, None, rng)
        u, v = _directed_chung_lu(rng, N, n_dir, w)
        keys = _sorted_unique(np.concatenate([u * N + v, v * N + u]))
        src, dst = _with_self_loops(N, keys // N, keys % N)
        X, WQ, WK, WV, wg, bg = _params(rng, N, d, H * r, io, True)
    elif name == "packed":
        n_seq = max(1, int(512 * scale))
        N, d, H, r, io = n_seq * 256, 512, 8, 64, "bf16"
        s, t = _uniform_distinct_neighbours(rng, n_seq, 256, 16)
        src, dst = _with_self_loops(N, s, t)
        X, WQ, WK, WV, wg, bg = _params(rng, N, d, H * r, io, False)
    elif name == "skewed":
        N, d, H, r, io = max(64, int((1 << 20) * scale)), 256, 8, 32, "bf16"
        s, t = _skewed_in_degree_graph(rng, N, 2.1, 32.0, min(50000.0, N - 1.0))
        src, dst = _with_self_loops(N, s, t)
        X, WQ, WK, WV, wg, bg = _params(rng, N, d, H * r, io, False)
    else:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}")
    eps = 1e-6
    return Workload(name, N, d, H, r, io, src, dst, X, WQ, WK, WV, wg, bg, eps, seed)


def uniform_in_neighbours(N, k, seed):
    """k distinct uniform in-neighbours != i for every node i, plus its self-loop, in O(N k)
    (rows with a repeated draw are redrawn).  Used for size sweeps at fixed degree, where
    the tiny config's exact sampler (quadratic in N) does not scale."""
    rng = np.random.default_rng(np.random.PCG64(seed))
    if N < 2 or k < 1:
        loop = np.arange(N, dtype=np.int32)
        return loop, loop.copy()
    k = min(k, N - 1)
    node = np.arange(N, dtype=np.int64)
    src = np.empty((N, k), dtype=np.int64)
    todo = node
    while todo.size:
        v = rng.integers(0, N - 1, (todo.size, k))
        v = np.where(v >= todo[:, None], v + 1, v)        # skip the node itself
        v.sort(axis=1)
        dup = (v[:, 1:] == v[:, :-1]).any(axis=1) if k > 1 else np.zeros(todo.size, bool)
        src[todo[~dup]] = v[~dup]
        todo = todo[dup]
    dst = np.repeat(node, k)
    src = np.concatenate([src.reshape(-1), node]).astype(np.int32)
    dst = np.concatenate([dst, node]).astype(np.int32)
    return src, dst


def make_custom(N, d, H, r, src, dst, io="f32", seed=0, b_g=0.0, eps=1e-6,
                x_scale=1.0, w_scale=None) -> Workload:
    """A workload on a caller-given edge list (self-loops are NOT added): used for edge
    cases such as empty graphs, isolated rows, complete graphs and duplicate edges."""
    rng = np.random.default_rng(np.random.PCG64(seed))
    X = rng.standard_normal((N, d), dtype=np.float32) * np.float32(x_scale)
    std = np.float32(w_scale if w_scale is not None else 1.0 / np.sqrt(max(d, 1)))
    D = H * r
    W_Q = rng.standard_normal((d, D), dtype=np.float32) * std
    W_K = rng.standard_normal((d, D), dtype=np.float32) * std
    W_V = rng.standard_normal((d, D), dtype=np.float32) * std
    w_g = rng.standard_normal((d,), dtype=np.float32) * std
    if io == "bf16":
        X, W_Q, W_K, W_V, w_g = (round_to_bf16(a) for a in (X, W_Q, W_K, W_V, w_g))
    return Workload("custom", N, d, H, r, io, np.asarray(src, np.int32),
                    np.asarray(dst, np.int32), X, W_Q, W_K, W_V, w_g, float(b_g),
                    float(eps), seed)
