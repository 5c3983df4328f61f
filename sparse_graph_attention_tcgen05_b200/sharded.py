"""Row-sharded forward of the layer across ranks: one process per GPU, torch.distributed
(NCCL over NVLink / NVSwitch) for the one exchange step.

The target rows are cut into contiguous blocks with about equal numbers of CSR entries
(the local branch's work is proportional to them).  Rank p owns rows
[bounds[p], bounds[p+1]).  In the K/V buffer every rank holds, the rows of rank p sit at
positions p*B .. p*B + (bounds[p+1] - bounds[p]) - 1, B the largest block, so that one
all-gather of equal blocks moves every rank's rows (the CSR column ids of each shard are
remapped to those positions; the padding rows are never read).  One forward is

  1. begin: the rank projects its own rows (q, gate logit; k, v into its block of the
     K/V buffer) and sums its partial global statistics S_p | z_p;
  2. exchange: one all-gather of the K/V blocks into every rank's buffer (in place) and
     one all-gather of the partials (method page "Gated Local-Global Graph Attention",
     "Key formulas": S and z are sums over all nodes, so they split into per-rank
     partial sums);
  3. end: the partials are summed in rank order (the same order on every rank), then the
     local branch and the readout produce the rank's own rows of Y.

Steps 1 and 3 run in libglga (glga_forward_begin / glga_forward_end); this module only
partitions rows, owns the exchange buffers and issues the collectives.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch
import torch.distributed as dist

from . import glga


def partition_rows(row_ptr, P: int) -> np.ndarray:
    """Boundaries [P + 1] of P contiguous row blocks with about equal CSR entries each:
    block p ends at the first row whose offset reaches (p+1)/P of the entries.  With no
    entries the rows are split evenly."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    N = row_ptr.shape[0] - 1
    E = int(row_ptr[-1])
    if P < 1:
        raise ValueError("need at least one rank")
    if E == 0:
        return np.round(np.linspace(0, N, P + 1)).astype(np.int64)
    targets = (np.arange(P + 1, dtype=np.int64) * E) // P
    b = np.searchsorted(row_ptr, targets, side="left").astype(np.int64)
    b[0], b[-1] = 0, N
    return np.maximum.accumulate(np.minimum(b, N))


def shard_csr(row_ptr, col_idx, b0: int, b1: int, bounds=None):
    """The CSR of rows [b0, b1) with local row numbering and global column ids, or, given
    the partition `bounds`, column ids remapped to K/V buffer positions (padded_positions)."""
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    rp = (row_ptr[b0:b1 + 1] - row_ptr[b0]).astype(np.int32)
    ci = np.asarray(col_idx)[row_ptr[b0]:row_ptr[b1]].astype(np.int64)
    if bounds is not None:
        ci = padded_positions(bounds, ci)
    return rp, ci.astype(np.int32)


def block_rows(bounds) -> int:
    """B: the rows of the largest block (at least 1), the stride of the K/V blocks."""
    b = np.asarray(bounds, dtype=np.int64)
    return max(1, int(np.diff(b).max())) if b.shape[0] > 1 else 1


def padded_positions(bounds, nodes):
    """Position of each node in the K/V buffer: owner p's block starts at p * B."""
    b = np.asarray(bounds, dtype=np.int64)
    nodes = np.asarray(nodes, dtype=np.int64)
    owner = np.searchsorted(b, nodes, side="right") - 1
    return owner * block_rows(b) + (nodes - b[owner])


class ShardPlan:
    """Rank `rank`'s part of a P-way row partition: its rows [b0, b1), their K/V positions
    [kv0, kv1), the K/V buffer's rows (P * B) and its CSR with remapped column ids."""

    def __init__(self, row_ptr, col_idx, P: int, rank: int, bounds=None):
        self.bounds = partition_rows(row_ptr, P) if bounds is None else np.asarray(bounds, dtype=np.int64)
        assert self.bounds.shape[0] == P + 1
        self.B = block_rows(self.bounds)
        self.n_kv = P * self.B
        self.b0, self.b1 = int(self.bounds[rank]), int(self.bounds[rank + 1])
        self.kv0 = rank * self.B
        self.kv1 = self.kv0 + (self.b1 - self.b0)
        self.row_ptr, self.col_idx = shard_csr(row_ptr, col_idx, self.b0, self.b1, self.bounds)


class LibraryShard:
    """One rank's part of the layer in libglga (glga_create_sharded): owns the K/V buffer
    [N, 2*H*r] that the exchange fills (N = P * B rows in the padded layout, the rank's own
    rows at [b0, b1)), and the rank's partial statistics."""

    def __init__(self, N, d, H, r, io, row_ptr_own, col_idx_own, b0, b1, device=None,
                 options=None, stream=None):
        device = torch.device("cuda") if device is None else device
        self.N, self.d, self.H, self.r, self.io = int(N), int(d), int(H), int(r), io
        self.b0, self.b1 = int(b0), int(b1)
        self.dtype = glga.torch_dtype(io)
        self.kv = torch.empty(self.N, 2 * self.H * self.r, dtype=self.dtype, device=device)
        self.n_part = self.H * self.r * (self.r + 1)
        self.own = torch.zeros(self.n_part, dtype=torch.float32, device=device)
        rp = torch.from_numpy(np.ascontiguousarray(row_ptr_own, dtype=np.int32)).to(device)
        ci = torch.from_numpy(np.ascontiguousarray(col_idx_own, dtype=np.int32)).to(device)
        E = int(ci.numel())
        h = ctypes.c_void_p()
        opt = ctypes.byref(options) if options is not None else None
        glga._check(glga.lib().glga_create_sharded(
            ctypes.byref(h), self.N, self.b0, self.b1, self.d, self.H, self.r,
            glga.GLGA_F32 if io == "f32" else glga.GLGA_BF16, rp.data_ptr(),
            ci.data_ptr() if E else None, E, self.kv.data_ptr(), opt, glga._stream(stream)),
            "glga_create_sharded")
        self._h = h

    def begin(self, X_own, W_Q, W_K, W_V, w_g, stream=None):
        glga._check(glga.lib().glga_forward_begin(
            self._h, glga._ptr(X_own), glga._ptr(W_Q), glga._ptr(W_K), glga._ptr(W_V),
            glga._ptr(w_g), self.own.data_ptr(), glga._stream(stream)), "glga_forward_begin")

    def end(self, partials, b_g, eps, Y=None, stream=None):
        if Y is None:
            Y = torch.empty(self.b1 - self.b0, self.H * self.r, dtype=self.dtype, device=self.kv.device)
        glga._check(glga.lib().glga_forward_end(
            self._h, partials.data_ptr(), int(partials.shape[0]), float(b_g), float(eps),
            glga._ptr(Y), glga._stream(stream)), "glga_forward_end")
        return Y

    def last_device_error(self, stream=None) -> int:
        return int(glga.lib().glga_last_device_error(self._h, glga._stream(stream)))

    def set_timing(self, enable: bool):
        glga._check(glga.lib().glga_set_timing(self._h, 1 if enable else 0), "glga_set_timing")

    def stage_times(self) -> dict:
        ms = (ctypes.c_float * 6)()
        n = ctypes.c_int32()
        glga._check(glga.lib().glga_stage_times(self._h, ms, 6, ctypes.byref(n)), "glga_stage_times")
        return {glga.STAGES[i]: float(ms[i]) for i in range(n.value)}

    def kernel_launches(self) -> int:
        n = ctypes.c_int64()
        glga._check(glga.lib().glga_kernel_launches(self._h, ctypes.byref(n)), "glga_kernel_launches")
        return int(n.value)

    def close(self):
        if getattr(self, "_h", None):
            glga.lib().glga_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ShardedForward:
    """begin -> exchange -> end for one rank.  `shard` provides begin(X_own, ...),
    end(partials, b_g, eps) -> Y_own, the K/V buffer `kv` [world * B, 2D] in the padded
    layout (its own rows in block `rank`) and the partial `own` [n_part].  Every rank
    issues the same collectives in the same order."""

    def __init__(self, shard, rank: int, world: int, group=None):
        self.shard, self.rank, self.world, self.group = shard, rank, world, group
        assert shard.kv.shape[0] % world == 0
        self.B = shard.kv.shape[0] // world
        # flat [world * n_part] for the all-gather, viewed as [world, n_part] (rank order)
        self._flat = torch.empty(world * shard.n_part, dtype=shard.own.dtype, device=shard.own.device)
        self.partials = self._flat.view(world, shard.n_part)

    def exchange(self):
        dist.all_gather_into_tensor(self._flat, self.shard.own, group=self.group)
        own = self.shard.kv[self.rank * self.B:(self.rank + 1) * self.B]
        dist.all_gather_into_tensor(self.shard.kv, own, group=self.group)   # in place

    def __call__(self, X_own, W_Q, W_K, W_V, w_g, b_g, eps, Y=None):
        self.shard.begin(X_own, W_Q, W_K, W_V, w_g)
        self.exchange()
        return self.shard.end(self.partials, b_g, eps, Y)
