"""Host side of the row-sharded forward on CPU: the row partition, and the whole
begin -> exchange -> end protocol of sharded.ShardedForward on two and three gloo ranks
(one process each).  The ranks' arithmetic is done by a float64 stand-in built from the
oracle (test infrastructure; the product's shards run libglga), so the test checks that
the partition, the padded K/V layout and its all-gather, and the rank-ordered sum of the
partial statistics reproduce the unsharded layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_graph_attention_tcgen05_b200.sharded import (ShardedForward, ShardPlan, block_rows, padded_positions,
                                                         partition_rows, shard_csr)
from sparse_graph_attention_tcgen05_b200.workloads import make_workload


def test_partition_is_contiguous_and_balances_entries():
    w = make_workload("citation")
    rp, _ = oracle.csr_from_coo(w.N, w.src, w.dst)
    for P in (1, 2, 3, 8):
        b = partition_rows(rp, P)
        assert b[0] == 0 and b[-1] == w.N and np.all(np.diff(b) >= 0)
        per = np.diff(rp[b])
        # each block within one row's worth of entries of the ideal share
        assert per.max() - w.E / P <= np.diff(rp).max() + 1
    # more ranks than rows: trailing blocks are empty, nothing is lost
    b = partition_rows(np.array([0, 2, 3, 5]), 6)
    assert b[0] == 0 and b[-1] == 3 and np.all(np.diff(b) >= 0)
    # no edges: rows split evenly
    np.testing.assert_array_equal(partition_rows(np.zeros(11, np.int64), 5), [0, 2, 4, 6, 8, 10])


def test_padded_positions_are_block_offsets():
    bounds = np.array([0, 3, 3, 10, 12])                 # block 1 is empty, B = 7
    assert block_rows(bounds) == 7
    np.testing.assert_array_equal(padded_positions(bounds, np.arange(12)),
                                  [0, 1, 2, 14, 15, 16, 17, 18, 19, 20, 21, 22])
    rp = np.array([0, 2, 2, 5, 6, 6, 6, 7, 9, 9, 10, 11, 12])
    ci = np.array([0, 11, 3, 4, 9, 2, 10, 1, 7, 5, 6, 8])
    rpo, cio = shard_csr(rp, ci, 3, 10, bounds)
    np.testing.assert_array_equal(rpo, [0, 1, 1, 1, 2, 4, 4, 5])
    np.testing.assert_array_equal(cio, padded_positions(bounds, ci[5:10]))
    plan = ShardPlan(rp, ci, 4, 2)
    assert plan.B == block_rows(plan.bounds) and plan.n_kv == 4 * plan.B
    assert plan.kv0 == 2 * plan.B and plan.kv1 - plan.kv0 == plan.b1 - plan.b0


class OracleShard:
    """float64 CPU stand-in for sharded.LibraryShard (same interface; K/V buffer in the
    padded layout of ShardPlan)."""

    def __init__(self, w, plan):
        rp_own, ci_own, b0, b1 = plan.row_ptr, plan.col_idx, plan.kv0, plan.kv1
        self.w, self.b0, self.b1 = w, b0, b1
        self.D = w.H * w.r
        self.kv = torch.full((plan.n_kv, 2 * self.D), float("nan"), dtype=torch.float64)
        self.n_part = w.H * w.r * (w.r + 1)
        self.own = torch.zeros(self.n_part, dtype=torch.float64)
        self.rp, self.ci = rp_own, ci_own

    def begin(self, X_own, W_Q, W_K, W_V, w_g):
        K, V = oracle.project(X_own, W_K), oracle.project(X_own, W_V)
        self.kv[self.b0:self.b1, :self.D] = torch.from_numpy(K)
        self.kv[self.b0:self.b1, self.D:] = torch.from_numpy(V)
        S, z = oracle.global_stats(K, V, self.w.H, self.w.r)
        self.own[:] = torch.from_numpy(np.concatenate([S, z[:, :, None]], axis=2).reshape(-1))
        self.Q, self.t = oracle.project(X_own, W_Q), oracle.gate_logit(X_own, w_g)

    def end(self, partials, b_g, eps, Y=None):
        H, r = self.w.H, self.w.r
        tot = np.zeros(self.n_part)
        for p in range(partials.shape[0]):          # rank order
            tot += partials[p].numpy()
        tot = tot.reshape(H, r, r + 1)
        kv = self.kv.numpy()
        out = oracle.rows_output(np.arange(self.b1 - self.b0), H, r, self.rp, self.ci, self.Q,
                                 kv[:, :self.D], kv[:, self.D:], self.t,
                                 np.ascontiguousarray(tot[:, :, :r]), np.ascontiguousarray(tot[:, :, r]),
                                 b_g, eps)
        return torch.from_numpy(out["Y"])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, name, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = make_workload(name)
        rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
        plan = ShardPlan(rp, ci, world, rank)
        fwd = ShardedForward(OracleShard(w, plan), rank, world)
        Y = fwd(w.X[plan.b0:plan.b1], w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps)
        results[rank] = (plan.b0, plan.b1, Y.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,name", [(2, "tiny"), (3, "citation")])
def test_sharded_protocol_reproduces_the_layer(world, name):
    port = _free_port()
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    w = make_workload(name)
    ref = oracle.forward_workload(w)["Y"]
    got = np.concatenate([results[r][2] for r in range(world)])
    assert [results[r][0] for r in range(world)] == sorted(results[r][0] for r in range(world))
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12)
