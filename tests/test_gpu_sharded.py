"""Row-sharded forward on the GPU (glga_create_sharded, glga_forward_begin/end).

With one GPU the ranks are emulated one after another in this process: every shard runs
its begin phase, the test copies each owner's block of K/V rows (the padded layout of
sharded.ShardPlan) into every other shard's buffer and stacks the partial statistics in
rank order (what the two NCCL all-gathers do between processes), then every shard runs
its end phase.  No kernel waits on another
rank.  A one-rank NCCL process group runs sharded.ShardedForward's real collectives."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.sharded import LibraryShard, ShardedForward, ShardPlan, partition_rows
from sparse_graph_attention_tcgen05_b200.workloads import make_workload
from tests.gpu_helpers import assert_close_to_oracle, run_gpu, to_dev

pytestmark = pytest.mark.gpu


def _emulate(w, bounds, csr):
    rp, ci = csr
    P = len(bounds) - 1
    dt = glga.torch_dtype(w.io)
    W = [to_dev(a, dt) for a in (w.W_Q, w.W_K, w.W_V, w.w_g)]
    shards, plans = [], []
    for p in range(P):
        plan = ShardPlan(rp, ci, P, p, bounds=bounds)
        sh = LibraryShard(plan.n_kv, w.d, w.H, w.r, w.io, plan.row_ptr, plan.col_idx, plan.kv0, plan.kv1)
        sh.kv.fill_(float("nan"))                            # padding rows are never read
        sh.begin(to_dev(w.X[plan.b0:plan.b1], dt), *W)
        shards.append(sh)
        plans.append(plan)
    torch.cuda.synchronize()
    for plan, owner in zip(plans, shards):                   # the K/V exchange
        a, b = plan.kv0, plan.kv1
        for other in shards:
            if other is not owner and b > a:
                other.kv[a:b].copy_(owner.kv[a:b])
    partials = torch.stack([sh.own for sh in shards])        # the partials, rank order
    Ys = [sh.end(partials, w.b_g, w.eps) for sh in shards]
    torch.cuda.synchronize()
    for sh in shards:
        assert sh.last_device_error() == 0
        sh.close()
    return torch.cat(Ys)


@pytest.mark.parametrize("name,P", [("tiny", 2), ("citation", 3), ("arxiv", 4)])
def test_emulated_ranks_match_the_oracle(name, P):
    w = make_workload(name, scale=0.05 if name == "arxiv" else 1.0)
    csr = oracle.csr_from_coo(w.N, w.src, w.dst)
    Y = _emulate(w, partition_rows(csr[0], P), csr)
    ref = oracle.forward_workload(w, csr=csr)
    assert_close_to_oracle(w, Y, ref)
    plain = run_gpu(w, csr=csr)["Y"]
    scale = float(plain.float().abs().max())
    tol = 1e-5 if w.io == "f32" else 2e-2
    assert float((Y.float() - plain.float()).abs().max()) <= tol * scale


def test_a_rank_without_rows():
    w = make_workload("citation")
    csr = oracle.csr_from_coo(w.N, w.src, w.dst)
    bounds = np.array([0, 0, 1000, w.N])
    Y = _emulate(w, bounds, csr)
    assert_close_to_oracle(w, Y, oracle.forward_workload(w, csr=csr))


def test_sharded_context_refuses_the_one_shot_forward():
    w = make_workload("tiny")
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    sh = LibraryShard(w.N, w.d, w.H, w.r, w.io, rp, ci, 0, w.N)
    dt = glga.torch_dtype(w.io)
    args = [to_dev(a, dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    Y = torch.empty(w.N, w.D, dtype=dt, device="cuda")
    st = glga.lib().glga_forward(sh._h, *(a.data_ptr() for a in args), 0.0, 1e-6, Y.data_ptr(), None)
    assert st == 1
    sh.close()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("io_name", ["tiny", "arxiv"])
def test_one_rank_nccl_group_equals_the_plain_layer(io_name):
    w = make_workload(io_name, scale=0.05 if io_name == "arxiv" else 1.0)
    csr = oracle.csr_from_coo(w.N, w.src, w.dst)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        plan = ShardPlan(csr[0], csr[1], 1, 0)
        sh = LibraryShard(plan.n_kv, w.d, w.H, w.r, w.io, plan.row_ptr, plan.col_idx, plan.kv0, plan.kv1)
        dt = glga.torch_dtype(w.io)
        fwd = ShardedForward(sh, 0, 1)
        Y = fwd(*(to_dev(a, dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)), w.b_g, w.eps)
        torch.cuda.synchronize()
        assert sh.last_device_error() == 0
        sh.close()
    finally:
        dist.destroy_process_group()
    plain = run_gpu(w, csr=csr)["Y"]
    assert torch.equal(Y.cpu(), plain.cpu())
