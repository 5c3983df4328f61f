"""The backward pass on the GPU (glga_backward) against the float64 reference gradients
of oracle/backward.py (pinned by finite differences of the C oracle).  Tolerances per
gradient tensor, relative to its largest entry: fp32 io 2e-4 (fp32 arithmetic over sums of
up to N terms); bf16 io 3e-2 (the forward's Q, K, V and L are stored in bf16, 2^-9
relative, and every gradient term is a product of two or three of them)."""
import numpy as np
import pytest
import torch

import oracle
from oracle.backward import backward as ref_backward
from oracle.backward import backward_chunked
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_custom, make_workload, round_to_bf16
from tests.gpu_helpers import to_dev

pytestmark = pytest.mark.gpu

TOLB = {"f32": 2e-4, "bf16": 3e-2}
NAMES = ("dX", "dW_Q", "dW_K", "dW_V", "dw_g", "db_g")


def _run(w, dY, options=None):
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    o = options or glga.default_options()
    o.backward = 1
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, o)
    dt = glga.torch_dtype(w.io)
    args = [to_dev(a, dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    layer.forward(*args, b_g=w.b_g, eps=w.eps)
    g1 = layer.backward(*args, w.b_g, w.eps, to_dev(dY, dt))
    g2 = layer.backward(*args, w.b_g, w.eps, to_dev(dY, dt))
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0
    for k in NAMES:                                   # fixed summation order
        assert torch.equal(g1[k], g2[k]), k
    layer.close()
    return {k: v.cpu().numpy().astype(np.float64) for k, v in g1.items()}


def _check(w, seed=0, chunked=False):
    rng = np.random.default_rng(seed)
    dY = rng.standard_normal((w.N, w.D)).astype(np.float32)
    if w.io == "bf16":
        dY = round_to_bf16(dY)
    got = _run(w, dY)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    ref_fn = backward_chunked if chunked else ref_backward
    ref = ref_fn(w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps, rp, ci, w.H, w.r, dY)
    errs = {}
    for k in NAMES:
        r = np.asarray(ref[k], dtype=np.float64).reshape(got[k].shape)
        scale = max(np.abs(r).max(), 1e-30)
        errs[k] = float(np.abs(got[k] - r).max() / scale)
    print(f"\n{w.name} N={w.N} H={w.H} r={w.r} {w.io}: " + ", ".join(f"{k} {e:.2e}" for k, e in errs.items()))
    for k in NAMES:
        assert np.all(np.isfinite(got[k])) and errs[k] <= TOLB[w.io], (k, errs[k])


def test_tiny_fp32():
    _check(make_workload("tiny"))


def test_citation_fp32():
    _check(make_workload("citation"))


def test_arxiv_shape_bf16():
    _check(make_workload("arxiv", scale=0.02))


def test_arxiv_full_size_bf16():
    """The configuration `bench.py --backward` times: the whole arxiv-shaped graph (N =
    169,343, E = 2,474,639; rows of up to 22,812 entries cut into 32-entry chunks; target
    and source sides on two streams), every gradient tensor compared in full with the
    float64 reference taken one group of target rows at a time."""
    _check(make_workload("arxiv"), chunked=True)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_skewed_degrees_and_isolated_rows(io):
    rng = np.random.default_rng(11)
    N = 300
    deg = np.minimum(rng.zipf(1.6, N), 250)
    deg[::7] = 0                                      # isolated targets
    dst = np.repeat(np.arange(N), deg)
    src = rng.integers(0, N, dst.shape[0])
    w = make_custom(N, 24, 2, 32, src.astype(np.int32), dst.astype(np.int32), io=io, seed=3, b_g=0.1)
    _check(w, seed=2)


def test_backward_needs_the_option():
    w = make_workload("tiny")
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx)
    args = [to_dev(a, torch.float32) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    with pytest.raises(glga.GLGAError) as ei:
        layer.backward(*args, w.b_g, w.eps, torch.zeros(w.N, w.D, device="cuda"))
    assert ei.value.status == 1
    layer.close()


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_edgeless_graph(io):
    # no local terms at all: only the global branch and the gate carry gradient
    w = make_custom(70, 16, 2, 8, np.zeros(0, np.int32), np.zeros(0, np.int32), io=io, seed=4, b_g=0.3)
    _check(w, seed=5)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_very_heavy_target_and_source(io):
    # target 7 and source 11 each carry 5,000 entries (157 chunks of 32, the last one
    # ragged), beside a light background of 3 entries per row; H*r = 32 puts one feature
    # on each lane
    rng = np.random.default_rng(8)
    N = 600
    dst = np.concatenate([np.full(5000, 7), rng.integers(0, N, 5000), np.repeat(np.arange(N), 3)])
    src = np.concatenate([rng.integers(0, N, 5000), np.full(5000, 11), rng.integers(0, N, 3 * N)])
    w = make_custom(N, 32, 2, 16, src.astype(np.int32), dst.astype(np.int32), io=io, seed=9, b_g=-0.2)
    _check(w, seed=10)


def test_bf16_rows_not_16_byte_multiples():
    # d = 13: X rows of 26 bytes cannot be loaded by TMA, so this bf16 layer's dW and dX run
    # on the CUDA-core GEMM kernels instead of the tensor-core ones
    rng = np.random.default_rng(21)
    N = 257
    dst = np.concatenate([np.repeat(np.arange(N), 3), np.full(90, 5)])
    src = rng.integers(0, N, dst.shape[0])
    w = make_custom(N, 13, 2, 16, src.astype(np.int32), dst.astype(np.int32), io="bf16", seed=23, b_g=0.4)
    _check(w, seed=24)


@pytest.mark.parametrize("H,r,N", [(8, 16, 1000), (4, 32, 1000), (2, 64, 1000), (4, 32, 40000)])
def test_tensor_core_readout_backward(H, r, N):
    # bf16 layers with H*r = 128 run the readout backward on the tensor cores (one thread
    # per tile row and column half, phi(Q) B_g and dnum blockdiag(S) as tcgen05 MMAs): every
    # head width it takes, a ragged last 128-row tile, and at N = 40,000 more tiles than
    # CTAs (the persistent loop)
    rng = np.random.default_rng(N + r)
    src = np.concatenate([rng.integers(0, N, 4 * N), np.arange(N)]).astype(np.int32)
    dst = np.concatenate([np.repeat(np.arange(N), 4), np.arange(N)]).astype(np.int32)
    w = make_custom(N, 64, H, r, src, dst, io="bf16", seed=N * 3 + H, b_g=0.2)
    _check(w, seed=H, chunked=N > 5000)


@pytest.mark.parametrize("H,r,N", [(8, 16, 100), (2, 64, 300), (4, 32, 148 * 128 + 77)])
def test_one_pass_dx_dw(H, r, N):
    # bf16 layers with d = 128 and H*r = 128 form dX, dW, dw_g and db_g in one tensor-core
    # pass over the bf16 copy of dZ that the gather kernels write (dX and the whole dW
    # block in TMEM together): every head width, a single ragged 128-row tile (rows without
    # in-edges among them), and more tiles than thread blocks with a ragged last one
    rng = np.random.default_rng(N + H)
    src = np.concatenate([rng.integers(0, N, 3 * N), np.arange(N)]).astype(np.int32)
    dst = np.concatenate([np.repeat(np.arange(N), 3), np.arange(N)]).astype(np.int32)
    w = make_custom(N, 128, H, r, src, dst, io="bf16", seed=N + 7, b_g=-0.1)
    _check(w, seed=r, chunked=N > 5000)


def test_duplicate_edges_heavy_rows_and_isolated_rows_bf16():
    # the tensor-core layer shape (H*r = 128, d = 128) on a graph with repeated entries
    # (the (p, ds) hand-over maps each repeat to its own transposed position), a target and
    # a source row of 300 entries each (64-edge chunks, the last one ragged), and rows
    # with no entries at all on either side
    rng = np.random.default_rng(31)
    N = 700
    dst = np.concatenate([np.full(300, 5), rng.integers(0, N, 300), np.repeat(np.arange(0, N, 3), 2)])
    src = np.concatenate([rng.integers(0, N, 300), np.full(300, 9), np.repeat(np.arange(0, N, 3), 2)[::-1]])
    keep = (dst % 7 != 3) & (src % 11 != 4)            # rows without in- or out-entries
    w = make_custom(N, 128, 4, 32, src[keep].astype(np.int32), dst[keep].astype(np.int32), io="bf16",
                    seed=32, b_g=0.05)
    _check(w, seed=33)
