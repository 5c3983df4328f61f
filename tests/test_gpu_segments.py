"""Segmented (batched) layers on the GPU against the oracle: every contiguous node range
has its own global statistics S, z (method page "Gated Local-Global Graph Attention",
Implementation notes: X [batch, N, d]).  Covers tile-aligned segments (the packed token
layout), segments that start inside a 128-row readout tile (the fix-up path), empty and
one-node segments, several head groups, and one segment equal to the plain layer."""
import numpy as np
import pytest
import torch

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_custom, make_workload
from tests.gpu_helpers import TOL, assert_close_to_oracle, to_dev

pytestmark = pytest.mark.gpu


def _run(w, seg, options=None):
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, options, segments=seg)
    args = [to_dev(a, glga.torch_dtype(w.io)) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    Y = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0
    inter = layer.intermediates()
    layer.close()
    return Y, inter


def _oracle(w, seg):
    return oracle.forward_workload(w, csr=oracle.csr_from_coo(w.N, w.src, w.dst), seg_ptr=seg)


def _check_stats(w, inter, ref):
    S, z = inter["S"].cpu().numpy(), inter["z"].cpu().numpy()
    assert S.shape == ref["S"].shape and z.shape == ref["z"].shape
    tol = 1e-5 if w.io == "f32" else 2e-2
    for k in range(S.shape[0]):
        sc = max(np.abs(ref["S"][k]).max(), 1e-30)
        assert np.abs(S[k] - ref["S"][k]).max() <= tol * sc, k
        zc = max(np.abs(ref["z"][k]).max(), 1e-30)
        assert np.abs(z[k] - ref["z"][k]).max() <= tol * zc, k


def test_packed_sequences_each_with_their_own_statistics():
    w = make_workload("packed", scale=0.04)          # 20 sequences of 256 tokens
    seg = np.arange(0, w.N + 1, 256, dtype=np.int64)
    Y, inter = _run(w, seg)
    ref = _oracle(w, seg)
    assert_close_to_oracle(w, Y, ref)
    _check_stats(w, inter, ref)
    # the per-sequence statistics differ from the whole-batch ones: the segmented
    # result is not the plain layer's
    plain = oracle.forward_workload(w)
    assert np.abs(plain["Y"] - ref["Y"]).max() > 3 * TOL[w.io] * np.abs(ref["Y"]).max()


def _unaligned(io, H, r, seed, sizes):
    rng = np.random.default_rng(seed)
    N = int(sum(sizes))
    seg = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    src, dst = [], []
    for k in range(len(sizes)):
        a, b = int(seg[k]), int(seg[k + 1])
        if b == a:
            continue
        n = b - a
        deg = rng.integers(0, 12, n)
        t = np.repeat(np.arange(a, b), deg)
        src.append(rng.integers(a, b, t.shape[0])); dst.append(t)
        src.append(np.arange(a, b)); dst.append(np.arange(a, b))
    # a few edges across segments: the local branch follows the graph, the statistics
    # stay per segment
    x = rng.integers(0, N, 40)
    src.append(x); dst.append(rng.integers(0, N, 40))
    src = np.concatenate(src).astype(np.int32)
    dst = np.concatenate(dst).astype(np.int32)
    w = make_custom(N, 20, H, r, src, dst, io=io, seed=seed + 1, b_g=-0.4)
    return w, seg


@pytest.mark.parametrize("io,H,r", [("f32", 2, 32), ("bf16", 2, 32), ("f32", 8, 8),
                                    ("bf16", 4, 64), ("bf16", 16, 16)])
def test_segments_inside_tiles(io, H, r):
    sizes = [100, 0, 1, 300, 27, 128, 5, 0, 260, 3, 90]
    w, seg = _unaligned(io, H, r, seed=7, sizes=sizes)
    Y, inter = _run(w, seg)
    ref = _oracle(w, seg)
    assert_close_to_oracle(w, Y, ref)
    _check_stats(w, inter, ref)


@pytest.mark.parametrize("io,H,r", [("bf16", 2, 32), ("f32", 8, 8), ("bf16", 4, 64)])
def test_many_tiny_segments(io, H, r):
    # every non-empty segment fits one statistics range: the statistics kernel writes each
    # segment's S, z and readout operand itself (no reduction pass); empty segments too
    rng = np.random.default_rng(3)
    sizes = rng.integers(0, 8, 400)
    w, seg = _unaligned(io, H, r, seed=9, sizes=sizes)
    Y, inter = _run(w, seg)
    ref = _oracle(w, seg)
    assert_close_to_oracle(w, Y, ref)
    _check_stats(w, inter, ref)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_one_segment_is_the_plain_layer(io):
    w, _ = _unaligned(io, 2, 32, seed=11, sizes=[700])
    Y1, _ = _run(w, np.array([0, w.N], dtype=np.int64))
    Y0, _ = _run(w, None)
    assert torch.equal(Y0.cpu(), Y1.cpu())
