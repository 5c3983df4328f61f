"""Pins of the float64 oracle to things other than itself.

Each test checks the oracle against a value the pages print, a closed form, a library
routine, a dense brute force written in a different form (N x N masked matrices), or an
invariant the mathematics fixes.  Together they are chosen so that a dropped term, a
wrong sign or index, or a transposed operand in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from sparse_graph_attention_tcgen05_b200.workloads import make_custom, make_workload
from tests.conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# ------------------------------------------------------------------------------------
# dense brute force: N x N masked scores, library softmax, explicit quadratic form for G
# ------------------------------------------------------------------------------------
def dense_reference(w):
    """Y from dense matrices.  The adjacency is an N x N count matrix (a duplicate edge
    counts twice), the local branch is a masked softmax over each target's row done with
    scipy's softmax, and the global branch is the un-reassociated quadratic form
    sum_j phi(q_i).phi(k_j) v_j / (sum_j phi(q_i).phi(k_j) + eps)."""
    N, H, r = w.N, w.H, w.r
    X = w.X.astype(np.float64)
    Q = X @ w.W_Q.astype(np.float64)
    K = X @ w.W_K.astype(np.float64)
    V = X @ w.W_V.astype(np.float64)
    t = X @ w.w_g.astype(np.float64)
    A = np.zeros((N, N))
    np.add.at(A, (w.dst.astype(np.int64), w.src.astype(np.int64)), 1.0)
    phiQ = np.where(Q > 0, Q + 1, np.exp(np.minimum(Q, 0)))
    phiK = np.where(K > 0, K + 1, np.exp(np.minimum(K, 0)))
    Y = np.zeros((N, H * r))
    L = np.zeros((N, H * r))
    G = np.zeros((N, H * r))
    for h in range(H):
        sl = slice(h * r, (h + 1) * r)
        scores = Q[:, sl] @ K[:, sl].T / math.sqrt(r)
        has = A.sum(1) > 0
        logits = np.where(A > 0, scores + np.log(np.where(A > 0, A, 1.0)), -np.inf)
        P = np.zeros_like(scores)
        P[has] = scipy.special.softmax(logits[has], axis=1)
        L[:, sl] = P @ V[:, sl]
        kern = phiQ[:, sl] @ phiK[:, sl].T              # N x N, phi(q_i).phi(k_j)
        G[:, sl] = (kern @ V[:, sl]) / (kern.sum(1, keepdims=True) + w.eps)
    g = 1.0 / (1.0 + np.exp(-(t + w.b_g)))
    Y = g[:, None] * L + (1 - g[:, None]) * G
    return {"Y": Y, "L": L, "G": G, "g": g}


def run_oracle(w, rows=None):
    return oracle.forward_workload(w, rows=rows)


def rand_graph(N, k, seed, self_loops=True):
    rng = np.random.default_rng(seed)
    src, dst = [], []
    for i in range(N):
        c = rng.choice(N, size=min(k, N), replace=False)
        for j in c:
            if j != i:
                src.append(j); dst.append(i)
        if self_loops:
            src.append(i); dst.append(i)
    return np.array(src, np.int32), np.array(dst, np.int32)


# ------------------------------------------------------------------------------------
# page witnesses
# ------------------------------------------------------------------------------------
def witness_workload(H):
    src = np.array([0, 1], np.int32)
    dst = np.array([2, 2], np.int32)
    w = make_custom(3, 1, H, 1, src, dst, b_g=1e4)
    w.X = np.array([[1.0], [-1.0], [1.0]], np.float32)
    if H == 1:
        w.W_Q = np.array([[1.0]], np.float32)
        w.W_K = np.array([[0.6]], np.float32)
        w.W_V = np.array([[1.0]], np.float32)
    else:
        w.W_Q = np.array([[1.0, -1.0]], np.float32)
        w.W_K = np.array([[0.6, 0.6]], np.float32)
        w.W_V = np.array([[1.0, 1.0]], np.float32)
    w.w_g = np.zeros(1, np.float32)
    return w


def test_single_head_witness_loss():
    gold = read_golden("tinymesh_witnesses.txt")
    out = run_oracle(witness_workload(1))
    y2 = out["Y"][2, 0]
    loss = (1.0 - y2) ** 2
    assert round(loss, 6) == gold["single_head_initial_loss"]
    # isolated rows 0 and 1: empty weighted sum, and Y = L because the gate is saturated
    assert out["L"][0, 0] == 0.0 and out["L"][1, 0] == 0.0


def test_two_head_witness_and_head_permutation():
    gold = read_golden("tinymesh_witnesses.txt")
    w = witness_workload(2)
    out = run_oracle(w)
    y = out["Y"][2]
    loss = ((1.0 - y[0]) ** 2 + (-1.0 - y[1]) ** 2) / 2
    assert round(loss, 6) == gold["two_head_initial_loss"]
    assert y[0] == pytest.approx(-y[1], abs=1e-15)
    # swapping the heads' parameters swaps only the output columns
    w2 = witness_workload(2)
    w2.W_Q = w2.W_Q[:, ::-1].copy()
    out2 = run_oracle(w2)
    np.testing.assert_allclose(out2["Y"][:, ::-1], out["Y"], rtol=0, atol=1e-15)


def test_cost_proxy_ratio():
    """The local loop does exactly |E| * r score multiply-adds per head (no N^2 work);
    with |E|/N = 8 and r = 16 the page's printed ratios come out."""
    gold = read_golden("glga_cost_proxy.txt")
    for N in (64, 512):
        rng = np.random.default_rng(N)
        src = np.concatenate([rng.choice(np.delete(np.arange(N), i), 8, replace=False)
                              for i in range(N)]).astype(np.int32)
        dst = np.repeat(np.arange(N), 8).astype(np.int32)
        w = make_custom(N, 4, 1, 16, src, dst)
        out = run_oracle(w)
        E = src.shape[0]
        assert out["ops"][0] == E * 16 and out["ops"][1] == E * 16
        assert out["ops"][2] == N * 16 * 17
        ratio = N * N * 16 / (out["ops"][0] + N * 16 * 16)
        assert round(ratio, 2) == gold[str(N)]


# ------------------------------------------------------------------------------------
# dense brute force, complete graph, closed forms
# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("seed,N,H,r,k", [(0, 17, 1, 8, 4), (1, 40, 3, 8, 6), (2, 64, 2, 16, 9)])
def test_matches_dense_masked_bruteforce(seed, N, H, r, k):
    src, dst = rand_graph(N, k, seed)
    w = make_custom(N, 12, H, r, src, dst, seed=seed, b_g=0.3)
    out = run_oracle(w)
    ref = dense_reference(w)
    for key in ("L", "G", "g", "Y"):
        np.testing.assert_allclose(out[key], ref[key], rtol=1e-12, atol=1e-12)


def test_tiny_config_matches_bruteforce():
    w = make_workload("tiny")
    out = run_oracle(w)
    ref = dense_reference(w)
    np.testing.assert_allclose(out["Y"], ref["Y"], rtol=1e-11, atol=1e-12)


def test_complete_graph_is_dense_attention():
    """A complete graph with self-loops gives per-head softmax(QK^T/sqrt r) V, computed
    here with torch's scaled_dot_product_attention (no mask)."""
    N, H, r, d = 24, 2, 8, 10
    ii, jj = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    w = make_custom(N, d, H, r, jj.reshape(-1), ii.reshape(-1), seed=5, b_g=1e4)
    out = run_oracle(w)
    X = torch.tensor(w.X, dtype=torch.float64)
    q = (X @ torch.tensor(w.W_Q, dtype=torch.float64)).view(N, H, r).transpose(0, 1)
    k = (X @ torch.tensor(w.W_K, dtype=torch.float64)).view(N, H, r).transpose(0, 1)
    v = (X @ torch.tensor(w.W_V, dtype=torch.float64)).view(N, H, r).transpose(0, 1)
    att = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0]
    ref = att.transpose(0, 1).reshape(N, H * r).numpy()
    np.testing.assert_allclose(out["L"], ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out["Y"], ref, rtol=1e-12, atol=1e-13)  # gate saturated


def test_self_loop_only_node_returns_its_value():
    N = 9
    src = np.array([3, 5, 1, 4], np.int32)       # node 4 has only its self-loop
    dst = np.array([0, 0, 2, 4], np.int32)
    w = make_custom(N, 6, 2, 8, src, dst, seed=3)
    out = run_oracle(w)
    V = w.X.astype(np.float64) @ w.W_V.astype(np.float64)
    np.testing.assert_allclose(out["L"][4], V[4], rtol=1e-14, atol=1e-15)
    # a single in-neighbour gets weight one as well
    np.testing.assert_allclose(out["L"][2], V[1], rtol=1e-14, atol=1e-15)
    # isolated rows get L = 0 and Y = (1 - g) G
    for i in (1, 3, 5, 6, 7, 8):
        assert np.all(out["L"][i] == 0.0)
        np.testing.assert_allclose(out["Y"][i], (1 - out["g"][i]) * out["G"][i], rtol=1e-15)


def test_equal_values_give_weights_summing_to_one():
    """If every v_j is the same vector v, L_i = v for every target with an edge (the
    softmax weights sum to one) and G_i = v * (phi.z)/(phi.z + eps)."""
    N, d, H, r = 30, 5, 2, 8
    src, dst = rand_graph(N, 5, 7)
    w = make_custom(N, d, H, r, src, dst, seed=7)
    w.X[:, 0] = 1.5
    w.W_V[1:, :] = 0.0
    v = 1.5 * w.W_V[0].astype(np.float64)
    out = run_oracle(w)
    np.testing.assert_allclose(out["L"], np.broadcast_to(v, out["L"].shape), rtol=1e-13)
    Q = w.X.astype(np.float64) @ w.W_Q.astype(np.float64)
    for h in range(H):
        sl = slice(h * r, (h + 1) * r)
        phq = np.where(Q[:, sl] > 0, Q[:, sl] + 1, np.exp(np.minimum(Q[:, sl], 0)))
        qz = phq @ out["z"][h]
        np.testing.assert_allclose(out["G"][:, sl], v[sl][None, :] * (qz / (qz + w.eps))[:, None],
                                   rtol=1e-12)


def test_gate_saturation_selects_branches():
    N = 20
    src, dst = rand_graph(N, 4, 11)
    w = make_custom(N, 7, 2, 8, src, dst, seed=11, b_g=1e4)
    out = run_oracle(w)
    assert np.all(out["Y"] == out["L"])
    w.b_g = -1e4
    out = run_oracle(w)
    assert np.all(out["Y"] == out["G"])


def test_gate_value_closed_form():
    N = 6
    src, dst = rand_graph(N, 2, 2)
    w = make_custom(N, 3, 1, 8, src, dst, seed=2, b_g=-0.7)
    out = run_oracle(w)
    t = w.X.astype(np.float64) @ w.w_g.astype(np.float64)
    np.testing.assert_allclose(out["g"], scipy.special.expit(t - 0.7), rtol=1e-14)


def test_phi_is_elu_plus_one():
    xs = torch.tensor([-30.0, -2.5, -1e-3, 0.0, 1e-3, 0.7, 4.0], dtype=torch.float64)
    ref = torch.nn.functional.elu(xs, alpha=1.0) + 1.0
    for x, y in zip(xs.tolist(), ref.tolist()):
        # elu(x) + 1 = expm1(x) + 1 cancels for x << 0, so allow one ulp of 1.0 there
        assert oracle.phi(x) == pytest.approx(y, rel=1e-15, abs=2.3e-16)
    assert oracle.phi(-30.0) == pytest.approx(math.exp(-30.0), rel=1e-15)


def test_global_stats_against_einsum_and_graph_independence():
    N, H, r = 50, 3, 8
    rng = np.random.default_rng(4)
    K = rng.standard_normal((N, H * r)); V = rng.standard_normal((N, H * r))
    S, z = oracle.global_stats(K, V, H, r)
    pk = torch.nn.functional.elu(torch.tensor(K)).numpy() + 1.0
    for h in range(H):
        sl = slice(h * r, (h + 1) * r)
        np.testing.assert_allclose(S[h], np.einsum("ja,jc->ac", pk[:, sl], V[:, sl]), rtol=1e-13)
        np.testing.assert_allclose(z[h], pk[:, sl].sum(0), rtol=1e-13)
    # node order does not matter (up to rounding of the sum order)
    p = rng.permutation(N)
    S2, z2 = oracle.global_stats(K[p], V[p], H, r)
    np.testing.assert_allclose(S2, S, rtol=1e-12); np.testing.assert_allclose(z2, z, rtol=1e-12)


def test_reassociation_error_small():
    """The page verified linear-kernel reassociation below 2.4e-7 (fp32); in float64 the
    reassociated readout and the quadratic form agree to ~1e-15 relative."""
    w = make_workload("tiny")
    out = run_oracle(w)
    ref = dense_reference(w)
    err = np.abs(out["G"] - ref["G"]).max() / np.abs(ref["G"]).max()
    assert err < 1e-12


def test_large_scores_stable_and_hard_argmax():
    N, H, r = 25, 1, 8
    src, dst = rand_graph(N, 6, 9)
    w = make_custom(N, 8, H, r, src, dst, seed=9, b_g=1e4)
    w.W_Q = w.W_Q * np.float32(300.0)
    out = run_oracle(w)
    assert np.all(np.isfinite(out["Y"]))
    X = w.X.astype(np.float64)
    Q, K, V = X @ w.W_Q.astype(np.float64), X @ w.W_K.astype(np.float64), X @ w.W_V.astype(np.float64)
    rp, ci = oracle.csr_from_coo(N, w.src, w.dst)
    for i in range(N):
        js = ci[rp[i]:rp[i + 1]]
        s = Q[i] @ K[js].T / math.sqrt(r)
        top = np.sort(s)[::-1]
        if len(js) > 1 and top[0] - top[1] > 40:           # clear winner: e^-40 ~ 4e-18
            np.testing.assert_allclose(out["L"][i], V[js[np.argmax(s)]], rtol=1e-9, atol=1e-9)


def test_vertex_permutation_permutes_rows():
    N = 35
    src, dst = rand_graph(N, 5, 21)
    w = make_custom(N, 9, 2, 8, src, dst, seed=21, b_g=0.2)
    out = run_oracle(w)
    p = np.random.default_rng(1).permutation(N)          # new id of old node i is p[i]
    inv = np.argsort(p)
    w2 = make_custom(N, 9, 2, 8, p[src], p[dst], seed=21, b_g=0.2)
    w2.X = w.X[inv].copy(); w2.W_Q, w2.W_K, w2.W_V, w2.w_g = w.W_Q, w.W_K, w.W_V, w.w_g
    out2 = run_oracle(w2)
    np.testing.assert_allclose(out2["Y"][p], out["Y"], rtol=1e-12, atol=1e-14)


def test_heads_are_independent():
    N, r = 30, 8
    src, dst = rand_graph(N, 5, 13)
    w = make_custom(N, 6, 3, r, src, dst, seed=13, b_g=0.1)
    out = run_oracle(w)
    for h in range(3):
        sl = slice(h * r, (h + 1) * r)
        wh = make_custom(N, 6, 1, r, src, dst, seed=13, b_g=0.1)
        wh.X, wh.w_g = w.X, w.w_g
        wh.W_Q, wh.W_K, wh.W_V = (np.ascontiguousarray(a[:, sl]) for a in (w.W_Q, w.W_K, w.W_V))
        oh = run_oracle(wh)
        np.testing.assert_allclose(oh["Y"], out["Y"][:, sl], rtol=1e-14, atol=1e-15)


def test_duplicate_edge_counts_twice():
    """Each stored edge is one softmax term (tinymesh: edge-level softmax)."""
    N = 5
    src = np.array([1, 2, 2], np.int32); dst = np.array([0, 0, 0], np.int32)
    w = make_custom(N, 4, 1, 8, src, dst, seed=8, b_g=1e4)
    out = run_oracle(w)
    ref = dense_reference(w)                       # count matrix: A[0,2] = 2
    np.testing.assert_allclose(out["L"][0], ref["L"][0], rtol=1e-13)


def test_empty_and_single_node_graphs():
    w = make_custom(4, 3, 1, 8, np.zeros(0, np.int32), np.zeros(0, np.int32), seed=1)
    out = run_oracle(w)
    assert np.all(out["L"] == 0.0)
    np.testing.assert_allclose(out["Y"], (1 - out["g"])[:, None] * out["G"], rtol=1e-15)
    w1 = make_custom(1, 3, 1, 8, np.array([0], np.int32), np.array([0], np.int32), seed=1)
    o1 = run_oracle(w1)
    V = w1.X.astype(np.float64) @ w1.W_V.astype(np.float64)
    np.testing.assert_allclose(o1["L"][0], V[0], rtol=1e-14)


def test_sampled_rows_equal_full_rows():
    w = make_workload("tiny")
    full = run_oracle(w)
    rows = np.array([255, 0, 17, 128])
    part = run_oracle(w, rows=rows)
    np.testing.assert_array_equal(part["Y"], full["Y"][rows])


# ------------------------------------------------------------------------------------
# topology: CSR against numpy's lexsort, buckets against their definition
# ------------------------------------------------------------------------------------
def lexsort_csr(N, src, dst):
    order = np.lexsort((src, dst))
    row_ptr = np.concatenate([[0], np.cumsum(np.bincount(dst, minlength=N))]).astype(np.int32)
    return row_ptr, src[order].astype(np.int32)


@pytest.mark.parametrize("name", ["tiny", "citation", "arxiv"])
def test_csr_matches_lexsort(name):
    w = make_workload(name)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    rp2, ci2 = lexsort_csr(w.N, w.src, w.dst)
    np.testing.assert_array_equal(rp, rp2)
    np.testing.assert_array_equal(ci, ci2)


def test_csr_coo_permutation_duplicates_and_validation():
    rng = np.random.default_rng(3)
    N, E = 300, 5000
    src = rng.integers(0, N, E).astype(np.int32)   # duplicates and self-loops included
    dst = rng.integers(0, N, E).astype(np.int32)
    rp, ci = oracle.csr_from_coo(N, src, dst)
    p = rng.permutation(E)
    rp2, ci2 = oracle.csr_from_coo(N, src[p], dst[p])
    np.testing.assert_array_equal(rp, rp2); np.testing.assert_array_equal(ci, ci2)
    assert rp[-1] == E
    with pytest.raises(ValueError):
        oracle.csr_from_coo(N, np.array([N], np.int32), np.array([0], np.int32))
    with pytest.raises(ValueError):
        oracle.csr_from_coo(N, np.array([0], np.int32), np.array([-1], np.int32))
    rp0, ci0 = oracle.csr_from_coo(0, np.zeros(0, np.int32), np.zeros(0, np.int32))
    assert rp0.tolist() == [0] and ci0.shape == (0,)


@pytest.mark.parametrize("warp_max,chunk", [(32, 1024), (0, 1), (5, 7), (64, 64)])
def test_buckets_partition_rows_and_edges(warp_max, chunk):
    w = make_workload("citation")
    rp, _ = oracle.csr_from_coo(w.N, w.src, w.dst)
    b = oracle.degree_buckets(rp, warp_max, chunk)
    deg = np.diff(rp)
    small = np.nonzero(deg <= warp_max)[0]
    # bucket 0: descending degree, ties by ascending row (numpy's stable lexsort)
    np.testing.assert_array_equal(b["warp_rows"], small[np.lexsort((small, -deg[small]))])
    np.testing.assert_array_equal(b["cta_rows"], np.nonzero((deg > warp_max) & (deg <= chunk))[0])
    np.testing.assert_array_equal(b["split_rows"], np.nonzero(deg > chunk)[0])
    # chunks tile every split row's edges exactly once, in order
    cover = np.zeros(rp[-1], np.int32)
    for row, beg in zip(b["chunk_row"], b["chunk_begin"]):
        end = min(beg + chunk, rp[row + 1])
        assert rp[row] <= beg < end
        cover[beg:end] += 1
    split_edges = np.concatenate([np.arange(rp[i], rp[i + 1]) for i in b["split_rows"]] or [np.zeros(0, int)])
    assert np.all(cover[split_edges] == 1)
    assert cover.sum() == len(split_edges)


# ---------------------------------------------------------------------------------------
# Segments (the batch dimension of the method page's "Implementation notes"): each
# contiguous node range has its own S and z.
# ---------------------------------------------------------------------------------------
def _batch(sizes, k, seed, d=12, H=2, r=8):
    """Graphs of the given sizes (edges only inside each graph, self-loops included),
    relabelled into one node range; shared weights."""
    rng = np.random.default_rng(seed)
    src, dst, offs = [], [], [0]
    for n in sizes:
        if n > 0:
            s = rng.integers(0, n, n * k)
            t = np.repeat(np.arange(n), k)
            s = np.concatenate([s, np.arange(n)]) + offs[-1]
            t = np.concatenate([t, np.arange(n)]) + offs[-1]
            src.append(s); dst.append(t)
        offs.append(offs[-1] + n)
    N = offs[-1]
    src = np.concatenate(src).astype(np.int32) if src else np.zeros(0, np.int32)
    dst = np.concatenate(dst).astype(np.int32) if dst else np.zeros(0, np.int32)
    w = make_custom(N, d, H, r, src, dst, io="f32", seed=seed + 1, b_g=0.3)
    return w, np.array(offs, dtype=np.int64)


def test_batch_of_graphs_equals_independent_layers():
    """A batch of separate graphs with one segment per graph gives, row for row, what the
    layer gives on each graph alone (statistics over that graph's nodes only)."""
    sizes = [37, 0, 90, 1, 64, 5]
    w, seg = _batch(sizes, 4, seed=21)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    out = oracle.forward_workload(w, csr=(rp, ci), seg_ptr=seg)
    assert out["S"].shape == (len(sizes), w.H, w.r, w.r)
    for k, n in enumerate(sizes):
        a, b = int(seg[k]), int(seg[k + 1])
        if n == 0:
            assert not out["S"][k].any() and not out["z"][k].any()
            continue
        m = (w.dst >= a) & (w.dst < b)
        rp1, ci1 = oracle.csr_from_coo(n, w.src[m] - a, w.dst[m] - a)
        alone = oracle.forward(n, w.d, w.H, w.r, w.X[a:b], w.W_Q, w.W_K, w.W_V, w.w_g,
                               w.b_g, w.eps, rp1, ci1)
        np.testing.assert_allclose(out["Y"][a:b], alone["Y"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(out["S"][k], alone["S"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(out["z"][k], alone["z"], rtol=1e-12)


def test_one_segment_is_the_unsegmented_layer():
    w = make_workload("tiny")
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    a = oracle.forward_workload(w, csr=(rp, ci))
    b = oracle.forward_workload(w, csr=(rp, ci), seg_ptr=[0, w.N])
    np.testing.assert_array_equal(a["Y"], b["Y"])
    np.testing.assert_array_equal(a["S"], b["S"][0])


def test_segment_statistics_against_einsum():
    """S and z of each segment are the sums over exactly its nodes: a segment boundary
    moved by one node moves exactly that node's contribution."""
    w, seg = _batch([20, 30, 25], 3, seed=5)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    X = w.X.astype(np.float64)
    K = X @ w.W_K.astype(np.float64); V = X @ w.W_V.astype(np.float64)
    pk = torch.nn.functional.elu(torch.tensor(K)).numpy() + 1.0
    for cut in (seg, np.array([0, 21, 50, 75])):
        out = oracle.forward_workload(w, csr=(rp, ci), seg_ptr=cut)
        for k in range(3):
            a, b = cut[k], cut[k + 1]
            for h in range(w.H):
                sl = slice(h * w.r, (h + 1) * w.r)
                np.testing.assert_allclose(out["S"][k, h], np.einsum("ja,jc->ac", pk[a:b, sl], V[a:b, sl]),
                                           rtol=1e-10, atol=1e-12)
                np.testing.assert_allclose(out["z"][k, h], pk[a:b, sl].sum(0), rtol=1e-10)


def test_bad_segments_are_rejected():
    w = make_workload("tiny")
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    for seg in ([1, w.N], [0, w.N - 1], [0, 10, 5, w.N], [0]):
        with pytest.raises(ValueError):
            oracle.forward_workload(w, csr=(rp, ci), seg_ptr=seg)


# ---------------------------------------------------------------------------------------
# The block around the layer: Z = LayerNorm(X + Y Wo) (method page, Implementation notes)
# ---------------------------------------------------------------------------------------
def test_block_output_against_torch_layer_norm():
    rng = np.random.default_rng(8)
    N, D, d = 37, 24, 16
    X, Y = rng.standard_normal((N, d)), rng.standard_normal((N, D))
    Wo = rng.standard_normal((D, d)) / np.sqrt(D)
    g, b = rng.standard_normal(d), rng.standard_normal(d)
    Z = oracle.block_output(X, Y, Wo, g, b, 1e-5)
    ln = torch.nn.functional.layer_norm(torch.tensor(X + Y @ Wo), (d,), torch.tensor(g),
                                        torch.tensor(b), eps=1e-5)
    np.testing.assert_allclose(Z, ln.numpy(), rtol=1e-12, atol=1e-12)


def test_block_output_closed_forms():
    rng = np.random.default_rng(9)
    N, D, d = 11, 8, 6
    X, Y = rng.standard_normal((N, d)), rng.standard_normal((N, D))
    ones, zeros = np.ones(d), np.zeros(d)
    # unit gain, zero bias: every row has mean 0 and (nearly, by eps) variance 1
    Z = oracle.block_output(X, Y, rng.standard_normal((D, d)), ones, zeros, 0.0)
    np.testing.assert_allclose(Z.mean(1), 0, atol=1e-12)
    np.testing.assert_allclose((Z ** 2).mean(1), 1, rtol=1e-12)
    # Wo = 0: the layer's output drops out, Z = LayerNorm(X)
    Z0 = oracle.block_output(X, Y, np.zeros((D, d)), ones, zeros, 0.0)
    Xc = X - X.mean(1, keepdims=True)
    np.testing.assert_allclose(Z0, Xc / np.sqrt((Xc ** 2).mean(1, keepdims=True)), rtol=1e-12)
    # gain and bias act per feature after the normalisation
    g, b = rng.standard_normal(d), rng.standard_normal(d)
    np.testing.assert_allclose(oracle.block_output(X, Y, np.zeros((D, d)), g, b, 0.0), Z0 * g + b, rtol=1e-12)
    # a constant row shift is removed by the normalisation
    np.testing.assert_allclose(oracle.block_output(X + 3.0, Y, np.zeros((D, d)), ones, zeros, 0.0), Z0,
                               rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------------------
# Backward (reference gradients): the float64 torch forward equals the C oracle, and its
# autograd gradients equal central finite differences of the C oracle.
# ---------------------------------------------------------------------------------------
def _small_problem(seed=0, N=14, d=5, H=2, r=4):
    rng = np.random.default_rng(seed)
    src = rng.integers(0, N, 3 * N)
    dst = rng.integers(0, N, 3 * N)
    keep = dst != 3                                   # row 3 isolated
    src = np.concatenate([src[keep], np.arange(N)[np.arange(N) != 3]])
    dst = np.concatenate([dst[keep], np.arange(N)[np.arange(N) != 3]])
    w = make_custom(N, d, H, r, src.astype(np.int32), dst.astype(np.int32), io="f32", seed=seed + 1,
                    b_g=0.3)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    return w, rp, ci


def test_backward_reference_forward_equals_the_c_oracle():
    from oracle.backward import backward
    w, rp, ci = _small_problem()
    dY = np.random.default_rng(2).standard_normal((w.N, w.D))
    out = backward(w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps, rp, ci, w.H, w.r, dY)
    ref = oracle.forward_workload(w, csr=(rp, ci))["Y"]
    np.testing.assert_allclose(out["Y"], ref, rtol=1e-12, atol=1e-13)


def test_backward_matches_finite_differences_of_the_c_oracle():
    """<grad, u> against (f(x + h u) - f(x - h u)) / 2h for random directions u, where
    f = sum(Y * dY) is evaluated by the C oracle."""
    from oracle.backward import backward
    w, rp, ci = _small_problem(seed=4)
    rng = np.random.default_rng(3)
    dY = rng.standard_normal((w.N, w.D))
    base = dict(X=w.X.astype(np.float64), W_Q=w.W_Q.astype(np.float64), W_K=w.W_K.astype(np.float64),
                W_V=w.W_V.astype(np.float64), w_g=w.w_g.astype(np.float64), b_g=np.float64(w.b_g))
    g = backward(base["X"], base["W_Q"], base["W_K"], base["W_V"], base["w_g"], base["b_g"], w.eps,
                 rp, ci, w.H, w.r, dY)

    def f(vals):
        # the C oracle takes float32 inputs; evaluate it through its float64 row kernel
        # with float64 projections done here (X @ W in float64)
        Q, K, V = vals["X"] @ vals["W_Q"], vals["X"] @ vals["W_K"], vals["X"] @ vals["W_V"]
        t = vals["X"] @ vals["w_g"]
        S, z = oracle.global_stats(K, V, w.H, w.r)
        out = oracle.rows_output(np.arange(w.N), w.H, w.r, rp, ci, Q, K, V, t, S, z, float(vals["b_g"]), w.eps)
        return float((out["Y"] * dY).sum())

    key = {"X": "dX", "W_Q": "dW_Q", "W_K": "dW_K", "W_V": "dW_V", "w_g": "dw_g", "b_g": "db_g"}
    h = 1e-5
    for name, gname in key.items():
        for _ in range(2):
            u = rng.standard_normal(np.shape(base[name]))
            plus = dict(base); plus[name] = base[name] + h * u
            minus = dict(base); minus[name] = base[name] - h * u
            fd = (f(plus) - f(minus)) / (2 * h)
            an = float((np.asarray(g[gname]) * u).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("max_edges,max_rows", [(7, 3), (20, 1000), (1 << 18, 1 << 16)])
def test_backward_chunked_equals_backward(max_edges, max_rows):
    """The bounded-memory reference gradients (row groups of at most max_edges entries and
    max_rows rows; a row heavier than max_edges forms its own group) equal the whole-graph
    ones, here with a 40-entry row, an isolated row and duplicated entries."""
    from oracle.backward import NAMES, backward, backward_chunked
    rng = np.random.default_rng(12)
    N = 23
    src = np.concatenate([rng.integers(0, N, 60), rng.integers(0, N, 40), [5, 5]])
    dst = np.concatenate([rng.integers(0, N, 60), np.full(40, 9), [2, 2]])
    keep = dst != 4                                   # row 4 isolated
    w = make_custom(N, 6, 3, 4, src[keep].astype(np.int32), dst[keep].astype(np.int32), io="f32",
                    seed=13, b_g=-0.4)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    dY = rng.standard_normal((w.N, w.D))
    ref = backward(w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps, rp, ci, w.H, w.r, dY)
    got = backward_chunked(w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps, rp, ci, w.H, w.r, dY,
                           max_edges=max_edges, max_rows=max_rows)
    for k in NAMES:
        np.testing.assert_allclose(got[k], np.reshape(ref[k], np.shape(got[k])), rtol=1e-11,
                                   atol=1e-12 * max(1.0, np.abs(ref[k]).max()), err_msg=k)


def test_backward_chunked_edgeless_graph():
    from oracle.backward import NAMES, backward, backward_chunked
    w = make_custom(9, 5, 2, 4, np.zeros(0, np.int32), np.zeros(0, np.int32), io="f32", seed=3, b_g=0.2)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    dY = np.random.default_rng(1).standard_normal((w.N, w.D))
    ref = backward(w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps, rp, ci, w.H, w.r, dY)
    got = backward_chunked(w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps, rp, ci, w.H, w.r, dY, max_edges=4)
    for k in NAMES:
        np.testing.assert_allclose(got[k], np.reshape(ref[k], np.shape(got[k])), rtol=1e-11, atol=1e-13, err_msg=k)
