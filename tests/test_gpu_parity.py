"""GPU parity: every call goes through the C ABI (via the ctypes binding) and is compared
with the float64 oracle on the same seeded inputs.

Integer work (CSR construction, degree buckets) must be bit-exact; the forward must be
within max|err| <= 1e-4 * max|Y| (fp32 I/O) or 2e-2 * max|Y| (bf16 I/O)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_custom
from tests.gpu_helpers import (TOL, assert_close_to_oracle, oracle_csr, run_gpu, sample_rows,
                               to_dev, workload)

pytestmark = pytest.mark.gpu

ALL = ["tiny", "citation", "arxiv", "packed", "skewed"]


# ------------------------------------------------------------------------------------
# integer work: bit-exact
# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", ALL)
def test_csr_from_coo_bit_exact(name):
    w = workload(name)
    rp, ci = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    orp, oci = oracle_csr(name)
    np.testing.assert_array_equal(rp.cpu().numpy(), orp)
    np.testing.assert_array_equal(ci.cpu().numpy(), oci)


def test_csr_from_coo_order_invariant_and_duplicates():
    rng = np.random.default_rng(5)
    N, E = 1000, 60000
    src = rng.integers(0, N, E).astype(np.int32)
    dst = (rng.zipf(1.5, E) % N).astype(np.int32)       # skewed rows, many duplicates
    p = rng.permutation(E)
    a = glga.csr_from_coo(N, to_dev(src), to_dev(dst))
    b = glga.csr_from_coo(N, to_dev(src[p]), to_dev(dst[p]))
    orp, oci = oracle.csr_from_coo(N, src, dst)
    for rp, ci in (a, b):
        np.testing.assert_array_equal(rp.cpu().numpy(), orp)
        np.testing.assert_array_equal(ci.cpu().numpy(), oci)


def test_csr_from_coo_rejects_bad_endpoints_and_handles_empty():
    with pytest.raises(glga.GLGAError) as ei:
        glga.csr_from_coo(4, to_dev(np.array([0, 4], np.int32)), to_dev(np.array([1, 1], np.int32)))
    assert ei.value.status == 2
    rp, ci = glga.csr_from_coo(5, to_dev(np.zeros(0, np.int32)), to_dev(np.zeros(0, np.int32)))
    assert rp.cpu().tolist() == [0] * 6 and ci.numel() == 0


@pytest.mark.parametrize("name", ALL)
def test_buckets_bit_exact(name):
    w = workload(name)
    orp, oci = oracle_csr(name)
    o = glga.default_options()
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, to_dev(orp), to_dev(oci))
    got = {k: v.cpu().numpy() for k, v in layer.buckets().items()}
    ref = oracle.degree_buckets(orp, o.warp_max_degree, o.chunk_edges)
    assert layer.bucket_counts() == ref["counts"].tolist()
    for k in ("warp_rows", "cta_rows", "split_rows", "chunk_row", "chunk_begin"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
    layer.close()


@pytest.mark.parametrize("wmax,chunk", [(0, 1), (3, 5), (8, 64), (64, 64), (1000, 100000)])
def test_buckets_bit_exact_thresholds(wmax, chunk):
    w = workload("citation")
    orp, oci = oracle_csr("citation")
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, to_dev(orp), to_dev(oci), glga.Options(wmax, chunk))
    got = {k: v.cpu().numpy() for k, v in layer.buckets().items()}
    ref = oracle.degree_buckets(orp, wmax, chunk)
    for k in ("warp_rows", "cta_rows", "split_rows", "chunk_row", "chunk_begin"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
    layer.close()


def test_invalid_csr_is_rejected_at_create():
    N = 6
    good_rp = np.array([0, 1, 2, 3, 4, 5, 6], np.int32)
    good_ci = np.arange(6, dtype=np.int32)
    cases = [
        (np.array([1, 1, 2, 3, 4, 5, 6], np.int32), good_ci),      # row_ptr[0] != 0
        (np.array([0, 1, 2, 3, 4, 5, 5], np.int32), good_ci),      # row_ptr[N] != E
        (np.array([0, 2, 1, 3, 4, 5, 6], np.int32), good_ci),      # decreasing
        (good_rp, np.array([0, 1, 2, 6, 4, 5], np.int32)),          # col out of range
        (good_rp, np.array([0, 1, -1, 3, 4, 5], np.int32)),
    ]
    for rp, ci in cases:
        with pytest.raises(glga.GLGAError) as ei:
            glga.Layer(N, 8, 1, 8, "f32", to_dev(rp), to_dev(ci))
        assert ei.value.status == 2


# ------------------------------------------------------------------------------------
# forward parity on the five workloads
# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "citation"])
def test_forward_parity_all_rows(name):
    w = workload(name)
    out = run_gpu(w, keep_layer=True)
    rp, ci = oracle_csr(name)
    ref = oracle.forward_workload(w, csr=(rp, ci))
    assert_close_to_oracle(w, out["Y"], ref)
    inter = out["layer"].intermediates()
    torch.cuda.synchronize()
    np.testing.assert_allclose(inter["S"].cpu().numpy(), ref["S"], rtol=0,
                               atol=1e-4 * np.abs(ref["S"]).max())
    np.testing.assert_allclose(inter["z"].cpu().numpy(), ref["z"], rtol=0,
                               atol=1e-4 * np.abs(ref["z"]).max())
    np.testing.assert_allclose(inter["t"].cpu().numpy(), ref["t"], rtol=0,
                               atol=1e-4 * np.abs(ref["t"]).max())
    out["layer"].close()


@pytest.mark.parametrize("name", ["arxiv", "packed", "skewed"])
def test_forward_parity_full_size_sampled_rows(name):
    w = workload(name)
    rp, ci = oracle_csr(name)
    out = run_gpu(w, keep_layer=True)
    rows = sample_rows(w, rp)
    ref = oracle.forward_workload(w, rows=rows, csr=(rp, ci))
    assert_close_to_oracle(w, out["Y"], ref, rows=rows)
    inter = out["layer"].intermediates()
    torch.cuda.synchronize()
    # global statistics over all N nodes: compared in full
    for key in ("S", "z"):
        g = inter[key].cpu().numpy()
        np.testing.assert_allclose(g, ref[key], rtol=0, atol=TOL[w.io] * np.abs(ref[key]).max())
    tg = inter["t"].cpu().numpy()[rows]
    np.testing.assert_allclose(tg, ref["t"], rtol=0, atol=TOL[w.io] * np.abs(ref["t"]).max())
    out["layer"].close()


def test_determinism_bitwise():
    w = workload("arxiv")
    out = run_gpu(w, keep_layer=True)
    layer = out["layer"]
    Y1 = out["Y"].clone()
    Y2 = layer.forward(*out["args"], b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    layer.close()


def test_forward_captures_in_cuda_graph():
    """A forward enqueues work without host synchronisation, so it can be captured."""
    w = workload("citation")
    out = run_gpu(w, keep_layer=True)
    layer, args = out["layer"], out["args"]
    Y = torch.empty_like(out["Y"])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.forward(*args, b_g=w.b_g, eps=w.eps, Y=Y)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    Y.zero_()
    with torch.cuda.graph(g):
        layer.forward(*args, b_g=w.b_g, eps=w.eps, Y=Y)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, out["Y"])
    del g
    layer.close()


# ------------------------------------------------------------------------------------
# edge cases and every bucket path
# ------------------------------------------------------------------------------------
def _custom_check(w, options=None, tol=None):
    out = run_gpu(w, options=options)
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    ref = oracle.forward_workload(w, csr=(rp, ci))
    if np.abs(ref["Y"]).max() == 0:
        assert float(out["Y"].abs().max()) == 0.0
        return 0.0
    return assert_close_to_oracle(w, out["Y"], ref, tol=tol)


def _rand_edges(N, k, seed, self_loops=True):
    rng = np.random.default_rng(seed)
    src = rng.integers(0, N, N * k)
    dst = np.repeat(np.arange(N), k)
    if self_loops:
        src = np.concatenate([src, np.arange(N)]); dst = np.concatenate([dst, np.arange(N)])
    return src.astype(np.int32), dst.astype(np.int32)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("H,r", [(1, 8), (3, 16), (2, 64), (1, 128), (8, 16), (5, 32), (4, 8)])
def test_head_shapes(io, H, r):
    if H * r * (4 if io == "f32" else 2) > 2048:
        pytest.skip("row too wide")
    src, dst = _rand_edges(300, 6, seed=H * 100 + r)
    w = make_custom(300, 40, H, r, src, dst, io=io, seed=r + H, b_g=0.2)
    _custom_check(w)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("d", [1, 13, 64, 200])
def test_input_widths_and_ragged_rows(io, d):
    N = 129 + d                                   # never a multiple of the 128-row tile
    src, dst = _rand_edges(N, 5, seed=d)
    w = make_custom(N, d, 2, 16, src, dst, io=io, seed=d, b_g=-0.4)
    _custom_check(w)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("opts", [(0, 1), (0, 8), (2, 3), (4, 100000), (100000, 100000)])
def test_every_bucket_path(io, opts):
    """Skewed degrees with thresholds that push rows through the warp, block and chunk
    paths (chunk size 1 and 3 exercise many-chunk merges)."""
    rng = np.random.default_rng(11)
    N = 400
    deg = np.minimum(rng.zipf(1.6, N), 300)
    dst = np.repeat(np.arange(N), deg)
    src = rng.integers(0, N, dst.shape[0])
    w = make_custom(N, 24, 2, 32, src.astype(np.int32), dst.astype(np.int32), io=io, seed=3, b_g=0.1)
    _custom_check(w, options=glga.Options(*opts))


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_empty_graph_and_isolated_rows(io):
    w = make_custom(70, 9, 2, 8, np.zeros(0, np.int32), np.zeros(0, np.int32), io=io, seed=4)
    _custom_check(w)
    src = np.array([1, 2, 3, 60], np.int32)
    dst = np.array([0, 0, 5, 69], np.int32)
    w = make_custom(70, 9, 2, 8, src, dst, io=io, seed=4)
    _custom_check(w)


def test_zero_nodes():
    w = make_custom(0, 8, 1, 8, np.zeros(0, np.int32), np.zeros(0, np.int32))
    rp = to_dev(np.zeros(1, np.int32))
    layer = glga.Layer(0, 8, 1, 8, "f32", rp, to_dev(np.zeros(0, np.int32)))
    args = [to_dev(a) for a in (w.X.reshape(0, 8), w.W_Q, w.W_K, w.W_V, w.w_g)]
    Y = layer.forward(*args, b_g=0.0, eps=1e-6)
    torch.cuda.synchronize()
    assert Y.shape == (0, 8)
    layer.close()


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_single_node_and_self_loop_only(io):
    w = make_custom(1, 5, 1, 16, np.array([0], np.int32), np.array([0], np.int32), io=io, seed=9)
    _custom_check(w)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complete_graph(io):
    N = 200
    ii, jj = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    w = make_custom(N, 16, 4, 16, jj.reshape(-1).astype(np.int32), ii.reshape(-1).astype(np.int32),
                    io=io, seed=12, b_g=1.0)
    _custom_check(w)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_duplicate_edges(io):
    src = np.array([1, 1, 1, 2, 3, 3], np.int32)
    dst = np.array([0, 0, 0, 0, 4, 4], np.int32)
    w = make_custom(6, 7, 1, 32, src, dst, io=io, seed=13)
    _custom_check(w)


def test_large_scores_stay_finite():
    src, dst = _rand_edges(256, 8, seed=21)
    w = make_custom(256, 16, 2, 16, src, dst, io="f32", seed=21, w_scale=2.0)
    w.W_Q = w.W_Q * np.float32(25.0)
    _custom_check(w)


def test_gate_saturation():
    src, dst = _rand_edges(150, 4, seed=22)
    for b in (1e4, -1e4):
        w = make_custom(150, 12, 2, 16, src, dst, io="f32", seed=22, b_g=b)
        _custom_check(w)


def test_workspace_is_linear_in_graph_size():
    w = workload("arxiv")
    rp, ci = oracle_csr("arxiv")
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, to_dev(rp), to_dev(ci))
    b = layer.workspace_bytes()
    s = 2
    linear = (w.N * (3 * w.D * s + 4 + 8) + 8 * w.E + 4 * 1024 * 1024 +
              w.d * 4 * w.D * s * 2)
    assert b <= 2 * linear, (b, linear)
    assert b < w.E * w.D * s            # nothing proportional to E * r
    layer.close()


@pytest.mark.parametrize("N,d,H,r,io", [(700, 128, 4, 32, "bf16"), (300, 512, 8, 64, "bf16"),
                                        (517, 256, 8, 32, "bf16"), (260, 1433, 8, 8, "f32"),
                                        (200, 13, 2, 16, "bf16"), (333, 40, 3, 16, "f32")])
def test_projection_outputs_every_column(N, d, H, r, io):
    """Q, K, V and the gate logit of the tcgen05 GEMM against the oracle's projections, all
    rows and columns (several column tiles; tile widths not multiples of 32)."""
    src = np.arange(N, dtype=np.int32)
    w = make_custom(N, d, H, r, src, src, io=io, seed=N)
    out = run_gpu(w, keep_layer=True)
    inter = {k: v.float().cpu().numpy() for k, v in out["layer"].intermediates().items()}
    torch.cuda.synchronize()
    # fp32 (3-term tf32 split, fp32 accumulation in the tensor cores): each element obeys
    #   |err| <= (3 * 2^-22 + 3 * ceil(dp / 8) * 2^-23) * A,   A = sum_k |x_k| |w_k|,
    # the first term for the dropped lo*lo product and the tf32 residues of the hi/lo
    # planes, the second for one f32 rounding of the running sum (itself at most A) per
    # MMA step of 8 K elements, for each of the three products.  Measured worst case over
    # these shapes: 1.13e-5 * max|ref| and 1.9e-6 * A (d = 1433); the global 5e-5 * max|ref|
    # check keeps a 4x margin over it.  bf16: the outputs are rounded to bf16 (2^-9).
    tol = 5e-5 if io == "f32" else 8e-3
    dp = -(-d // 32) * 32
    for key, W in (("Q", w.W_Q), ("K", w.W_K), ("V", w.W_V)):
        ref = oracle.project(w.X, W)
        np.testing.assert_allclose(inter[key], ref, rtol=0, atol=tol * np.abs(ref).max(), err_msg=key)
        if io == "f32":
            A = np.abs(w.X.astype(np.float64)) @ np.abs(W.astype(np.float64))
            bound = (3 * 2.0 ** -22 + 3 * (dp // 8) * 2.0 ** -23) * A + 1e-30
            assert np.all(np.abs(inter[key] - ref) <= bound), key
    ref_t = oracle.gate_logit(w.X, w.w_g)
    np.testing.assert_allclose(inter["t"], ref_t, rtol=0, atol=1e-5 * np.abs(ref_t).max())
    out["layer"].close()
