"""Failure paths on the GPU, exercised without a GPU fault: a bounded wait that runs out
(an mbarrier nothing arrives on), the debug builds' index checks against a planted bad
column index, and simulated allocation failures in glga_create."""
import numpy as np
import pytest
import torch

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_custom
from tests.gpu_helpers import assert_close_to_oracle, run_gpu, to_dev, workload

pytestmark = pytest.mark.gpu

GLGA_ERR_INVALID_ARG, GLGA_ERR_OOM, GLGA_ERR_TIMEOUT, GLGA_ERR_DEVICE = 1, 4, 6, 7


def _oracle(w):
    return oracle.forward_workload(w, csr=oracle.csr_from_coo(w.N, w.src, w.dst))


def _layer(w, options=None):
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, options)
    args = [to_dev(a, glga.torch_dtype(w.io)) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    return layer, row_ptr.cpu().numpy(), args


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    w = workload("tiny")
    layer, row_ptr, args = _layer(w)
    layer.debug_bounded_wait(20_000_000)          # 20 ms; nothing ever arrives
    assert layer.last_device_error() == GLGA_ERR_TIMEOUT
    assert layer.last_device_error() == 0         # reading the flag clears it
    Y = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0
    assert_close_to_oracle(w, Y, _oracle(w))
    with pytest.raises(glga.GLGAError) as ei:
        layer.debug_bounded_wait(10)              # below the accepted range
    assert ei.value.status == GLGA_ERR_INVALID_ARG
    layer.close()


def _skewed_graph(io, seed=11):
    rng = np.random.default_rng(seed)
    N = 400
    deg = np.minimum(rng.zipf(1.6, N), 300)
    deg[:3] = [250, 40, 2]                        # one row per bucket with the options below
    dst = np.repeat(np.arange(N), deg)
    src = rng.integers(0, N, dst.shape[0])
    return make_custom(N, 24, 2, 32, src.astype(np.int32), dst.astype(np.int32), io=io, seed=3, b_g=0.1)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_debug_checks_give_identical_results(io):
    w = _skewed_graph(io)
    opts = glga.Options(8, 64, 0, 0)
    plain = run_gpu(w, options=opts)["Y"].cpu()
    dbg = run_gpu(w, options=glga.Options(8, 64, 1, 0))["Y"].cpu()
    assert torch.equal(plain, dbg)


@pytest.mark.parametrize("which", ["warp", "block", "chunk"])
@pytest.mark.parametrize("bad", [400, 1 << 30, -3])
def test_debug_checks_catch_a_bad_column_index(which, bad):
    """Rows 0, 1, 2 have 250, 40 and 2 edges: with warp_max_degree 8 and chunk_edges 64
    they take the chunk, block and warp paths.  One of their CSR entries is overwritten
    with an index outside [0, N); the debug build masks it and reports it."""
    w = _skewed_graph("f32")
    layer, row_ptr, args = _layer(w, glga.Options(8, 64, 1, 0))
    row = {"chunk": 0, "block": 1, "warp": 2}[which]
    assert row_ptr[row + 1] - row_ptr[row] == [250, 40, 2][row]
    Y = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0
    layer.debug_set_col_idx(int(row_ptr[row]) + 1, bad)
    Y = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert layer.last_device_error() == GLGA_ERR_DEVICE
    assert torch.isfinite(Y.float()).all()
    layer.close()


def test_set_col_idx_is_refused_without_debug_checks():
    w = workload("tiny")
    layer, _, _ = _layer(w)
    with pytest.raises(glga.GLGAError) as ei:
        layer.debug_set_col_idx(0, 5)
    assert ei.value.status == GLGA_ERR_INVALID_ARG
    layer.close()


def test_every_failed_allocation_in_create_is_cleaned_up():
    w = _skewed_graph("bf16")
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    args = [to_dev(a, glga.torch_dtype(w.io)) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    # one full create / forward / destroy first, so that lazily loaded kernels and torch's
    # cached blocks are in place before the free memory is read
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, glga.Options(8, 64, 0, 0))
    Y = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    layer.close()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    n = 1
    while True:
        try:
            layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, glga.Options(8, 64, 0, n))
        except glga.GLGAError as e:
            assert e.status == GLGA_ERR_OOM, (n, e)
            n += 1
            assert n < 200
            continue
        break
    assert n > 10                                  # every context buffer was a failure point
    Y = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0
    assert_close_to_oracle(w, Y, _oracle(w))
    layer.close()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert abs(free0 - free1) < 8 << 20            # no leaked context buffers
