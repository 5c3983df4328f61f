"""Global statistics accumulated in the projection GEMM's epilogue.

For one-segment bf16 layers with H*r = 128 and r dividing 64 the projection kernel forms
S_h = sum_j phi(k_j^h) (v_j^h)^T and z_h = sum_j phi(k_j^h) (method page "Gated
Local-Global Graph Attention", Key formulas) from the K and V tiles it has just staged for
its stores when `fuse_stats` asks for it; by default the statistics kernel forms them.
Both paths are checked against the float64 oracle over all N nodes, against each other
(the same bf16 products, summed in another order), and the fused path for bitwise
repeatability.  Sizes cover one
partial row block, several row blocks per CTA and a ragged last block.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_custom
from tests.gpu_helpers import TOL, assert_close_to_oracle, run_gpu

pytestmark = pytest.mark.gpu


def _edges(N, k, seed):
    rng = np.random.default_rng(seed)
    src = np.concatenate([rng.integers(0, N, N * k), np.arange(N)]).astype(np.int32)
    dst = np.concatenate([np.repeat(np.arange(N), k), np.arange(N)]).astype(np.int32)
    return src, dst


def _run(w, fuse):
    o = glga.default_options()
    o.fuse_stats = fuse
    out = run_gpu(w, options=o, keep_layer=True)
    inter = out["layer"].intermediates()
    torch.cuda.synchronize()
    return out, {k: inter[k].cpu().numpy().astype(np.float64) for k in ("S", "z")}


@pytest.mark.parametrize("H,r", [(4, 32), (2, 64), (8, 16)])
@pytest.mark.parametrize("N", [77, 1000, 40000])
def test_fused_statistics_match_oracle_and_statistics_kernel(N, H, r):
    src, dst = _edges(N, 4, seed=N + r)
    w = make_custom(N, 96, H, r, src, dst, io="bf16", seed=N * 7 + H, b_g=0.3)
    fused, st_f = _run(w, 1)
    sep, st_s = _run(w, 0)
    # the fused path launches one kernel fewer (no statistics kernel)
    assert fused["layer"].kernel_launches() == sep["layer"].kernel_launches() - 1
    rp, ci = oracle.csr_from_coo(w.N, w.src, w.dst)
    rows = np.unique(np.concatenate([np.arange(min(N, 300)), np.arange(max(0, N - 200), N)]))
    ref = oracle.forward_workload(w, rows=rows, csr=(rp, ci))
    for key in ("S", "z"):
        scale = np.abs(ref[key]).max()
        for got in (st_f[key], st_s[key]):
            np.testing.assert_allclose(got, ref[key], rtol=0, atol=TOL["bf16"] * scale, err_msg=key)
        # same bf16 operands and float32 accumulation, another summation order
        np.testing.assert_allclose(st_f[key], st_s[key], rtol=0, atol=2e-5 * scale * max(1.0, N / 1e4),
                                   err_msg=key)
    assert_close_to_oracle(w, fused["Y"], ref, rows=rows)
    # bitwise repeatable: a fixed tile walk per CTA and a fixed-order reduction
    layer, args = fused["layer"], fused["args"]
    layer.forward(*args, b_g=w.b_g, eps=w.eps)
    again = layer.intermediates()
    torch.cuda.synchronize()
    for key in ("S", "z"):
        assert np.array_equal(again[key].cpu().numpy().astype(np.float64), st_f[key]), key
    fused["layer"].close()
    sep["layer"].close()

