"""The block around the layer on the GPU, Z = LayerNorm(X + Y Wo) (glga_block_output),
against the oracle's definition.  Y is the GPU layer's own output, so the comparison
isolates the block; one case also runs the whole chain against the oracle's Y."""
import numpy as np
import pytest
import torch

import oracle
from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_custom, make_workload, round_to_bf16
from tests.gpu_helpers import TOL, run_gpu, to_dev

pytestmark = pytest.mark.gpu


def _params(w, seed):
    rng = np.random.default_rng(seed)
    Wo = (rng.standard_normal((w.D, w.d)) / np.sqrt(w.D)).astype(np.float32)
    g = (1.0 + 0.1 * rng.standard_normal(w.d)).astype(np.float32)
    b = (0.1 * rng.standard_normal(w.d)).astype(np.float32)
    if w.io == "bf16":
        Wo, g, b = round_to_bf16(Wo), round_to_bf16(g), round_to_bf16(b)
    return Wo, g, b


def _check(w, seed=0, ln_eps=1e-5):
    out = run_gpu(w, keep_layer=True)
    layer, Y = out["layer"], out["Y"]
    Wo, g, b = _params(w, seed)
    dt = glga.torch_dtype(w.io)
    Z = layer.block_output(Y, out["args"][0], to_dev(Wo, dt), to_dev(g, dt), to_dev(b, dt), ln_eps)
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0
    layer.close()
    ref = oracle.block_output(w.X, Y.float().cpu().numpy(), Wo, g, b, ln_eps)
    Zg = Z.float().cpu().numpy().astype(np.float64)
    err = np.abs(Zg - ref).max() / np.abs(ref).max()
    assert np.all(np.isfinite(Zg)) and err <= TOL[w.io], err
    return Z, Y, (Wo, g, b)


def test_tiny_fp32_split_operands():
    _check(make_workload("tiny"))


def test_arxiv_shape_bf16_in_place_operand():
    w = make_workload("arxiv", scale=0.05)
    Z, Y, (Wo, g, b) = _check(w)
    # the whole chain against the oracle's own Y
    ref_y = oracle.forward_workload(w)["Y"]
    ref = oracle.block_output(w.X, ref_y, Wo, g, b, 1e-5)
    err = np.abs(Z.float().cpu().numpy() - ref).max() / np.abs(ref).max()
    assert err <= TOL["bf16"], err


def test_packed_shape_two_accumulator_halves():
    _check(make_workload("packed", scale=0.02))      # d = 512: two N = 256 halves


@pytest.mark.parametrize("io,d,H,r", [("bf16", 256, 8, 32), ("bf16", 64, 1, 32), ("f32", 96, 2, 16)])
def test_other_widths(io, d, H, r):
    rng = np.random.default_rng(5)
    N = 700                                           # ragged last tile
    dst = np.repeat(np.arange(N), 6)
    src = rng.integers(0, N, dst.shape[0])
    w = make_custom(N, d, H, r, src.astype(np.int32), dst.astype(np.int32), io=io, seed=6, b_g=0.2)
    _check(w, seed=7)


def test_unsupported_width_is_refused():
    w = make_workload("citation")                     # d = 1433
    out = run_gpu(w, keep_layer=True)
    layer = out["layer"]
    dt = glga.torch_dtype(w.io)
    with pytest.raises(glga.GLGAError) as ei:
        layer.block_output(out["Y"], out["args"][0], torch.zeros(w.D, w.d, dtype=dt, device="cuda"),
                           torch.ones(w.d, dtype=dt, device="cuda"), torch.zeros(w.d, dtype=dt, device="cuda"))
    assert ei.value.status == 3
    layer.close()
