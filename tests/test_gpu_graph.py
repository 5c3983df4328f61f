"""glga_forward recorded into a CUDA graph (Layer.capture): a replay gives the same bits as
an eager forward on the same buffers, also after the inputs are refilled in place."""
import numpy as np
import pytest
import torch

from sparse_graph_attention_tcgen05_b200 import glga
from sparse_graph_attention_tcgen05_b200.workloads import make_workload
from tests.gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,scale", [("tiny", 1.0), ("citation", 1.0), ("arxiv", 0.05), ("packed", 0.02)])
def test_graph_replay_matches_eager(name, scale):
    w = make_workload(name, scale=scale)
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx)
    dt = glga.torch_dtype(w.io)
    args = [to_dev(a, dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    eager = layer.forward(*args, b_g=w.b_g, eps=w.eps).clone()
    graph, Y = layer.capture(*args, w.b_g, w.eps)
    Y.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, eager)
    # new inputs, refilled in place: the replay follows them
    rng = np.random.default_rng(12)
    args[0].copy_(to_dev(rng.standard_normal(w.X.shape).astype(np.float32), dt))
    args[3].mul_(0.5)
    graph.replay()
    torch.cuda.synchronize()
    again = layer.forward(*args, b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(Y, again) and not torch.equal(Y, eager)
    assert layer.last_device_error() == 0
    del graph
    layer.close()


@pytest.mark.parametrize("name,scale", [("tiny", 1.0), ("arxiv", 0.05)])
def test_backward_graph_replay_matches_eager(name, scale):
    w = make_workload(name, scale=scale)
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    o = glga.default_options()
    o.backward = 1
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, o)
    dt = glga.torch_dtype(w.io)
    args = [to_dev(a, dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    dY = to_dev(np.random.default_rng(3).standard_normal((w.N, w.D)).astype(np.float32), dt)
    layer.forward(*args, b_g=w.b_g, eps=w.eps)
    eager = {k: v.clone() for k, v in layer.backward(*args, w.b_g, w.eps, dY).items()}
    graph, grads = layer.capture_backward(*args, w.b_g, w.eps, dY)
    for v in grads.values():
        v.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    for k in eager:
        assert torch.equal(grads[k], eager[k]), k
    # a new upstream gradient, refilled in place
    dY.mul_(-2.0)
    graph.replay()
    torch.cuda.synchronize()
    again = layer.backward(*args, w.b_g, w.eps, dY)
    torch.cuda.synchronize()
    for k in eager:
        assert torch.equal(grads[k], again[k]), k
    assert layer.last_device_error() == 0
    del graph
    layer.close()


@pytest.mark.parametrize("name,scale", [("tiny", 1.0), ("arxiv", 0.05)])
def test_host_inputs_slab_upload_matches_separate_copies(name, scale):
    """glga.HostInputs: one pinned slab uploaded per step gives the forward the same inputs
    (bit for bit) as five separate copies, in every slot, and a refill of the host views
    reaches the device with the next upload only."""
    w = make_workload(name, scale=scale)
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx)
    dt = glga.torch_dtype(w.io)
    arrays = (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)
    stage = glga.HostInputs(w.N, w.d, w.D, dt, torch.device("cuda"), slots=2)
    for k, a in zip(stage.NAMES, arrays):
        stage.host[k].copy_(torch.from_numpy(np.ascontiguousarray(a)).to(dt))
    plain = layer.forward(*(to_dev(a, dt) for a in arrays), b_g=w.b_g, eps=w.eps).clone()
    for slot in (0, 1):
        ins = stage.upload(slot)
        for t in ins:
            assert t.is_cuda and t.is_contiguous() and t.data_ptr() % 256 == 0
        Y = layer.forward(*ins, b_g=w.b_g, eps=w.eps)
        torch.cuda.synchronize()
        assert torch.equal(Y, plain)
    stage.host["X"].mul_(-1)
    stale = layer.forward(*stage.device_inputs[0], b_g=w.b_g, eps=w.eps).clone()
    fresh = layer.forward(*stage.upload(0), b_g=w.b_g, eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(stale, plain) and not torch.equal(fresh, plain)
    assert layer.last_device_error() == 0
    layer.close()


def test_captured_graph_keeps_its_buffers_alive():
    """A forward graph holds X, the weights and Y: with every caller reference dropped,
    their memory is not handed to new tensors that a replay would then overwrite."""
    w = make_workload("arxiv", scale=0.02)
    row_ptr, col_idx = glga.csr_from_coo(w.N, to_dev(w.src), to_dev(w.dst))
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx)
    dt = glga.torch_dtype(w.io)
    args = [to_dev(a, dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
    eager = layer.forward(*args, b_g=w.b_g, eps=w.eps).clone()
    graph, Y = layer.capture(*args, w.b_g, w.eps)
    del Y, args
    probes = [torch.full_like(eager, 7.0) for _ in range(4)]
    graph.replay()
    torch.cuda.synchronize()
    for p in probes:
        assert bool((p == 7.0).all())
    assert torch.equal(graph.glga_buffers[-1], eager)
    assert layer.last_device_error() == 0
    del graph
    layer.close()
