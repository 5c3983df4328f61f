"""CPU-side checks of the C ABI: the library loads, exports every entry point that
include/glga.h declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes

import numpy as np

import pytest

from sparse_graph_attention_tcgen05_b200 import glga


def test_library_exports_every_declared_symbol():
    names = glga.declared_symbols()
    assert "glga_create" in names and "glga_forward" in names and "glga_destroy" in names
    L = glga.lib()
    for n in names:
        assert hasattr(L, n), n
    assert len(names) >= 15


def test_status_strings_and_defaults():
    L = glga.lib()
    for s in range(8):
        assert L.glga_status_string(s)
    assert L.glga_status_string(99) == b"unknown status"
    o = glga.default_options()
    assert 0 <= o.warp_max_degree <= o.chunk_edges and o.chunk_edges >= 1


@pytest.mark.parametrize("kw,status", [
    (dict(r=24), 3),                 # r outside {8, 16, 32, 64, 128}
    (dict(r=12), 3),
    (dict(H=0), 1),
    (dict(d=0), 1),
    (dict(N=-1), 1),
    (dict(H=17, r=128, io=1), 3),    # row width 4352 bytes > 2048
    (dict(io=7), 1),
])
def test_create_rejects_bad_shapes_before_any_device_work(kw, status):
    args = dict(N=4, d=8, H=1, r=8, io=0)
    args.update(kw)
    h = ctypes.c_void_p()
    st = glga.lib().glga_create(ctypes.byref(h), args["N"], args["d"], args["H"], args["r"],
                                args["io"], 16, 16, 0, None, None)
    assert st == status
    assert h.value is None
    assert glga.lib().glga_last_error_message()


def test_create_rejects_bad_options():
    h = ctypes.c_void_p()
    o = glga.Options(64, 32)             # warp_max_degree > chunk_edges
    assert glga.lib().glga_create(ctypes.byref(h), 4, 8, 1, 8, 0, 16, 16, 0, ctypes.byref(o), None) == 1
    o = glga.Options(0, 0)
    assert glga.lib().glga_create(ctypes.byref(h), 4, 8, 1, 8, 0, 16, 16, 0, ctypes.byref(o), None) == 1


def test_null_arguments():
    L = glga.lib()
    assert L.glga_create(None, 4, 8, 1, 8, 0, 16, 16, 0, None, None) == 1
    assert L.glga_forward(None, 16, 16, 16, 16, 16, 0.0, 1e-6, 16, None) == 1
    assert L.glga_destroy(None) == 0
    assert L.glga_csr_from_coo(-1, 0, None, None, None, None, None) == 1
    assert L.glga_csr_from_coo(4, 3, None, None, 16, 16, None) == 1
    n = ctypes.c_int64()
    assert L.glga_kernel_launches(None, ctypes.byref(n)) == 1
    assert L.glga_workspace_bytes(None, ctypes.byref(n)) == 1
    assert L.glga_default_options(None) == 1


def test_debug_options_default_off_and_are_checked():
    o = glga.default_options()
    assert (o.debug_checks, o.debug_fail_alloc) == (0, 0)
    h = ctypes.c_void_p()
    o = glga.Options(8, 64, 0, -1)           # negative allocation index
    assert glga.lib().glga_create(ctypes.byref(h), 4, 8, 1, 8, 0, 16, 16, 0, ctypes.byref(o), None) == 1


def test_debug_entry_points_reject_a_null_context():
    L = glga.lib()
    assert L.glga_debug_bounded_wait(None, 1_000_000, None) == 1
    assert L.glga_debug_set_col_idx(None, 0, 0, None) == 1


def test_segmented_create_rejects_malformed_segments():
    """Host-side checks of glga_create_segmented (before any device call)."""
    L = glga.lib()
    h = ctypes.c_void_p()
    N = 10
    for seg in ([1, N], [0, N - 1], [0, 6, 4, N]):
        arr = np.array(seg, dtype=np.int64)
        assert L.glga_create_segmented(ctypes.byref(h), N, 8, 1, 8, 0, 16, 16, 0, arr.ctypes.data,
                                       len(seg) - 1, None, None) == 1
    arr = np.array([0, N], dtype=np.int64)
    assert L.glga_create_segmented(ctypes.byref(h), N, 8, 1, 8, 0, 16, 16, 0, None, 1, None, None) == 1
    assert L.glga_create_segmented(ctypes.byref(h), N, 8, 1, 8, 0, 16, 16, 0, arr.ctypes.data, 0,
                                   None, None) == 1


def test_every_declared_entry_point_has_a_binding_signature():
    """ctypes would pass 64-bit integers as C ints without argtypes."""
    L = glga.lib()
    for name in glga.declared_symbols():
        assert getattr(L, name).argtypes is not None, name


def test_host_inputs_slab_layout(monkeypatch):
    """glga.HostInputs lays X and the weights out in one slab, each piece 256-byte aligned,
    non-overlapping, in forward's argument order (host side only: pinning is stubbed)."""
    import torch
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    for N, d, D, dt in ((1000, 128, 64, torch.bfloat16), (7, 3, 5, torch.float32)):
        st = glga.HostInputs(N, d, D, dt, "cpu", slots=2)
        shapes = {"X": (N, d), "W_Q": (d, D), "W_K": (d, D), "W_V": (d, D), "w_g": (d,)}
        base, end = st.slab.data_ptr(), -1
        for k in st.NAMES:
            v = st.host[k]
            assert tuple(v.shape) == shapes[k] and v.is_contiguous()
            off = v.data_ptr() - base
            assert off % 256 == 0 and off > end
            end = off + v.numel() * v.element_size() - 1
        assert end < st.nbytes
        for slot in range(2):
            assert [tuple(t.shape) for t in st.device_inputs[slot]] == [shapes[k] for k in st.NAMES]
        st.host["W_K"].fill_(3)
        assert float(st.slab.sum()) == 3 * d * D
