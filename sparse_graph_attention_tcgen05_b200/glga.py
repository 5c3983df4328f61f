"""Python binding of libglga (the C ABI in include/glga.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch supplies device memory (tensor.data_ptr()) and streams
(torch.cuda.current_stream().cuda_stream).  The binding raises if libglga.so is missing;
there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libglga.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "glga.h")

GLGA_F32, GLGA_BF16 = 0, 1
STATUS = {0: "GLGA_OK", 1: "GLGA_ERR_INVALID_ARG", 2: "GLGA_ERR_BAD_GRAPH",
          3: "GLGA_ERR_UNSUPPORTED", 4: "GLGA_ERR_OOM", 5: "GLGA_ERR_CUDA",
          6: "GLGA_ERR_TIMEOUT", 7: "GLGA_ERR_DEVICE"}
STAGES = ("prep", "gemm", "stats", "local", "readout", "forward")


class GLGAError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {message}")
        self.status = status


class Options(ctypes.Structure):
    _fields_ = [("warp_max_degree", ctypes.c_int32), ("chunk_edges", ctypes.c_int32),
                ("debug_checks", ctypes.c_int32), ("debug_fail_alloc", ctypes.c_int32),
                ("backward", ctypes.c_int32), ("fuse_stats", ctypes.c_int32)]


_lib = None
_vp, _i64, _i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32


def declared_symbols() -> list[str]:
    """Names of the entry points declared in include/glga.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"GLGA_API\s+[\w\s\*]*?\b(glga_\w+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_graph_attention_tcgen05_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "glga_default_options": ([ctypes.POINTER(Options)], _i32),
        "glga_create": ([ctypes.POINTER(_vp), _i64, _i32, _i32, _i32, _i32, _vp, _vp, _i64,
                         ctypes.POINTER(Options), _vp], _i32),
        "glga_forward": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float, _vp, _vp], _i32),
        "glga_create_segmented": ([ctypes.POINTER(_vp), _i64, _i32, _i32, _i32, _i32, _vp, _vp, _i64,
                                   _vp, _i64, ctypes.POINTER(Options), _vp], _i32),
        "glga_create_sharded": ([ctypes.POINTER(_vp), _i64, _i64, _i64, _i32, _i32, _i32, _i32, _vp, _vp,
                                 _i64, _vp, ctypes.POINTER(Options), _vp], _i32),
        "glga_forward_begin": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
        "glga_forward_end": ([_vp, _vp, _i32, ctypes.c_float, ctypes.c_float, _vp, _vp], _i32),
        "glga_backward": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float, _vp, _vp, _vp, _vp,
                           _vp, _vp, _vp, _vp], _i32),
        "glga_block_output": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp], _i32),
        "glga_destroy": ([_vp], _i32),
        "glga_csr_from_coo": ([_i64, _i64, _vp, _vp, _vp, _vp, _vp], _i32),
        "glga_bucket_counts": ([_vp, ctypes.POINTER(_i64)], _i32),
        "glga_get_buckets": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
        "glga_get_intermediates": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
        "glga_set_timing": ([_vp, ctypes.c_int], _i32),
        "glga_stage_times": ([_vp, ctypes.POINTER(ctypes.c_float), _i32, ctypes.POINTER(_i32)], _i32),
        "glga_workspace_bytes": ([_vp, ctypes.POINTER(_i64)], _i32),
        "glga_kernel_launches": ([_vp, ctypes.POINTER(_i64)], _i32),
        "glga_global_stats_static": ([_vp, _i64, _i32, _i32, _i32, _vp, _vp], _i32),
        "glga_global_stats_static_error": ([_vp], _i32),
        "glga_debug_static_bounded_wait": ([_i64, _vp], _i32),
        "glga_last_device_error": ([_vp, _vp], _i32),
        "glga_debug_bounded_wait": ([_vp, _i64, _vp], _i32),
        "glga_debug_set_col_idx": ([_vp, _i64, _i32, _vp], _i32),
        "glga_status_string": ([_i32], ctypes.c_char_p),
        "glga_last_error_message": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(status: int, where: str):
    if status != 0:
        msg = lib().glga_last_error_message().decode(errors="replace")
        raise GLGAError(status, where, msg)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def torch_dtype(io: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[io]


def default_options() -> Options:
    o = Options()
    _check(lib().glga_default_options(ctypes.byref(o)), "glga_default_options")
    return o


def csr_from_coo(N: int, src: torch.Tensor, dst: torch.Tensor, stream=None):
    """Target-grouped CSR (rows = targets, ascending sources) built on the GPU."""
    assert src.is_cuda and dst.is_cuda and src.dtype == torch.int32 and dst.dtype == torch.int32
    src, dst = src.contiguous(), dst.contiguous()
    E = src.numel()
    row_ptr = torch.empty(N + 1, dtype=torch.int32, device=src.device)
    col_idx = torch.empty(max(E, 1), dtype=torch.int32, device=src.device)
    _check(lib().glga_csr_from_coo(N, E, _ptr(src), _ptr(dst), _ptr(row_ptr), _ptr(col_idx),
                                   _stream(stream)), "glga_csr_from_coo")
    return row_ptr, col_idx[:E]


def global_stats_static(KV: torch.Tensor, H: int, r: int, io: str, Sz=None, stream=None):
    """S [H, r, r] and z [H, r] from KV [N, 2*H*r] (row j = k_j | v_j) without any device
    allocation inside the library (partial sums use its fixed static scratch).  Returns
    the Sz buffer: S followed by z."""
    assert KV.is_cuda and KV.is_contiguous() and KV.dtype == torch_dtype(io)
    N = KV.shape[0]
    if Sz is None:
        Sz = torch.empty(H * r * r + H * r, dtype=torch.float32, device=KV.device)
    _check(lib().glga_global_stats_static(_ptr(KV) if N else None, N, H, r,
                                          GLGA_F32 if io == "f32" else GLGA_BF16, _ptr(Sz),
                                          _stream(stream)), "glga_global_stats_static")
    return Sz


def global_stats_static_error(stream=None) -> int:
    """Status of the global_stats_static calls on the current device since the last report
    (glga_global_stats_static_error; synchronises the stream and clears the flag)."""
    return int(lib().glga_global_stats_static_error(_stream(stream)))


class Layer:
    """One gated local-global graph-attention layer bound to a fixed graph.

    `row_ptr`/`col_idx` are CUDA int32 tensors (target-grouped CSR).  `io` is "f32" or
    "bf16": the element type of X, the weights and Y.  `segments` (optional) are the
    n_seg + 1 node offsets of a batch of graphs (glga_create_segmented): each segment gets
    its own global statistics."""

    def __init__(self, N, d, H, r, io, row_ptr, col_idx, options: Options | None = None,
                 stream=None, segments=None):
        self.N, self.d, self.H, self.r, self.io = int(N), int(d), int(H), int(r), io
        self.D = self.H * self.r
        self.dtype = torch_dtype(io)
        self.device = row_ptr.device
        assert row_ptr.is_cuda and row_ptr.dtype == torch.int32 and row_ptr.numel() == N + 1
        assert col_idx.dtype == torch.int32
        self.E = int(col_idx.numel())
        h = ctypes.c_void_p()
        opt = ctypes.byref(options) if options is not None else None
        io_code = GLGA_F32 if io == "f32" else GLGA_BF16
        rpt, cit = row_ptr.contiguous(), col_idx.contiguous()   # alive through create
        rp = _ptr(rpt)
        ci = _ptr(cit) if self.E else None
        if segments is None:
            self.n_seg = None
            _check(lib().glga_create(ctypes.byref(h), self.N, self.d, self.H, self.r, io_code, rp, ci,
                                     self.E, opt, _stream(stream)), "glga_create")
        else:
            seg = np.ascontiguousarray(np.asarray(segments, dtype=np.int64))
            self.n_seg = int(seg.shape[0]) - 1
            _check(lib().glga_create_segmented(ctypes.byref(h), self.N, self.d, self.H, self.r, io_code,
                                               rp, ci, self.E, seg.ctypes.data, self.n_seg, opt,
                                               _stream(stream)), "glga_create_segmented")
        self._h = h

    # -- forward ---------------------------------------------------------------------
    def forward(self, X, W_Q, W_K, W_V, w_g, b_g: float, eps: float, Y=None, stream=None):
        for t in (X, W_Q, W_K, W_V, w_g):
            assert t.dtype == self.dtype and t.is_cuda and t.is_contiguous()
        assert X.shape == (self.N, self.d) and w_g.numel() == self.d
        if Y is None:
            Y = torch.empty(self.N, self.D, dtype=self.dtype, device=X.device)
        _check(lib().glga_forward(self._h, _ptr(X), _ptr(W_Q), _ptr(W_K), _ptr(W_V), _ptr(w_g),
                                  float(b_g), float(eps), _ptr(Y), _stream(stream)),
               "glga_forward")
        return Y

    __call__ = forward

    def capture(self, X, W_Q, W_K, W_V, w_g, b_g: float, eps: float, Y=None):
        """Records one glga_forward on these buffers into a CUDA graph and returns
        (graph, Y): graph.replay() reruns the whole forward on the same X, weights and Y
        (refill them in place between replays; b_g and eps are fixed at capture; the graph
        holds references to all six buffers, so they live as long as it does).  The
        forward enqueues kernels only (no allocation, no host synchronisation, tensor maps
        passed by value), so it records whole; one eager call first settles the lazy
        per-kernel attributes outside the capture.  With stage timing on, the stage events
        are captured as event record nodes, so stage_times() after a replay reports that
        replay's stages."""
        if Y is None:
            Y = torch.empty(self.N, self.D, dtype=self.dtype, device=X.device)
        side = torch.cuda.Stream(device=X.device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward(X, W_Q, W_K, W_V, w_g, b_g, eps, Y=Y)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            self.forward(X, W_Q, W_K, W_V, w_g, b_g, eps, Y=Y)
        # the replays read and write these buffers: the graph keeps them alive, so that a
        # caller dropping its own references cannot hand their memory to another tensor
        graph.glga_buffers = (X, W_Q, W_K, W_V, w_g, Y)
        return graph, Y

    # -- introspection ---------------------------------------------------------------
    def bucket_counts(self):
        c = (_i64 * 4)()
        _check(lib().glga_bucket_counts(self._h, c), "glga_bucket_counts")
        return [int(x) for x in c]

    def buckets(self, stream=None) -> dict:
        n = self.bucket_counts()
        out = {k: torch.empty(max(m, 1), dtype=torch.int32, device=self.device)
               for k, m in zip(("warp_rows", "cta_rows", "split_rows", "chunk_row", "chunk_begin"),
                               (n[0], n[1], n[2], n[3], n[3]))}
        _check(lib().glga_get_buckets(self._h, *(_ptr(out[k]) for k in
                                                 ("warp_rows", "cta_rows", "split_rows",
                                                  "chunk_row", "chunk_begin")),
                                      _stream(stream)), "glga_get_buckets")
        sizes = {"warp_rows": n[0], "cta_rows": n[1], "split_rows": n[2], "chunk_row": n[3],
                 "chunk_begin": n[3]}
        return {k: v[: sizes[k]] for k, v in out.items()}

    def intermediates(self, stream=None) -> dict:
        dev = self.device
        out = {"Q": torch.empty(self.N, self.D, dtype=self.dtype, device=dev),
               "K": torch.empty(self.N, self.D, dtype=self.dtype, device=dev),
               "V": torch.empty(self.N, self.D, dtype=self.dtype, device=dev),
               "t": torch.empty(self.N, dtype=torch.float32, device=dev),
               "S": torch.empty(self.n_seg or 1, self.H, self.r, self.r, dtype=torch.float32, device=dev),
               "z": torch.empty(self.n_seg or 1, self.H, self.r, dtype=torch.float32, device=dev),
               "L": torch.empty(self.N, self.D, dtype=self.dtype, device=dev)}
        _check(lib().glga_get_intermediates(self._h, *(_ptr(out[k]) for k in ("Q", "K", "V", "t", "S", "z", "L")),
                                            _stream(stream)), "glga_get_intermediates")
        if self.n_seg is None:           # one global segment: S [H, r, r], z [H, r]
            out["S"], out["z"] = out["S"][0], out["z"][0]
        return out

    def backward(self, X, W_Q, W_K, W_V, w_g, b_g: float, eps: float, dY, stream=None) -> dict:
        """fp32 gradients of sum(Y * dY) (glga_backward); call after forward() with the
        same inputs."""
        for t in (X, W_Q, W_K, W_V, w_g, dY):
            assert t.dtype == self.dtype and t.is_cuda and t.is_contiguous()
        dev = X.device
        f32 = torch.float32
        out = {"dX": torch.empty(self.N, self.d, dtype=f32, device=dev),
               "dW_Q": torch.empty(self.d, self.D, dtype=f32, device=dev),
               "dW_K": torch.empty(self.d, self.D, dtype=f32, device=dev),
               "dW_V": torch.empty(self.d, self.D, dtype=f32, device=dev),
               "dw_g": torch.empty(self.d, dtype=f32, device=dev),
               "db_g": torch.empty(1, dtype=f32, device=dev)}
        _check(lib().glga_backward(self._h, _ptr(X), _ptr(W_Q), _ptr(W_K), _ptr(W_V), _ptr(w_g),
                                   float(b_g), float(eps), _ptr(dY),
                                   *(_ptr(out[k]) for k in ("dX", "dW_Q", "dW_K", "dW_V", "dw_g", "db_g")),
                                   _stream(stream)), "glga_backward")
        return out

    def capture_backward(self, X, W_Q, W_K, W_V, w_g, b_g: float, eps: float, dY):
        """Records one glga_backward on these buffers into a CUDA graph and returns
        (graph, grads): graph.replay() recomputes the gradients into the same tensors from
        the state of the last forward (run forward() or its graph first when the inputs
        change).  The backward enqueues kernels and events between its two streams (the
        tensor maps of its GEMMs passed by value), so it records whole; one eager call
        first settles the lazily loaded kernels outside the capture."""
        side = torch.cuda.Stream(device=X.device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.backward(X, W_Q, W_K, W_V, w_g, b_g, eps, dY)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            grads = self.backward(X, W_Q, W_K, W_V, w_g, b_g, eps, dY)
        graph.glga_buffers = (X, W_Q, W_K, W_V, w_g, dY, grads)   # kept alive with the graph
        return graph, grads

    def block_output(self, Y, X, Wo, gamma, beta, ln_eps: float = 1e-5, Z=None, stream=None):
        """Z = LayerNorm(X + Y Wo) (glga_block_output)."""
        for t in (Y, X, Wo, gamma, beta):
            assert t.dtype == self.dtype and t.is_cuda and t.is_contiguous()
        if Z is None:
            Z = torch.empty(X.shape[0], self.d, dtype=self.dtype, device=X.device)
        _check(lib().glga_block_output(self._h, _ptr(Y), _ptr(X), _ptr(Wo), _ptr(gamma), _ptr(beta),
                                       float(ln_eps), _ptr(Z), _stream(stream)), "glga_block_output")
        return Z

    def set_timing(self, enable: bool):
        _check(lib().glga_set_timing(self._h, 1 if enable else 0), "glga_set_timing")

    def stage_times(self) -> dict:
        ms = (ctypes.c_float * 6)()
        n = _i32()
        _check(lib().glga_stage_times(self._h, ms, 6, ctypes.byref(n)), "glga_stage_times")
        return {STAGES[i]: float(ms[i]) for i in range(n.value)}

    def workspace_bytes(self) -> int:
        b = _i64()
        _check(lib().glga_workspace_bytes(self._h, ctypes.byref(b)), "glga_workspace_bytes")
        return int(b.value)

    def kernel_launches(self) -> int:
        n = _i64()
        _check(lib().glga_kernel_launches(self._h, ctypes.byref(n)), "glga_kernel_launches")
        return int(n.value)

    def last_device_error(self, stream=None) -> int:
        return int(lib().glga_last_device_error(self._h, _stream(stream)))

    def debug_bounded_wait(self, limit_ns: int, stream=None):
        """Enqueue the bounded-wait probe (see glga_debug_bounded_wait)."""
        _check(lib().glga_debug_bounded_wait(self._h, int(limit_ns), _stream(stream)),
               "glga_debug_bounded_wait")

    def debug_set_col_idx(self, e: int, value: int, stream=None):
        """Overwrite one CSR entry of a debug_checks context (see glga_debug_set_col_idx)."""
        _check(lib().glga_debug_set_col_idx(self._h, int(e), int(value), _stream(stream)),
               "glga_debug_set_col_idx")

    def close(self):
        if getattr(self, "_h", None):
            lib().glga_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class HostInputs:
    """Page-locked host staging of one layer's inputs for host-to-device use.

    X [N, d] and W_Q, W_K, W_V [d, D] and w_g [d] live in ONE pinned slab, each piece at a
    256-byte aligned offset, so a step's inputs cross PCIe as a single host->device copy
    instead of five (measured on B200 with arxiv-sized inputs: the four small weight copies
    issued beside X's lengthened a pipelined copy-in/forward/copy-out step by 7-14 %).
    `slots` device twins of the slab let copies of one step overlap the forward of another.

    Fill the host views (`host["X"]`, ...) in place; `upload(slot, stream)` enqueues the
    copy of the whole slab into device slot `slot` on `stream` and returns that slot's
    device views in forward's argument order (X, W_Q, W_K, W_V, w_g).  The copy reads the
    slab when the stream reaches it: refill the host views only after it has completed
    (an event recorded after upload).  Ordering the copy against forwards that still read
    the slot is the caller's as well (stream events)."""

    NAMES = ("X", "W_Q", "W_K", "W_V", "w_g")

    def __init__(self, N: int, d: int, D: int, dtype: torch.dtype, device, slots: int = 2):
        shapes = {"X": (N, d), "W_Q": (d, D), "W_K": (d, D), "W_V": (d, D), "w_g": (d,)}
        esz = torch.empty((), dtype=dtype).element_size()
        align = 256 // esz
        self._offs, total = {}, 0
        for k in self.NAMES:
            self._offs[k] = total
            n = int(np.prod(shapes[k]))
            total += (n + align - 1) // align * align
        self._shapes = shapes
        self.slab = torch.zeros(total, dtype=dtype).pin_memory()
        self.host = self._views(self.slab)
        self._dev = [torch.empty(total, dtype=dtype, device=device) for _ in range(int(slots))]
        self.device_inputs = [tuple(self._views(b)[k] for k in self.NAMES) for b in self._dev]

    def _views(self, buf: torch.Tensor) -> dict:
        out = {}
        for k in self.NAMES:
            n = int(np.prod(self._shapes[k]))
            out[k] = buf[self._offs[k]:self._offs[k] + n].view(self._shapes[k])
        return out

    @property
    def nbytes(self) -> int:
        """Bytes one upload copies (the slab, alignment padding included)."""
        return self.slab.numel() * self.slab.element_size()

    def upload(self, slot: int, stream=None):
        """Enqueue the host->device copy of the slab into `slot`; returns its device views."""
        s = stream if stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(s):
            self._dev[slot].copy_(self.slab, non_blocking=True)
        return self.device_inputs[slot]
