"""Python binding of ``libbsa.so``: block-sparse causal attention on B200
(forward, gradients, selected-page decode).

Argument marshalling only.  Every step of the computation runs in the
library's CUDA kernel or its host layout compiler; this module converts Python
values and torch tensors to the C ABI declared in ``include/bsa.h`` and turns
non-zero status codes into :class:`BsaError`.  There is no fallback: if the
shared library is missing or cannot be loaded, every call raises.

Names follow the C ABI: ``bsa_build_layout``, ``bsa_layout_csr``,
``bsa_layout_csc``, ``bsa_layout_order``, ``bsa_layout_segments``,
``bsa_forward``, ``bsa_forward_noalloc``, ``bsa_backward``, ``bsa_decode``,
``bsa_get_status``, ``bsa_debug_timeout_probe``, ``bsa_free`` and
``bsa_last_error``; the ``Layout`` class, ``attention``, ``attention_backward``
and ``decode`` are conveniences over them.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import numpy as np

from .workloads import (PATTERN_BAND_GLOBAL, PATTERN_DYADIC, PATTERN_RANDOM,  # noqa: F401
                        PATTERN_EXPLICIT)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

BSA_OK = 0
STATUS_NAMES = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_SHAPE", 3: "BSA_ERR_UNSUPPORTED",
                4: "BSA_ERR_NONCAUSAL", 5: "BSA_ERR_CUDA", 6: "BSA_ERR_OOM",
                7: "BSA_ERR_DEVICE_TIMEOUT"}

EXPORTED = ["bsa_build_layout", "bsa_layout_csr", "bsa_layout_csc", "bsa_layout_order", "bsa_layout_work",
            "bsa_layout_segments", "bsa_forward", "bsa_forward_host", "bsa_forward_noalloc", "bsa_backward",
            "bsa_decode",
            "bsa_bsbr_workspace_bytes", "bsa_bsbr_retrieval", "bsa_get_status", "bsa_debug_timeout_probe",
            "bsa_free", "bsa_last_error"]


class BsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


class bsa_pattern(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("window", ctypes.c_int32),
                ("global_first", ctypes.c_int32), ("dyadic_kmin", ctypes.c_int32),
                ("density", ctypes.c_double), ("seed", ctypes.c_uint64),
                ("mask", ctypes.POINTER(ctypes.c_uint8))]


_lib = None
_lib_lock = threading.Lock()


def load_library(path: str = LIB_PATH):
    """Load (once) and return the ctypes handle; raises if the library is absent."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"libbsa.so not found at {path}; build it with "
                               "`python -m block_sparse_long_bsa_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, U64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_float
        lib.bsa_build_layout.argtypes = [ctypes.POINTER(bsa_pattern), I, I, I, I, ctypes.POINTER(P)]
        lib.bsa_build_layout.restype = I
        lib.bsa_layout_csr.argtypes = [P, ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                       ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                       ctypes.POINTER(I), ctypes.POINTER(I)]
        lib.bsa_layout_csr.restype = I
        lib.bsa_layout_csc.argtypes = [P, ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                       ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                       ctypes.POINTER(I), ctypes.POINTER(I)]
        lib.bsa_layout_csc.restype = I
        lib.bsa_layout_order.argtypes = [P, ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                         ctypes.POINTER(I)]
        lib.bsa_layout_order.restype = I
        lib.bsa_layout_work.argtypes = [P, ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                        ctypes.POINTER(I)]
        lib.bsa_layout_work.restype = I
        lib.bsa_forward.argtypes = [P, P, P, P, I, I, I, I, I, F, P, P, P]
        lib.bsa_forward.restype = I
        lib.bsa_forward_noalloc.argtypes = [P, P, P, P, I, I, I, I, I, F, P, P, P]
        lib.bsa_forward_noalloc.restype = I
        lib.bsa_forward_host.argtypes = [P, P, P, P, I, I, I, I, I, F, P, P, P, P, P, P, P, I, P]
        lib.bsa_forward_host.restype = I
        lib.bsa_decode.argtypes = [P, P, P, P, I, I, P, P, I, I, I, I, F, P, P, P]
        lib.bsa_decode.restype = I
        lib.bsa_backward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, P, P, P, P, P]
        lib.bsa_backward.restype = I
        lib.bsa_layout_segments.argtypes = [P, ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                            ctypes.POINTER(ctypes.POINTER(ctypes.c_int32)),
                                            ctypes.POINTER(I), ctypes.POINTER(I)]
        lib.bsa_layout_segments.restype = I
        lib.bsa_bsbr_workspace_bytes.argtypes = [I, I, I, I]
        lib.bsa_bsbr_workspace_bytes.restype = ctypes.c_size_t
        lib.bsa_bsbr_retrieval.argtypes = [P, P, P, P, I, I, I, I, I, F, P, P, ctypes.c_size_t, P]
        lib.bsa_bsbr_retrieval.restype = I
        lib.bsa_get_status.argtypes = [P, P]
        lib.bsa_get_status.restype = I
        lib.bsa_debug_timeout_probe.argtypes = [P, I, U64, P]
        lib.bsa_debug_timeout_probe.restype = I
        lib.bsa_free.argtypes = [P]
        lib.bsa_free.restype = None
        lib.bsa_last_error.argtypes = []
        lib.bsa_last_error.restype = ctypes.c_char_p
        _lib = lib
        return lib


def bsa_last_error() -> str:
    msg = load_library().bsa_last_error()
    return msg.decode() if msg else ""


def _check(status: int):
    if status != BSA_OK:
        raise BsaError(status, bsa_last_error())


def _ptr(x) -> int:
    """Device/host address of a torch tensor, or an int passed through."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int:
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:
            pass
        return 0
    if isinstance(s, int):
        return s
    return s.cuda_stream


def bsa_build_layout(kind: int, n: int, B: int, layout_heads: int = 1, device: int = -1,
                     window: int = 0, global_first: int = 0, dyadic_kmin: int = 2,
                     density: float = 0.0, seed: int = 0, mask=None) -> int:
    """Compile a pattern; returns the opaque layout handle (an int)."""
    lib = load_library()
    spec = bsa_pattern(kind, window, global_first, dyadic_kmin, density, seed & ((1 << 64) - 1), None)
    keep = None
    if mask is not None:
        keep = np.ascontiguousarray(mask, dtype=np.uint8)
        spec.mask = keep.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
    out = ctypes.c_void_p()
    _check(lib.bsa_build_layout(ctypes.byref(spec), n, B, layout_heads, device, ctypes.byref(out)))
    return out.value


def bsa_layout_csc(layout: int):
    """Copies of the transposed layout (col_ptr, row_idx) as int32 numpy arrays."""
    lib = load_library()
    cp = ctypes.POINTER(ctypes.c_int32)()
    ri = ctypes.POINTER(ctypes.c_int32)()
    cols, nnz = ctypes.c_int(), ctypes.c_int()
    _check(lib.bsa_layout_csc(layout, ctypes.byref(cp), ctypes.byref(ri), ctypes.byref(cols),
                              ctypes.byref(nnz)))
    col_ptr = np.ctypeslib.as_array(cp, shape=(cols.value + 1,)).copy()
    row_idx = (np.ctypeslib.as_array(ri, shape=(nnz.value,)).copy() if nnz.value
               else np.zeros(0, np.int32))
    return col_ptr, row_idx


def bsa_layout_segments(layout: int):
    """Copies of the key/value-gradient work list: (seg_ptr [L+1], segs [count, 3])."""
    lib = load_library()
    sp = ctypes.POINTER(ctypes.c_int32)()
    sg = ctypes.POINTER(ctypes.c_int32)()
    lh, cnt = ctypes.c_int(), ctypes.c_int()
    _check(lib.bsa_layout_segments(layout, ctypes.byref(sp), ctypes.byref(sg), ctypes.byref(lh),
                                   ctypes.byref(cnt)))
    seg_ptr = np.ctypeslib.as_array(sp, shape=(lh.value + 1,)).copy()
    segs = (np.ctypeslib.as_array(sg, shape=(cnt.value * 3,)).copy().reshape(-1, 3) if cnt.value
            else np.zeros((0, 3), np.int32))
    return seg_ptr, segs


def bsa_layout_csr(layout: int):
    """Copies of (row_ptr, col_idx) as int32 numpy arrays."""
    lib = load_library()
    rp = ctypes.POINTER(ctypes.c_int32)()
    ci = ctypes.POINTER(ctypes.c_int32)()
    rows, nnz = ctypes.c_int(), ctypes.c_int()
    _check(lib.bsa_layout_csr(layout, ctypes.byref(rp), ctypes.byref(ci), ctypes.byref(rows),
                              ctypes.byref(nnz)))
    row_ptr = np.ctypeslib.as_array(rp, shape=(rows.value + 1,)).copy()
    col_idx = (np.ctypeslib.as_array(ci, shape=(nnz.value,)).copy() if nnz.value
               else np.zeros(0, np.int32))
    return row_ptr, col_idx


def bsa_layout_order(layout: int) -> np.ndarray:
    lib = load_library()
    od = ctypes.POINTER(ctypes.c_int32)()
    cnt = ctypes.c_int()
    _check(lib.bsa_layout_order(layout, ctypes.byref(od), ctypes.byref(cnt)))
    return np.ctypeslib.as_array(od, shape=(cnt.value,)).copy()


def bsa_layout_work(layout: int) -> np.ndarray:
    """The forward's work table as an int32 array [layout_heads * nb, 4]."""
    lib = load_library()
    wk = ctypes.POINTER(ctypes.c_int32)()
    cnt = ctypes.c_int()
    _check(lib.bsa_layout_work(layout, ctypes.byref(wk), ctypes.byref(cnt)))
    return np.ctypeslib.as_array(wk, shape=(cnt.value * 4,)).copy().reshape(cnt.value, 4)


def bsa_forward(q, k, v, layout: int, B: int, n: int, heads: int, kv_heads: int, d: int,
                scale: float, o, lse, stream=None) -> None:
    """Enqueue the forward on ``stream`` (default: torch's current stream)."""
    lib = load_library()
    _check(lib.bsa_forward(_ptr(q), _ptr(k), _ptr(v), layout, B, n, heads, kv_heads, d,
                           ctypes.c_float(scale), _ptr(o), _ptr(lse), _stream(stream)))


def bsa_forward_host(q_host, k_host, v_host, layout: int, B: int, n: int, heads: int, kv_heads: int, d: int,
                     scale: float, q, k, v, o, lse, o_host, lse_host, groups: int = 8, stream=None) -> None:
    """Forward from and to host memory (see include/bsa.h): copies in head
    groups overlap the other groups' compute; synchronise ``stream`` before
    reading ``o_host`` and ``lse_host``."""
    lib = load_library()
    _check(lib.bsa_forward_host(_ptr(q_host), _ptr(k_host), _ptr(v_host), layout, B, n, heads, kv_heads, d,
                                ctypes.c_float(scale), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                _ptr(o_host), _ptr(lse_host), groups, _stream(stream)))


def bsa_forward_noalloc(q, k, v, layout: int, B: int, n: int, heads: int, kv_heads: int, d: int,
                        scale: float, o, lse, stream=None) -> None:
    """Allocation-free forward (see include/bsa.h): ``layout`` may be host-only;
    its arrays are staged in the library's static device block."""
    lib = load_library()
    _check(lib.bsa_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), layout, B, n, heads, kv_heads, d,
                                   ctypes.c_float(scale), _ptr(o), _ptr(lse), _stream(stream)))


def bsa_decode(q, k_cache, v_cache, page_table, max_blocks: int, num_pages: int, positions,
               layout: int, batch: int, heads: int, kv_heads: int, d: int, scale: float,
               o, lse, stream=None) -> None:
    """Enqueue one selected-page decode step (see include/bsa.h)."""
    lib = load_library()
    _check(lib.bsa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table), max_blocks,
                          num_pages, _ptr(positions), layout, batch, heads, kv_heads, d,
                          ctypes.c_float(scale), _ptr(o), _ptr(lse), _stream(stream)))


def bsa_backward(q, k, v, o, lse, dout, layout: int, B: int, n: int, heads: int, kv_heads: int,
                 d: int, scale: float, dq, dk, dv, workspace, stream=None) -> None:
    """Enqueue the gradients of the forward (see include/bsa.h)."""
    lib = load_library()
    _check(lib.bsa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), layout, B, n,
                            heads, kv_heads, d, ctypes.c_float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                            _ptr(workspace), _stream(stream)))


def attention_backward(q, k, v, o, lse, dout, layout: "Layout", scale: float | None = None,
                       dq=None, dk=None, dv=None, workspace=None, stream=None):
    """torch convenience: the forward's tensors plus dout [heads, n, d] bf16;
    returns fp32 (dq, dk, dv), allocating what is not given."""
    import torch
    heads, n, d = q.shape
    kv_heads = k.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise BsaError(1, "q, k, v, o and dout must be contiguous bf16 tensors")
    if dq is None:
        dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    if dv is None:
        dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty((heads, n), dtype=torch.float32, device=q.device)
    for t in (lse, dq, dk, dv, workspace):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise BsaError(1, "lse, dq, dk, dv and workspace must be contiguous float32 tensors")
    bsa_backward(q, k, v, o, lse, dout, layout.handle, layout.B, n, heads, kv_heads, d, scale,
                 dq, dk, dv, workspace, stream)
    return dq, dk, dv


def bsa_bsbr_workspace_bytes(n: int, B: int, kv_heads: int, d: int) -> int:
    return int(load_library().bsa_bsbr_workspace_bytes(n, B, kv_heads, d))


def bsa_bsbr_retrieval(q, k, v, layout: int, B: int, n: int, heads: int, kv_heads: int, d: int,
                       scale: float, o, workspace, workspace_bytes: int, stream=None) -> None:
    """Enqueue BSBR's between-chunk retrieval term, added to ``o`` (see include/bsa.h)."""
    lib = load_library()
    _check(lib.bsa_bsbr_retrieval(_ptr(q), _ptr(k), _ptr(v), layout, B, n, heads, kv_heads, d,
                                  ctypes.c_float(scale), _ptr(o), _ptr(workspace), workspace_bytes,
                                  _stream(stream)))


def bsbr_attention(q, k, v, layout: "Layout", scale: float | None = None, workspace=None, stream=None):
    """torch convenience: the whole BSBR attention output for a block-diagonal
    ``layout`` (within-chunk forward, then the retrieval term added in place)."""
    import torch
    heads, n, d = q.shape
    kv_heads = k.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o, lse = attention(q, k, v, layout, scale=scale, stream=stream)
    need = bsa_bsbr_workspace_bytes(n, layout.B, kv_heads, d)
    if workspace is None:
        workspace = torch.empty((max(need, 16) + 15) // 16 * 4, dtype=torch.float32, device=q.device)
    bsa_bsbr_retrieval(q, k, v, layout.handle, layout.B, n, heads, kv_heads, d, scale, o, workspace,
                       workspace.numel() * workspace.element_size(), stream)
    return o, lse


def decode(q, k_cache, v_cache, page_table, positions, layout: "Layout", batch: int,
           scale: float | None = None, o=None, lse=None, stream=None):
    """torch convenience: q [batch*H, d]; caches [pages, H_kv, B, d] bf16;
    page_table [batch, max_blocks] and positions [batch] int32, all on the GPU."""
    import torch
    heads, d = q.shape
    kv_heads = k_cache.shape[1] * batch
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((heads,), dtype=torch.float32, device=q.device)
    for t in (q, k_cache, v_cache, o):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise BsaError(1, "q, caches and o must be contiguous bf16 tensors")
    for t in (page_table, positions):
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise BsaError(1, "page_table and positions must be contiguous int32 tensors")
    bsa_decode(q, k_cache, v_cache, page_table, page_table.shape[1], k_cache.shape[0], positions,
               layout.handle, batch, heads, kv_heads, d, scale, o, lse, stream)
    return o, lse


def bsa_get_status(layout: int, stream=None) -> None:
    _check(load_library().bsa_get_status(layout, _stream(stream)))


def bsa_debug_timeout_probe(layout: int, d: int, timeout_ns: int, stream=None) -> None:
    _check(load_library().bsa_debug_timeout_probe(layout, d, timeout_ns, _stream(stream)))


def bsa_free(layout: int) -> None:
    if layout:
        load_library().bsa_free(layout)


class Layout:
    """Owning wrapper of a layout handle (freed on ``close`` or collection)."""

    def __init__(self, kind, n, B, layout_heads=1, device=-1, **pattern):
        self.n, self.B, self.layout_heads, self.device = n, B, layout_heads, device
        self.handle = bsa_build_layout(kind, n, B, layout_heads, device, **pattern)

    @classmethod
    def for_workload(cls, w, device=-1):
        p = w.pattern
        return cls(p.kind, w.n, w.B, w.layout_heads, device, window=p.window,
                   global_first=p.global_first, dyadic_kmin=p.dyadic_kmin,
                   density=p.density, seed=p.seed)

    def csr(self):
        return bsa_layout_csr(self.handle)

    def order(self):
        return bsa_layout_order(self.handle)

    def close(self):
        if getattr(self, "handle", None):
            bsa_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def attention(q, k, v, layout: Layout, scale: float | None = None, o=None, lse=None, stream=None):
    """torch convenience: q [heads, n, d], k/v [kv_heads, n, d] bf16 CUDA tensors.

    Allocates o / lse when not given and enqueues one ``bsa_forward``.
    """
    import torch
    heads, n, d = q.shape
    kv_heads = k.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((heads, n), dtype=torch.float32, device=q.device)
    for t in (q, k, v, o):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise BsaError(1, "q, k, v, o must be contiguous bf16 tensors")
    if lse.dtype != torch.float32 or not lse.is_contiguous():
        raise BsaError(1, "lse must be a contiguous float32 tensor")
    bsa_forward(q, k, v, layout.handle, layout.B, n, heads, kv_heads, d, scale, o, lse, stream)
    return o, lse
