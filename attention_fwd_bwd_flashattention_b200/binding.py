"""Thin ctypes binding of the C ABI in include/relpos_attn.h.

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch provides device memory and the current stream.  If the
compiled library is missing this module raises; there is no other code path.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

T5, SHAW, TXL, DEBERTA, ALIBI = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
PATH_AUTO, PATH_SIMT, PATH_TC = 0, 1, 2

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "librelpos_attn.so")
_lib = None


class RelposError(RuntimeError):
    def __init__(self, code: int, what: str):
        detail = ""
        if code == -4:  # RELPOS_ERR_LAUNCH: name the CUDA error behind it
            detail = f"; cudaError {load().relpos_last_cuda_error()}"
        super().__init__(f"{what}: {strerror(code)} ({code}{detail})")
        self.code = code


class relpos_params_t(ctypes.Structure):
    _fields_ = [
        ("mech", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("kernel_path", ctypes.c_int32),
        ("B", ctypes.c_int64),
        ("H", ctypes.c_int64),
        ("L", ctypes.c_int64),
        ("d", ctypes.c_int64),
        ("scale", ctypes.c_float),
        ("t5_num_buckets", ctypes.c_int32),
        ("t5_max_distance", ctypes.c_int32),
        ("t5_bidirectional", ctypes.c_int32),
        ("shaw_clip", ctypes.c_int32),
        ("deberta_span", ctypes.c_int32),
        ("seqlens_k", ctypes.c_void_p),
        ("shaw_value", ctypes.c_int32),
        ("mem_len", ctypes.c_int64),
    ]


TRACE_MAX = 64


class relpos_trace_t(ctypes.Structure):
    _fields_ = [
        ("events", ctypes.POINTER(ctypes.c_void_p)),
        ("capacity", ctypes.c_int32),
        ("count", ctypes.c_int32),
        ("dropped", ctypes.c_int32),
        ("only", ctypes.c_char_p),
        ("names", ctypes.c_char_p * TRACE_MAX),
    ]


EXPORTS = ("relpos_attn_workspace_size", "relpos_attn_fwd", "relpos_attn_bwd", "relpos_attn_fwd_noalloc",
           "relpos_attn_resolved_path", "relpos_selftest_wait", "relpos_trace_begin", "relpos_trace_end",
           "relpos_last_cuda_error", "relpos_strerror", "relpos_attn_version")
NOALLOC_SCRATCH_BYTES = 16 << 20


def lib_path() -> str:
    return _LIB_PATH


RELEASE_LIB = _LIB_PATH
DEBUG_LIB = os.path.join(os.path.dirname(_LIB_PATH), "librelpos_attn_debug.so")


def use_library(path: str) -> None:
    """Bind every wrapper to the library at `path` from now on (e.g. the RELPOS_DEBUG
    build, _lib/librelpos_attn_debug.so, in tests)."""
    global _lib, _LIB_PATH
    _LIB_PATH = path
    _lib = None


def load() -> ctypes.CDLL:
    """Load the compiled library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {_LIB_PATH} (run python -m attention_fwd_bwd_flashattention_b200.build)")
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.POINTER(relpos_params_t)
    vp = ctypes.c_void_p
    lib.relpos_attn_workspace_size.argtypes = [P, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
    lib.relpos_attn_workspace_size.restype = ctypes.c_int
    lib.relpos_attn_fwd.argtypes = [P, vp, vp, vp, ctypes.POINTER(vp), vp, vp, vp, ctypes.c_size_t, vp, vp]
    lib.relpos_attn_fwd.restype = ctypes.c_int
    lib.relpos_attn_bwd.argtypes = [P, vp, vp, vp, ctypes.POINTER(vp), vp, vp, vp, vp, vp, vp, ctypes.POINTER(vp), vp,
                                    ctypes.c_size_t, vp, vp]
    lib.relpos_attn_bwd.restype = ctypes.c_int
    lib.relpos_attn_fwd_noalloc.argtypes = [P, vp, vp, vp, ctypes.POINTER(vp), vp, vp, vp, vp]
    lib.relpos_attn_fwd_noalloc.restype = ctypes.c_int
    lib.relpos_attn_resolved_path.argtypes = [P, ctypes.c_int]
    lib.relpos_attn_resolved_path.restype = ctypes.c_int
    lib.relpos_selftest_wait.argtypes = [ctypes.c_uint64, vp, vp, vp]
    lib.relpos_selftest_wait.restype = ctypes.c_int
    lib.relpos_trace_begin.argtypes = [ctypes.POINTER(relpos_trace_t)]
    lib.relpos_trace_begin.restype = ctypes.c_int
    lib.relpos_trace_end.argtypes = []
    lib.relpos_trace_end.restype = ctypes.c_int
    lib.relpos_strerror.argtypes = [ctypes.c_int]
    lib.relpos_strerror.restype = ctypes.c_char_p
    lib.relpos_last_cuda_error.argtypes = []
    lib.relpos_last_cuda_error.restype = ctypes.c_int
    lib.relpos_attn_version.argtypes = []
    lib.relpos_attn_version.restype = ctypes.c_int
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().relpos_strerror(int(code)).decode()


@dataclass
class Params:
    mech: int
    B: int
    H: int
    L: int
    d: int = 64
    dtype: int = BF16
    causal: bool = False
    scale: Optional[float] = None
    kernel_path: int = PATH_AUTO
    t5_num_buckets: int = 32
    t5_max_distance: int = 128
    t5_bidirectional: bool = True
    shaw_clip: int = 64
    deberta_span: int = 256
    seqlens_k: Optional[torch.Tensor] = None  # [B] int32 on the device, or None (all L)
    shaw_value: bool = False  # Shaw: rel[1] = aV, the value-side table
    mem_len: int = 0  # Transformer-XL (causal): memory length M; k, v and r then have M + L rows

    def c(self) -> relpos_params_t:
        scale = self.scale
        if scale is None:
            scale = 1.0 / math.sqrt(3 * self.d) if self.mech == DEBERTA else 1.0 / math.sqrt(self.d)
        if self.seqlens_k is not None:
            t = self.seqlens_k
            if t.dtype != torch.int32 or t.numel() != self.B or not t.is_contiguous():
                raise ValueError("seqlens_k must be a contiguous int32 tensor of B elements")
        return relpos_params_t(self.mech, self.dtype, int(self.causal), self.kernel_path, self.B, self.H, self.L, self.d,
                               float(scale), self.t5_num_buckets, self.t5_max_distance, int(self.t5_bidirectional),
                               self.shaw_clip, self.deberta_span, _ptr(self.seqlens_k), int(self.shaw_value),
                               int(self.mem_len))

    def n_rel(self) -> int:
        if self.mech == SHAW and self.shaw_value:
            return 2
        return {T5: 1, SHAW: 1, TXL: 3, DEBERTA: 2, ALIBI: 1}[self.mech]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _ptr_array(ts: Sequence[Optional[torch.Tensor]]):
    arr = (ctypes.c_void_p * 3)()
    for i in range(3):
        arr[i] = _ptr(ts[i]) if i < len(ts) else None
    return arr


def _on_device_of(t):
    """The library launches on the calling thread's current CUDA device: make the
    tensor's device current for the call (as torch's own ops do)."""
    if isinstance(t, torch.Tensor) and t.is_cuda:
        return torch.cuda.device(t.device)
    return contextlib.nullcontext()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# one-to-one wrappers of the C entry points
# ---------------------------------------------------------------------------
def relpos_attn_workspace_size(params: Params, pass_: int) -> int:
    n = ctypes.c_size_t(0)
    cp = params.c()
    rc = load().relpos_attn_workspace_size(ctypes.byref(cp), int(pass_), ctypes.byref(n))
    if rc != 0:
        raise RelposError(rc, "relpos_attn_workspace_size")
    return int(n.value)


def relpos_attn_resolved_path(params: Params, pass_: int = 0) -> int:
    cp = params.c()
    rc = load().relpos_attn_resolved_path(ctypes.byref(cp), int(pass_))
    if rc < 0:
        raise RelposError(rc, "relpos_attn_resolved_path")
    return rc


def tc_available(params: Params, pass_: int = 0) -> bool:
    """True when pass `pass_` (0 forward, 1 backward) runs on the tensor-core (tcgen05) kernels."""
    return relpos_attn_resolved_path(params, pass_) == PATH_TC


def relpos_attn_fwd(params: Params, q, k, v, rel, o, lse, workspace, dev_status=None, stream=None) -> None:
    cp = params.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _on_device_of(q):
        rc = load().relpos_attn_fwd(ctypes.byref(cp), _ptr(q), _ptr(k), _ptr(v), _ptr_array(rel), _ptr(o), _ptr(lse),
                                    _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    if rc != 0:
        raise RelposError(rc, "relpos_attn_fwd")


def relpos_attn_fwd_noalloc(params: Params, q, k, v, rel, o, lse, dev_status=None, stream=None) -> None:
    """Forward pass that allocates nothing: its scratch is the library's built-in
    device array (see relpos_attn_fwd_noalloc in include/relpos_attn.h)."""
    cp = params.c()
    with _on_device_of(q):
        rc = load().relpos_attn_fwd_noalloc(ctypes.byref(cp), _ptr(q), _ptr(k), _ptr(v), _ptr_array(rel), _ptr(o),
                                            _ptr(lse), _ptr(dev_status), _stream(stream))
    if rc != 0:
        raise RelposError(rc, "relpos_attn_fwd_noalloc")


def relpos_selftest_wait(limit_ns: int, dev_status, dev_elapsed_ns, stream=None) -> None:
    """Bounded-wait self-test (see include/relpos_attn.h): dev_status int32 [1] and
    dev_elapsed_ns int64 [1] device tensors receive RELPOS_ERR_TIMEOUT and the wait's
    duration."""
    rc = load().relpos_selftest_wait(int(limit_ns), _ptr(dev_status), _ptr(dev_elapsed_ns), _stream(stream))
    if rc != 0:
        raise RelposError(rc, "relpos_selftest_wait")


class Trace:
    """Device time of every kernel the library launches from this thread while the
    context is active (relpos_trace_begin / relpos_trace_end): each kernel is bracketed
    by two CUDA events on its launch stream.  After synchronising, ``kernels()`` gives
    [(name, milliseconds)] in launch order.  ``only``: record only the kernels of that
    name (two events per launch of it, nothing between the others)."""

    def __init__(self, capacity: int = TRACE_MAX, only: Optional[str] = None):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.events:  # torch creates the CUDA event at its first record
            e.record()
        self._handles = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.events])
        self.c = relpos_trace_t()
        self.c.events = ctypes.cast(self._handles, ctypes.POINTER(ctypes.c_void_p))
        self.c.capacity = capacity
        self._only = None if only is None else only.encode()
        self.c.only = self._only

    def __enter__(self):
        rc = load().relpos_trace_begin(ctypes.byref(self.c))
        if rc != 0:
            raise RelposError(rc, "relpos_trace_begin")
        return self

    def __exit__(self, *exc):
        load().relpos_trace_end()
        return False

    def kernels(self):
        return [(self.c.names[k].decode(), self.events[2 * k].elapsed_time(self.events[2 * k + 1]))
                for k in range(self.c.count)]


def relpos_attn_bwd(params: Params, q, k, v, rel, o, lse, dout, dq, dk, dv, drel, workspace, dev_status=None,
                    stream=None) -> None:
    cp = params.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _on_device_of(q):
        rc = load().relpos_attn_bwd(ctypes.byref(cp), _ptr(q), _ptr(k), _ptr(v), _ptr_array(rel), _ptr(o), _ptr(lse),
                                    _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr_array(drel), _ptr(workspace), ws_bytes,
                                    _ptr(dev_status), _stream(stream))
    if rc != 0:
        raise RelposError(rc, "relpos_attn_bwd")


# ---------------------------------------------------------------------------
# convenience: allocate outputs / workspace with torch and call the C entry points
# ---------------------------------------------------------------------------
def params_for(mech, q: torch.Tensor, causal: bool, scale=None, kernel_path=PATH_AUTO, **cfg) -> Params:
    B, H, L, d = q.shape
    dt = BF16 if q.dtype == torch.bfloat16 else F32
    return Params(mech=mech, B=B, H=H, L=L, d=d, dtype=dt, causal=causal, scale=scale, kernel_path=kernel_path, **cfg)


def workspace(params: Params, pass_: int, device) -> Optional[torch.Tensor]:
    n = relpos_attn_workspace_size(params, pass_)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def forward(params: Params, q, k, v, rel, ws=None, stream=None):
    """Returns (O, LSE)."""
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(params, 0, q.device)
    relpos_attn_fwd(params, q, k, v, rel, o, lse, ws, stream=stream)
    return o, lse


def backward(params: Params, q, k, v, rel, o, lse, dout, ws=None, stream=None):
    """Returns (dQ, dK, dV, [drel...]) with drel float32, shaped like rel."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    drel = [torch.empty(r.shape, dtype=torch.float32, device=q.device) for r in rel[: params.n_rel()]]
    if ws is None:
        ws = workspace(params, 1, q.device)
    relpos_attn_bwd(params, q, k, v, rel, o, lse, dout, dq, dk, dv, drel, ws, stream=stream)
    return dq, dk, dv, drel
