"""Python binding of libattn.so: multi-head causal scaled dot-product
self-attention, forward and backward, on B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/attn.h.  PyTorch supplies device
memory and the current CUDA stream.  There is no CPU or library fallback: if
the shared library is missing, importing this package raises ImportError.

Functions mirror the C entry points and take [B, H, T, D] contiguous CUDA
tensors (bf16 for ``attn_fwd``/``attn_bwd``, float32 for the ``_f32`` pair);
outputs may be passed in or are allocated.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")
# ATTN_LIBRARY selects another build of the same library, e.g. libattn_debug.so
# (the kernels with device-side bounds checks, see build.py --debug).
if os.environ.get("ATTN_LIBRARY"):
    LIB_PATH = os.path.abspath(os.environ["ATTN_LIBRARY"])

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python decoder_only_transformer_sdpa_b200/build.py` "
        "(nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _fp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_lib.attn_status_string.argtypes = [_i]
_lib.attn_status_string.restype = ctypes.c_char_p
_lib.attn_version.restype = _i
_lib.attn_last_launch_count.restype = _i
_lib.attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _fp, _i, _i, _i, _i, _f, _vp]
_lib.attn_fwd.restype = _i
_lib.attn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
_lib.attn_bwd_workspace_bytes.restype = _sz
_lib.attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp, _sz, _vp]
_lib.attn_bwd.restype = _i
_lib.attn_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp]
_lib.attn_bwd_noalloc.restype = _i
class attn_strides(ctypes.Structure):
    """Element strides (batch, head, token) of one [B, H, T, D] operand."""
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("t", ctypes.c_int64)]


_sp = ctypes.POINTER(attn_strides)
_lib.attn_fwd_strided.argtypes = [_vp, _vp, _vp, _vp, _fp, _i, _i, _i, _i, _f, _sp, _vp]
_lib.attn_fwd_strided.restype = _i
_lib.attn_bwd_strided.argtypes = [_vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _sp, _vp, _sz, _vp]
_lib.attn_bwd_strided.restype = _i
class attn_options(ctypes.Structure):
    """Options of the _ex entry points (include/attn.h): the mask and
    attention dropout."""
    _fields_ = [("causal", ctypes.c_int32), ("dropout_p", ctypes.c_float),
                ("dropout_seed", ctypes.c_uint64), ("dropout_offset", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32), ("dropout_mask", ctypes.c_void_p),
                ("dropout_mask_bytes", ctypes.c_size_t)]


_op = ctypes.POINTER(attn_options)
_lib.attn_fwd_ex.argtypes = [_vp, _vp, _vp, _vp, _fp, _i, _i, _i, _i, _f, _sp, _op, _vp]
_lib.attn_fwd_ex.restype = _i
_lib.attn_bwd_ex.argtypes = [_vp, _vp, _vp, _vp, _fp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _sp, _op,
                             _vp, _sz, _vp]
_lib.attn_bwd_ex.restype = _i
_lib.attn_fwd_f32_ex.argtypes = [_fp, _fp, _fp, _fp, _fp, _i, _i, _i, _i, _f, _op, _vp]
_lib.attn_fwd_f32_ex.restype = _i
_lib.attn_bwd_f32_ex.argtypes = [_fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _i, _i, _i, _i, _f, _op,
                                 _vp, _sz, _vp]
_lib.attn_bwd_f32_ex.restype = _i
_lib.attn_decode.argtypes = [_vp, _vp, _vp, _vp, _fp, _i, _i, _i, _i, _i, _f, _sp, _vp]
_lib.attn_decode.restype = _i
DECODE_MAX_QUERIES = 16
_lib.attn_fwd_f32.argtypes = [_fp, _fp, _fp, _fp, _fp, _i, _i, _i, _i, _f, _vp]
_lib.attn_fwd_f32.restype = _i
_lib.attn_bwd_f32_workspace_bytes.argtypes = [_i, _i, _i, _i]
_lib.attn_bwd_f32_workspace_bytes.restype = _sz
_lib.attn_bwd_f32.argtypes = [_fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _i, _i, _i, _i, _f, _vp, _sz, _vp]
_lib.attn_bwd_f32.restype = _i
_lib.attn_dropout_mask_bytes.argtypes = [_i, _i, _i]
_lib.attn_dropout_mask_bytes.restype = _sz
_lib.attn_device_error.argtypes = [_vp]
_lib.attn_device_error.restype = _i
_lib.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint32, _vp]
_lib.attn_selftest_wait_timeout.restype = _i
_lib.attn_selftest_device_check.argtypes = [_vp]
_lib.attn_selftest_device_check.restype = _i
_lib.attn_profile_next_call.argtypes = [_vp, _vp]
_lib.attn_profile_next_call.restype = _i

EXPORTED = ("attn_status_string", "attn_version", "attn_last_launch_count", "attn_fwd",
            "attn_bwd_workspace_bytes", "attn_bwd", "attn_fwd_f32", "attn_bwd_f32_workspace_bytes",
            "attn_bwd_f32", "attn_device_error", "attn_profile_next_call",
            "attn_selftest_wait_timeout", "attn_selftest_device_check", "attn_bwd_noalloc", "attn_fwd_strided",
            "attn_bwd_strided", "attn_fwd_ex", "attn_bwd_ex", "attn_fwd_f32_ex", "attn_bwd_f32_ex",
            "attn_decode", "attn_dropout_mask_bytes")


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {attn_status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The raw ctypes handle of libattn.so."""
    return _lib


def attn_status_string(status: int) -> str:
    return _lib.attn_status_string(int(status)).decode()


def attn_version() -> int:
    return int(_lib.attn_version())


def attn_last_launch_count() -> int:
    """Kernels enqueued by the most recent successful call on this thread."""
    return int(_lib.attn_last_launch_count())


def _torch():
    import torch
    return torch


def _stream_handle(stream) -> int:
    """The raw handle of `stream`, or of torch's current stream on the current
    device (read without building a Stream object when torch offers that)."""
    torch = _torch()
    if stream is None:
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:
            return int(raw(torch.cuda.current_device()))
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


class _device:
    """Makes `device` current for the call, switching only when it is not
    (a plain torch.cuda.device() switches and restores every time)."""
    __slots__ = ("idx", "prev")

    def __init__(self, device):
        self.idx = device.index

    def __enter__(self):
        torch = _torch()
        cur = torch.cuda.current_device()
        self.prev = None if cur == self.idx else cur
        if self.prev is not None:
            torch.cuda.set_device(self.idx)
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            _torch().cuda.set_device(self.prev)
        return False


def _check(t, name, dtype, shape=None):
    """The tensor's device address, after checking that it is a contiguous
    CUDA tensor of `dtype` (and `shape`); one combined test on the common
    path, the specific error otherwise."""
    try:
        if t.is_cuda and t.dtype == dtype and (shape is None or t.shape == shape) and t.is_contiguous():
            return t.data_ptr()
    except AttributeError:
        pass
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _shape4(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, T, D]")
    B, H, T, D = q.shape
    return B, H, T, D


def _raise(status: int, where: str):
    if status != 0:
        raise AttnError(status, where)


def _fwd(cfn, dtype, q, k, v, o, lse, scale, stream):
    torch = _torch()
    B, H, T, D = _shape4(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    ptrs = [_check(q, "q", dtype), _check(k, "k", dtype, q.shape), _check(v, "v", dtype, q.shape),
            _check(o, "o", dtype, q.shape), _check(lse, "lse", torch.float32, (B, H, T))]
    with _device(q.device):
        _raise(cfn(*ptrs, B, H, T, D, scale, _stream_handle(stream)), cfn.__name__)
    return o, lse


def _bwd(cfn, ws_fn, dtype, q, k, v, o, lse, dO, dq, dk, dv, scale, workspace, stream):
    torch = _torch()
    B, H, T, D = _shape4(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    need = int(ws_fn(B, H, T, D))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ptrs = [_check(q, "q", dtype), _check(k, "k", dtype, q.shape), _check(v, "v", dtype, q.shape),
            _check(o, "o", dtype, q.shape), _check(lse, "lse", torch.float32, (B, H, T)),
            _check(dO, "dO", dtype, q.shape), _check(dq, "dq", dtype, q.shape),
            _check(dk, "dk", dtype, q.shape), _check(dv, "dv", dtype, q.shape)]
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    with _device(q.device):
        _raise(cfn(*ptrs, B, H, T, D, scale, workspace.data_ptr(), ws_bytes, _stream_handle(stream)),
               cfn.__name__)
    return dq, dk, dv


def attn_fwd(q, k, v, o=None, lse=None, scale: Optional[float] = None, stream=None):
    """bf16 forward on the tensor cores: returns (O bf16, lse float32 [B,H,T])."""
    return _fwd(_lib.attn_fwd, _torch().bfloat16, q, k, v, o, lse, scale, stream)


def attn_bwd_workspace_bytes(B: int, H: int, T: int, D: int) -> int:
    return int(_lib.attn_bwd_workspace_bytes(B, H, T, D))


def attn_bwd(q, k, v, o, lse, dO, dq=None, dk=None, dv=None, scale: Optional[float] = None,
             workspace=None, stream=None):
    """bf16 backward: returns (dQ, dK, dV) bf16."""
    return _bwd(_lib.attn_bwd, _lib.attn_bwd_workspace_bytes, _torch().bfloat16, q, k, v, o, lse,
                dO, dq, dk, dv, scale, workspace, stream)


def attn_bwd_noalloc(q, k, v, o, lse, dO, dq=None, dk=None, dv=None,
                     scale: Optional[float] = None, stream=None):
    """bf16 backward whose scratch is a fixed array inside the library (for
    callers that cannot allocate device memory; see include/attn.h for the
    size limit and the sharing rules).  Returns (dQ, dK, dV)."""
    torch = _torch()
    B, H, T, D = _shape4(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    bf = torch.bfloat16
    ptrs = [_check(q, "q", bf), _check(k, "k", bf, q.shape), _check(v, "v", bf, q.shape),
            _check(o, "o", bf, q.shape), _check(lse, "lse", torch.float32, (B, H, T)),
            _check(dO, "dO", bf, q.shape), _check(dq, "dq", bf, q.shape),
            _check(dk, "dk", bf, q.shape), _check(dv, "dv", bf, q.shape)]
    with _device(q.device):
        _raise(_lib.attn_bwd_noalloc(*ptrs, B, H, T, D, scale, _stream_handle(stream)),
               "attn_bwd_noalloc")
    return dq, dk, dv


def attn_fwd_f32(q, k, v, o=None, lse=None, scale: Optional[float] = None, stream=None):
    """float32 forward on CUDA cores: returns (O, lse)."""
    return _fwd(_lib.attn_fwd_f32, _torch().float32, q, k, v, o, lse, scale, stream)


def attn_bwd_f32_workspace_bytes(B: int, H: int, T: int, D: int) -> int:
    return int(_lib.attn_bwd_f32_workspace_bytes(B, H, T, D))


def attn_bwd_f32(q, k, v, o, lse, dO, dq=None, dk=None, dv=None, scale: Optional[float] = None,
                 workspace=None, stream=None):
    """float32 backward: returns (dQ, dK, dV)."""
    return _bwd(_lib.attn_bwd_f32, _lib.attn_bwd_f32_workspace_bytes, _torch().float32, q, k, v, o,
                lse, dO, dq, dk, dv, scale, workspace, stream)


def attn_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the in-kernel error flag
    status: 0, or the timeout status if a bounded wait ran out."""
    return int(_lib.attn_device_error(_stream_handle(stream)))


def attn_profile_next_call(start=None, end=None) -> None:
    """Arm the next attn_fwd/attn_bwd call on this thread to record the two
    torch.cuda.Event objects around its main kernel, on the call's stream."""
    def h(ev):
        if ev is None:
            return None
        handle = int(ev.cuda_event)
        if handle == 0:
            raise ValueError("the torch.cuda.Event has no CUDA event yet: record it once first")
        return handle
    _raise(_lib.attn_profile_next_call(h(start), h(end)), "attn_profile_next_call")


def attn_selftest_wait_timeout(polls: int = 1024, stream=None) -> None:
    """Enqueue the bounded-wait failure self test (see include/attn.h)."""
    _raise(_lib.attn_selftest_wait_timeout(int(polls), _stream_handle(stream)),
           "attn_selftest_wait_timeout")


def _check_view(t, name, shape):
    """A bf16 CUDA [B, H, T, D] view with unit D stride; returns its pointer."""
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.stride(3) != 1:
        raise ValueError(f"{name} must have unit stride along D")
    return t.data_ptr()


def _strides_of(*tensors):
    arr = (attn_strides * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = attn_strides(t.stride(0), t.stride(1), t.stride(2))
    return arr


def empty_token_major(B: int, H: int, T: int, D: int, device):
    """A bf16 [B, H, T, D] view of a fresh [B, T, H*D] tensor (the layout the
    output projection consumes)."""
    torch = _torch()
    return torch.empty(B, T, H, D, dtype=torch.bfloat16, device=device).permute(0, 2, 1, 3)


def attn_fwd_strided(q, k, v, o=None, lse=None, scale: Optional[float] = None, stream=None):
    """Forward on strided [B, H, T, D] views (e.g. slices of the c_attn output
    [B, T, 3C]).  O defaults to a [B, T, C] buffer viewed as [B, H, T, D]."""
    torch = _torch()
    B, H, T, D = _shape4(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = empty_token_major(B, H, T, D, q.device) if o is None else o
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device) if lse is None else lse
    ptrs = [_check_view(q, "q", q.shape), _check_view(k, "k", q.shape),
            _check_view(v, "v", q.shape), _check_view(o, "o", q.shape),
            _check(lse, "lse", torch.float32, (B, H, T))]
    st = _strides_of(q, k, v, o)
    with _device(q.device):
        _raise(_lib.attn_fwd_strided(*ptrs, B, H, T, D, scale, st, _stream_handle(stream)),
               "attn_fwd_strided")
    return o, lse


def attn_bwd_strided(q, k, v, o, lse, dO, dq=None, dk=None, dv=None, scale: Optional[float] = None,
                     workspace=None, stream=None):
    """Backward on strided views; dq/dk/dv default to [B, T, C] buffers viewed
    as [B, H, T, D].  Returns (dQ, dK, dV)."""
    torch = _torch()
    B, H, T, D = _shape4(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq = empty_token_major(B, H, T, D, q.device) if dq is None else dq
    dk = empty_token_major(B, H, T, D, q.device) if dk is None else dk
    dv = empty_token_major(B, H, T, D, q.device) if dv is None else dv
    need = attn_bwd_workspace_bytes(B, H, T, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ptrs = [_check_view(q, "q", q.shape), _check_view(k, "k", q.shape),
            _check_view(v, "v", q.shape), _check_view(o, "o", q.shape),
            _check(lse, "lse", torch.float32, (B, H, T)), _check_view(dO, "dO", q.shape),
            _check_view(dq, "dq", q.shape), _check_view(dk, "dk", q.shape),
            _check_view(dv, "dv", q.shape)]
    st = _strides_of(q, k, v, o, dO, dq, dk, dv)
    ws_bytes = workspace.numel() * workspace.element_size()
    with _device(q.device):
        _raise(_lib.attn_bwd_strided(*ptrs, B, H, T, D, scale, st, workspace.data_ptr(), ws_bytes,
                                     _stream_handle(stream)), "attn_bwd_strided")
    return dq, dk, dv


def attn_dropout_mask_bytes(B: int, H: int, T: int) -> int:
    return int(_lib.attn_dropout_mask_bytes(B, H, T))


def _options(causal: bool, dropout_p: float = 0.0, seed: int = 0, offset: int = 0, mask=None):
    if mask is not None:
        torch = _torch()
        if mask.dtype != torch.uint8 or not mask.is_cuda or not mask.is_contiguous():
            raise ValueError("dropout_mask must be a contiguous CUDA uint8 tensor")
    return attn_options(1 if causal else 0, float(dropout_p), int(seed) & (2**64 - 1),
                        int(offset) & 0xFFFFFFFF, 0, None if mask is None else mask.data_ptr(),
                        0 if mask is None else mask.numel())


def _all_contiguous(*tensors) -> bool:
    return all(t.is_contiguous() for t in tensors)


def attn_fwd_ex(q, k, v, o=None, lse=None, scale: Optional[float] = None, causal: bool = True,
                dropout_p: float = 0.0, seed: int = 0, offset: int = 0, stream=None,
                dropout_mask=None):
    """bf16 forward with options: ``causal=False`` drops the mask (every query
    sees all T keys); ``dropout_p`` > 0 drops attention weights with the
    Philox keep mask of (seed, offset), and stores the drawn keep bits in
    ``dropout_mask`` (a uint8 tensor of attn_dropout_mask_bytes(B, H, T)
    bytes) when one is given, for attn_bwd_ex to reuse.  Contiguous or strided
    [B, H, T, D] views; O defaults to the layout of q (contiguous, else a
    [B, T, C] buffer).  Returns (O, lse)."""
    torch = _torch()
    B, H, T, D = _shape4(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q) if q.is_contiguous() else empty_token_major(B, H, T, D, q.device)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device) if lse is None else lse
    ptrs = [_check_view(q, "q", q.shape), _check_view(k, "k", q.shape),
            _check_view(v, "v", q.shape), _check_view(o, "o", q.shape),
            _check(lse, "lse", torch.float32, (B, H, T))]
    st = None if _all_contiguous(q, k, v, o) else _strides_of(q, k, v, o)
    opts = _options(causal, dropout_p, seed, offset, dropout_mask)
    with _device(q.device):
        _raise(_lib.attn_fwd_ex(*ptrs, B, H, T, D, scale, st, ctypes.byref(opts),
                                _stream_handle(stream)), "attn_fwd_ex")
    return o, lse


def attn_bwd_ex(q, k, v, o, lse, dO, dq=None, dk=None, dv=None, scale: Optional[float] = None,
                causal: bool = True, dropout_p: float = 0.0, seed: int = 0, offset: int = 0,
                workspace=None, stream=None, dropout_mask=None):
    """bf16 backward with options (the same ``causal``, ``dropout_p``, ``seed``
    and ``offset`` as given to attn_fwd_ex), on contiguous or strided views.
    ``dropout_mask``: the buffer the forward stored its keep bits in, read
    instead of drawing the mask again.  Returns (dQ, dK, dV)."""
    torch = _torch()
    B, H, T, D = _shape4(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    contig = q.is_contiguous()
    new = (lambda: torch.empty_like(q)) if contig else (lambda: empty_token_major(B, H, T, D, q.device))
    dq = new() if dq is None else dq
    dk = new() if dk is None else dk
    dv = new() if dv is None else dv
    need = attn_bwd_workspace_bytes(B, H, T, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ptrs = [_check_view(q, "q", q.shape), _check_view(k, "k", q.shape),
            _check_view(v, "v", q.shape), _check_view(o, "o", q.shape),
            _check(lse, "lse", torch.float32, (B, H, T)), _check_view(dO, "dO", q.shape),
            _check_view(dq, "dq", q.shape), _check_view(dk, "dk", q.shape),
            _check_view(dv, "dv", q.shape)]
    views = (q, k, v, o, dO, dq, dk, dv)
    st = None if _all_contiguous(*views) else _strides_of(*views)
    opts = _options(causal, dropout_p, seed, offset, dropout_mask)
    ws_bytes = workspace.numel() * workspace.element_size()
    with _device(q.device):
        _raise(_lib.attn_bwd_ex(*ptrs, B, H, T, D, scale, st, ctypes.byref(opts),
                                workspace.data_ptr(), ws_bytes, _stream_handle(stream)),
               "attn_bwd_ex")
    return dq, dk, dv


def attn_fwd_f32_ex(q, k, v, o=None, lse=None, scale: Optional[float] = None, causal: bool = True,
                    dropout_p: float = 0.0, seed: int = 0, offset: int = 0, stream=None):
    """float32 forward with options (contiguous tensors).  Returns (O, lse)."""
    opts = _options(causal, dropout_p, seed, offset)
    fn = lambda *a: _lib.attn_fwd_f32_ex(*a[:-1], ctypes.byref(opts), a[-1])
    fn.__name__ = "attn_fwd_f32_ex"
    return _fwd(fn, _torch().float32, q, k, v, o, lse, scale, stream)


def attn_bwd_f32_ex(q, k, v, o, lse, dO, dq=None, dk=None, dv=None, scale: Optional[float] = None,
                    causal: bool = True, dropout_p: float = 0.0, seed: int = 0, offset: int = 0,
                    workspace=None, stream=None):
    """float32 backward with options (contiguous tensors).  Returns (dQ, dK, dV)."""
    opts = _options(causal, dropout_p, seed, offset)
    fn = lambda *a: _lib.attn_bwd_f32_ex(*a[:-3], ctypes.byref(opts), *a[-3:])
    fn.__name__ = "attn_bwd_f32_ex"
    return _bwd(fn, _lib.attn_bwd_f32_workspace_bytes, _torch().float32, q, k, v, o, lse, dO, dq,
                dk, dv, scale, workspace, stream)


def attn_decode(q, k, v, o=None, lse=None, scale: Optional[float] = None, stream=None):
    """Decode attention: q [B, H, Tq, D] holds the Tq newest tokens' queries
    (Tq <= 16), k and v [B, H, Tk, D] the kept keys and values of all Tk
    tokens (views into a larger cache are fine: only the D stride must be 1).
    Query r is the token at position Tk - Tq + r.  Returns (O [B, H, Tq, D],
    lse [B, H, Tq])."""
    torch = _torch()
    B, H, Tq, D = _shape4(q)
    Tk = int(k.shape[2])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty_like(q, memory_format=torch.contiguous_format) if o is None else o
    lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device) if lse is None else lse
    ptrs = [_check_view(q, "q", (B, H, Tq, D)), _check_view(k, "k", (B, H, Tk, D)),
            _check_view(v, "v", (B, H, Tk, D)), _check_view(o, "o", (B, H, Tq, D)),
            _check(lse, "lse", torch.float32, (B, H, Tq))]
    st = None if _all_contiguous(q, k, v, o) else _strides_of(q, k, v, o)
    with _device(q.device):
        _raise(_lib.attn_decode(*ptrs, B, H, Tq, Tk, D, scale, st, _stream_handle(stream)),
               "attn_decode")
    return o, lse
