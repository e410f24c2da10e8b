"""Double-precision CPU oracle of causal multi-head attention (fwd + bwd), of
the same attention without the mask (``causal=False``) and of both with
dropout on the attention weights (``dropout_p``, ``seed``, ``offset``; the
keep mask is drawn by the oracle's own Philox4x32-10).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this package.  The product path (the CUDA
library and its Python binding) never imports it and shares no code with it.

The arithmetic lives in ``attn_oracle.c`` (plain loops in double, OpenMP over
heads); this module compiles it with gcc on first use and marshals numpy
float64 arrays through ctypes.  Every function takes [B, H, T, D] arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libattn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc -O2 -fopenmp, IEEE math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class OracleLib:
    """ctypes view of one compiled oracle library (the default one, or a
    variant a test builds from edited source to check that the pins bite)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        for suffix in ("", "_nc"):
            f = getattr(lib, "oracle_attn_fwd" + suffix)
            f.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, ctypes.c_double]
            f.restype = None
            f = getattr(lib, "oracle_attn_probs" + suffix)
            f.argtypes = [dp, dp, dp, i, i, i, i, ctypes.c_double]
            f.restype = None
            f = getattr(lib, "oracle_attn_bwd" + suffix)
            f.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, ctypes.c_double]
            f.restype = None
        u32, u64 = ctypes.c_uint32, ctypes.c_uint64
        lib.oracle_philox4x32_10.argtypes = [ctypes.POINTER(u32), ctypes.POINTER(u32),
                                             ctypes.POINTER(u32)]
        lib.oracle_philox4x32_10.restype = None
        lib.oracle_dropout_mask.argtypes = [i, i, i, ctypes.c_double, u64, u32,
                                            ctypes.POINTER(ctypes.c_uint8)]
        lib.oracle_dropout_mask.restype = None
        lib.oracle_attn_fwd_dropout.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, ctypes.c_double, i,
                                                ctypes.c_double, u64, u32, ctypes.c_int64]
        lib.oracle_attn_fwd_dropout.restype = None
        lib.oracle_attn_bwd_dropout.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i,
                                                ctypes.c_double, i, ctypes.c_double, u64, u32,
                                                ctypes.c_int64]
        lib.oracle_attn_bwd_dropout.restype = None
        lib.oracle_attn_decode.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, ctypes.c_double]
        lib.oracle_attn_decode.restype = None
        lib.oracle_threads.argtypes = []
        lib.oracle_threads.restype = i
        self.lib = lib

    def _fn(self, name: str, causal: bool):
        return getattr(self.lib, name if causal else name + "_nc")

    def attn_fwd(self, q, k, v, scale=None, causal=True, dropout_p=0.0, seed=0, offset=0,
                 head0=0):
        """Returns (O [B,H,T,D], lse [B,H,T]) in float64.  With dropout, head0
        is the flat head index (b*H + h) of q's first head in the full call."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, T, D = _shape(q)
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        o = np.empty_like(q)
        lse = np.empty((B, H, T), dtype=np.float64)
        if dropout_p:
            self.lib.oracle_attn_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, T, D,
                                             scale, int(bool(causal)), float(dropout_p), int(seed),
                                             int(offset), int(head0))
            return o, lse
        self._fn("oracle_attn_fwd", causal)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                            B, H, T, D, scale)
        return o, lse

    def attn_probs(self, q, k, scale=None, causal=True):
        """The softmax matrices P [B,H,T,T] (zero above the diagonal if causal)."""
        q, k = _f64(q), _f64(k)
        B, H, T, D = _shape(q)
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        p = np.empty((B, H, T, T), dtype=np.float64)
        self._fn("oracle_attn_probs", causal)(_ptr(q), _ptr(k), _ptr(p), B, H, T, D, scale)
        return p

    def attn_bwd(self, q, k, v, do, scale=None, causal=True, dropout_p=0.0, seed=0, offset=0,
                 head0=0):
        """Returns (dQ, dK, dV) in float64 for the loss sum(O * dO)."""
        q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
        B, H, T, D = _shape(q)
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        if dropout_p:
            self.lib.oracle_attn_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk),
                                             _ptr(dv), B, H, T, D, scale, int(bool(causal)),
                                             float(dropout_p), int(seed), int(offset), int(head0))
            return dq, dk, dv
        self._fn("oracle_attn_bwd", causal)(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq),
                                            _ptr(dk), _ptr(dv), B, H, T, D, scale)
        return dq, dk, dv

    def attn_decode(self, q, k, v, scale=None):
        """Decode: q [B,H,Tq,D] are the Tq newest tokens' queries, k, v
        [B,H,Tk,D] all Tk tokens' keys and values.  Returns (O [B,H,Tq,D],
        lse [B,H,Tq])."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, Tq, D = _shape(q)
        Tk = k.shape[2]
        if k.shape != (B, H, Tk, D) or v.shape != k.shape or not 1 <= Tq <= Tk:
            raise ValueError("q [B,H,Tq,D], k and v [B,H,Tk,D] with 1 <= Tq <= Tk")
        scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        o = np.empty_like(q)
        lse = np.empty((B, H, Tq), dtype=np.float64)
        self.lib.oracle_attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Tq, Tk, D,
                                    scale)
        return o, lse

    def philox4x32_10(self, ctr, key):
        """Philox4x32-10 of one 4-word counter under a 2-word key."""
        c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
        kk = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
        out = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(c, kk, out)
        return [int(x) for x in out]

    def dropout_mask(self, B, H, T, p, seed=0, offset=0):
        """The keep mask [B,H,T,T] (uint8, 1 = kept) over all (i, j)."""
        m = np.empty((B, H, T, T), dtype=np.uint8)
        self.lib.oracle_dropout_mask(B, H, T, float(p), int(seed), int(offset),
                                     m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
        return m

    def threads_used(self) -> int:
        """OpenMP threads the most recent call ran on."""
        return int(self.lib.oracle_threads())


def _load() -> OracleLib:
    global _lib
    with _lock:
        if _lib is None:
            _lib = OracleLib(build())
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor: upcast exactly on the CPU
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shape(q: np.ndarray):
    if q.ndim != 4:
        raise ValueError("expected [B, H, T, D]")
    return tuple(int(s) for s in q.shape)


def attn_fwd(q, k, v, scale=None, causal=True, dropout_p=0.0, seed=0, offset=0, head0=0):
    """Returns (O [B,H,T,D], lse [B,H,T]) in float64."""
    return _load().attn_fwd(q, k, v, scale, causal, dropout_p, seed, offset, head0)


def attn_probs(q, k, scale=None, causal=True):
    """The softmax matrices P [B,H,T,T] (zero above the diagonal if causal)."""
    return _load().attn_probs(q, k, scale, causal)


def attn_bwd(q, k, v, do, scale=None, causal=True, dropout_p=0.0, seed=0, offset=0, head0=0):
    """Returns (dQ, dK, dV) in float64 for the loss sum(O * dO)."""
    return _load().attn_bwd(q, k, v, do, scale, causal, dropout_p, seed, offset, head0)


def attn_decode(q, k, v, scale=None):
    """Decode attention of the Tq newest queries over Tk cached keys/values."""
    return _load().attn_decode(q, k, v, scale)


def philox4x32_10(ctr, key):
    """Philox4x32-10 of one counter (4 words) under one key (2 words)."""
    return _load().philox4x32_10(ctr, key)


def dropout_mask(B, H, T, p, seed=0, offset=0):
    """The dropout keep mask [B,H,T,T] (uint8, 1 = kept)."""
    return _load().dropout_mask(B, H, T, p, seed, offset)


def threads_used() -> int:
    """OpenMP threads the most recent oracle call ran on."""
    return _load().threads_used()


def source_path() -> str:
    return _SRC
