"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol include/attn.h declares, and rejects bad arguments before touching
CUDA (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import decoder_only_transformer_sdpa_b200 as lib_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")

OK, E_NULL, E_SHAPE, E_D, E_ALIGN, E_CUDA, E_TIMEOUT, E_WS, E_DEV, E_SCALE = 0, -1, -2, -3, -4, -5, -6, -7, -8, -9


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert {"attn_fwd", "attn_bwd", "attn_bwd_workspace_bytes", "attn_fwd_f32", "attn_bwd_f32",
            "attn_status_string"} <= set(names)


def test_library_exports_every_declared_symbol():
    lib = lib_mod.lib()
    for name in declared_functions():
        assert hasattr(lib, name), f"libattn.so does not export {name}"
    assert set(declared_functions()) == set(lib_mod.EXPORTED)


def test_exports_nothing_else():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", lib_mod.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    funcs = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert funcs == set(declared_functions())


def test_status_strings():
    for s in (OK, E_NULL, E_SHAPE, E_D, E_ALIGN, E_CUDA, E_TIMEOUT, E_WS, E_DEV, E_SCALE, 12345):
        assert isinstance(lib_mod.attn_status_string(s), str) and lib_mod.attn_status_string(s)
    assert lib_mod.attn_version() == 1


def test_workspace_sizes():
    B, H, T, D = 12, 12, 1024, 64
    rows = B * H * T
    rnd = lambda x: (x + 255) // 256 * 256
    tpad = lambda t: (t + 127) // 128 * 128
    assert lib_mod.attn_bwd_workspace_bytes(B, H, T, D) == rnd(rows * D * 4) + 2 * rnd(B * H * tpad(T) * 4)
    assert lib_mod.attn_bwd_workspace_bytes(1, 1, 1, 32) == 256 + 2 * 512
    assert lib_mod.attn_bwd_workspace_bytes(2, 3, 129, 64) == rnd(2 * 3 * 129 * 64 * 4) + 2 * rnd(6 * 256 * 4)
    assert lib_mod.attn_bwd_workspace_bytes(1, 1, 1, 48) == 0       # unsupported D
    assert lib_mod.attn_bwd_workspace_bytes(0, 1, 1, 64) == 0       # bad shape
    assert lib_mod.attn_bwd_f32_workspace_bytes(4, 4, 8, 8) == rnd(4 * 4 * 8 * 4)
    assert lib_mod.attn_bwd_f32_workspace_bytes(1, 1, 1, 129) == 0


# Fake but well-aligned device addresses: every call below fails validation
# before the library makes any CUDA call.
P = 1 << 20


def fwd(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, T=8, D=64, scale=0.125):
    return lib_mod.lib().attn_fwd(q, k, v, o, lse, B, H, T, D, scale, None)


def bwd(ptrs=None, B=1, H=1, T=8, D=64, scale=0.125, ws=P, ws_bytes=1 << 30):
    p = [P] * 9 if ptrs is None else ptrs
    return lib_mod.lib().attn_bwd(*p, B, H, T, D, scale, ws, ws_bytes, None)


def fwd32(q=P, o=P, B=1, H=1, T=8, D=8, scale=0.3):
    return lib_mod.lib().attn_fwd_f32(q, P, P, o, P, B, H, T, D, scale, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), E_NULL), (dict(lse=None), E_NULL),
    (dict(B=0), E_SHAPE), (dict(H=-1), E_SHAPE), (dict(T=0), E_SHAPE),
    (dict(D=48), E_D), (dict(D=256), E_D), (dict(D=0), E_D), (dict(D=16), E_D),
    (dict(scale=0.0), E_SCALE), (dict(scale=float("nan")), E_SCALE), (dict(scale=-1.0), E_SCALE),
    (dict(scale=float("inf")), E_SCALE),
    (dict(q=P + 8), E_ALIGN), (dict(o=P + 2), E_ALIGN), (dict(lse=P + 2), E_ALIGN),
    (dict(B=1 << 20, H=1 << 10, T=1 << 12), E_SHAPE),
])
def test_fwd_argument_errors(kw, expect):
    assert fwd(**kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=[P] * 8 + [None]), E_NULL),
    (dict(ptrs=[P] * 5 + [P + 8] + [P] * 3), E_ALIGN),
    (dict(D=100), E_D),
    (dict(ws=None), E_WS), (dict(ws_bytes=16), E_WS), (dict(ws=P + 16), E_WS),
    (dict(T=0), E_SHAPE), (dict(scale=float("nan")), E_SCALE),
])
def test_bwd_argument_errors(kw, expect):
    assert bwd(**kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), E_NULL), (dict(D=129), E_D), (dict(D=0), E_D), (dict(q=P + 2), E_ALIGN),
    (dict(B=0), E_SHAPE), (dict(scale=-2.0), E_SCALE),
])
def test_fwd_f32_argument_errors(kw, expect):
    assert fwd32(**kw) == expect


def test_bwd_f32_workspace_error():
    lib = lib_mod.lib()
    assert lib.attn_bwd_f32(*([P] * 9), 1, 1, 8, 8, 0.3, P, 8, None) == E_WS


def test_selftest_argument_errors():
    assert lib_mod.lib().attn_selftest_wait_timeout(0, None) == E_SHAPE
    assert lib_mod.lib().attn_selftest_wait_timeout((1 << 22) + 1, None) == E_SHAPE


def _strides(n, b=1 << 16, h=64, t=1 << 10):
    import ctypes
    arr = (lib_mod.attn_strides * n)()
    for i in range(n):
        arr[i] = lib_mod.attn_strides(b, h, t)
    return arr


@pytest.mark.parametrize("bad", [dict(t=0), dict(h=-8), dict(b=12), dict(t=3), dict(t=1 << 40)])
def test_strided_argument_errors(bad):
    lib = lib_mod.lib()
    good = _strides(8)
    assert lib.attn_fwd_strided(P, P, P, P, P, 1, 1, 8, 64, 0.125, None, None) == E_NULL
    assert lib.attn_bwd_strided(*([P] * 9), 1, 1, 8, 64, 0.125, None, P, 1 << 30, None) == E_NULL
    for i in range(4):
        st = _strides(4)
        st[i] = lib_mod.attn_strides(**{**dict(b=1 << 16, h=64, t=1 << 10), **bad})
        assert lib.attn_fwd_strided(P, P, P, P, P, 1, 1, 8, 64, 0.125, st, None) == E_ALIGN
    for i in range(8):
        st = _strides(8)
        st[i] = lib_mod.attn_strides(**{**dict(b=1 << 16, h=64, t=1 << 10), **bad})
        assert lib.attn_bwd_strided(*([P] * 9), 1, 1, 8, 64, 0.125, st, P, 1 << 30, None) == E_ALIGN
    # valid strides still hit the ordinary checks first-class (unsupported D)
    assert lib.attn_fwd_strided(P, P, P, P, P, 1, 1, 8, 48, 0.125, good, None) == E_D


def _opts(causal):
    return ctypes.byref(lib_mod.attn_options(causal))


@pytest.mark.parametrize("causal", [2, -1, 7])
def test_options_reject_unknown_mask(causal):
    lib = lib_mod.lib()
    E_OPTION = -10
    assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, 0.125, None, _opts(causal), None) == E_OPTION
    assert lib.attn_bwd_ex(*([P] * 9), 1, 1, 8, 64, 0.125, None, _opts(causal), P, 1 << 30,
                           None) == E_OPTION
    assert lib.attn_fwd_f32_ex(P, P, P, P, P, 1, 1, 8, 8, 0.35, _opts(causal), None) == E_OPTION
    assert lib.attn_bwd_f32_ex(*([P] * 9), 1, 1, 8, 8, 0.35, _opts(causal), P, 1 << 30,
                               None) == E_OPTION
    assert lib_mod.attn_status_string(E_OPTION) != lib_mod.attn_status_string(12345)


@pytest.mark.parametrize("causal", [0, 1])
def test_options_pass_to_the_ordinary_checks(causal):
    """Valid options (and NULL options or strides) reach the same argument
    checks as the plain entry points, before anything touches CUDA."""
    lib = lib_mod.lib()
    for o in (_opts(causal), None):
        assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 48, 0.125, None, o, None) == E_D
        assert lib.attn_fwd_ex(None, P, P, P, P, 1, 1, 8, 64, 0.125, None, o, None) == E_NULL
        assert lib.attn_fwd_ex(P, P, P, P, P, 0, 1, 8, 64, 0.125, None, o, None) == E_SHAPE
        assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, float("nan"), None, o, None) == E_SCALE
        assert lib.attn_bwd_ex(*([P] * 9), 1, 1, 8, 64, 0.125, None, o, None, 0, None) == E_WS
        assert lib.attn_fwd_f32_ex(P, P, P, P, P, 1, 1, 8, 129, 0.1, o, None) == E_D
        bad = _strides(8, t=3)
        assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, 0.125, bad, o, None) == E_ALIGN
        assert lib.attn_bwd_ex(*([P] * 9), 1, 1, 8, 64, 0.125, bad, o, P, 1 << 30, None) == E_ALIGN


@pytest.mark.parametrize("p", [-0.1, 1.0, 1.5, float("nan"), float("inf"), 0.999995])
def test_options_reject_bad_dropout(p):
    lib = lib_mod.lib()
    E_OPTION = -10
    o = ctypes.byref(lib_mod.attn_options(1, p, 7, 0, 0))
    assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, 0.125, None, o, None) == E_OPTION
    assert lib.attn_bwd_ex(*([P] * 9), 1, 1, 8, 64, 0.125, None, o, P, 1 << 30, None) == E_OPTION
    assert lib.attn_fwd_f32_ex(P, P, P, P, P, 1, 1, 8, 8, 0.35, o, None) == E_OPTION


def test_options_reserved_must_be_zero():
    lib = lib_mod.lib()
    o = ctypes.byref(lib_mod.attn_options(1, 0.1, 7, 0, 1))
    assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, 0.125, None, o, None) == -10


def test_options_struct_layout():
    """The ctypes mirror of attn_options matches the C layout: int32, float,
    uint64 (8-aligned), uint32, uint32, pointer, size_t = 40 bytes."""
    assert ctypes.sizeof(lib_mod.attn_options) == 40
    assert lib_mod.attn_options.dropout_seed.offset == 8
    assert lib_mod.attn_options.dropout_offset.offset == 16
    assert lib_mod.attn_options.dropout_mask.offset == 24
    assert lib_mod.attn_options.dropout_mask_bytes.offset == 32


@pytest.mark.parametrize("p", [0.0, 1e-6, 0.1, 0.99999])
def test_valid_dropout_reaches_ordinary_checks(p):
    lib = lib_mod.lib()
    o = ctypes.byref(lib_mod.attn_options(0, p, 1 << 40, 3, 0))
    assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 48, 0.125, None, o, None) == E_D
    assert lib.attn_bwd_ex(*([P] * 9), 1, 1, 8, 64, 0.125, None, o, None, 0, None) == E_WS


@pytest.mark.parametrize("B,H,Tq,Tk,D,expect", [
    (1, 1, 0, 8, 64, E_SHAPE), (1, 1, 17, 64, 64, E_SHAPE), (1, 1, 9, 8, 64, E_SHAPE),
    (0, 1, 1, 8, 64, E_SHAPE), (1, 1, 1, 0, 64, E_SHAPE), (1, 1, 1, 8, 48, E_D),
    (1, 1, 1, 8, 128, E_D)])
def test_decode_argument_errors(B, H, Tq, Tk, D, expect):
    lib = lib_mod.lib()
    assert lib.attn_decode(P, P, P, P, P, B, H, Tq, Tk, D, 0.125, None, None) == expect


def test_decode_pointer_and_stride_errors():
    lib = lib_mod.lib()
    assert lib.attn_decode(None, P, P, P, P, 1, 1, 1, 8, 64, 0.125, None, None) == E_NULL
    assert lib.attn_decode(P + 2, P, P, P, P, 1, 1, 1, 8, 64, 0.125, None, None) == E_ALIGN
    assert lib.attn_decode(P, P, P, P, P, 1, 1, 1, 8, 64, -1.0, None, None) == E_SCALE
    bad = _strides(4, t=12)
    assert lib.attn_decode(P, P, P, P, P, 1, 1, 1, 8, 64, 0.125, bad, None) == E_ALIGN


def test_dropout_mask_bytes_and_rejection():
    """The kept-mask size is (B*H) * Tp/8 * Tp bytes with Tp = T rounded up to
    128; a buffer below it is rejected before any device work."""
    assert lib_mod.attn_dropout_mask_bytes(1, 1, 1) == 16 * 128
    assert lib_mod.attn_dropout_mask_bytes(2, 3, 129) == 6 * 32 * 256
    assert lib_mod.attn_dropout_mask_bytes(12, 12, 1024) == 144 * 128 * 1024
    assert lib_mod.attn_dropout_mask_bytes(0, 1, 8) == 0
    lib = lib_mod.lib()
    E_OPTION = -10
    small = ctypes.byref(lib_mod.attn_options(1, 0.1, 7, 0, 0, P, 16 * 128 - 1))
    assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 1, 64, 0.125, None, small, None) == E_OPTION
    assert lib.attn_bwd_ex(*([P] * 9), 1, 1, 1, 64, 0.125, None, small, P, 1 << 30, None) == E_OPTION
    odd = ctypes.byref(lib_mod.attn_options(1, 0.1, 7, 0, 0, P + 8, 1 << 20))
    assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 1, 64, 0.125, None, odd, None) == E_ALIGN
    # without dropout the mask fields are ignored: the ordinary checks decide
    off = ctypes.byref(lib_mod.attn_options(1, 0.0, 7, 0, 0, P, 1))
    assert lib.attn_fwd_ex(P, P, P, P, P, 1, 1, 1, 48, 0.125, None, off, None) == E_D


def test_debug_library_exports_the_same_abi():
    """build() also makes libattn_debug.so (the kernels with the device-side
    bounds checks); it exports exactly the release library's symbols, and its
    failed-check status has its own message."""
    import subprocess
    dbg = os.path.join(os.path.dirname(lib_mod.LIB_PATH), "libattn_debug.so")
    assert os.path.exists(dbg), "libattn_debug.so is not built (build.py --debug)"
    names = lambda p: {ln.split()[-1] for ln in subprocess.run(
        ["nm", "-D", "--defined-only", p], capture_output=True, text=True, check=True).stdout.splitlines()
        if ln.split()[-1].startswith("attn_")}
    assert names(dbg) == names(lib_mod.LIB_PATH)
    E_CHECK = -11
    assert "bounds check" in lib_mod.attn_status_string(E_CHECK)
