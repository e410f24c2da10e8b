"""The debug build of the library (libattn_debug.so: the kernels with their
device-side bounds checks on tile coordinates, TMEM columns and shared-memory
offsets) raises no check on the parity shapes, and computes what the release
build computes: the checks only read."""
import importlib.util
import os

import pytest
import torch

from tests import parity
from workloads import random_qkv

pytestmark = pytest.mark.gpu

PKG = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "decoder_only_transformer_sdpa_b200")


def _load(lib_name):
    """A separate instance of the binding bound to the named library."""
    old = os.environ.get("ATTN_LIBRARY")
    os.environ["ATTN_LIBRARY"] = os.path.join(PKG, lib_name)
    try:
        spec = importlib.util.spec_from_file_location("attn_" + lib_name.replace(".", "_"),
                                                      os.path.join(PKG, "__init__.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        if old is None:
            del os.environ["ATTN_LIBRARY"]
        else:
            os.environ["ATTN_LIBRARY"] = old
    return mod


def _run(A, inp, causal, drop):
    dev = torch.device("cuda", 0)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    B, H, T, D = q.shape
    mask = torch.zeros(A.attn_dropout_mask_bytes(B, H, T), dtype=torch.uint8, device=dev) if drop else None
    kw = dict(causal=causal, dropout_p=0.1 if drop else 0.0, seed=3, offset=1, dropout_mask=mask)
    o, lse = A.attn_fwd_ex(q, k, v, **kw)
    dq, dk, dv = A.attn_bwd_ex(q, k, v, o, lse, do, **kw)
    status = A._lib.attn_device_error(None)
    return status, dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


@pytest.mark.parametrize("D,T", [(64, 1024), (64, 333), (32, 200), (128, 300), (64, 1)])
@pytest.mark.parametrize("causal,drop", [(True, False), (False, False), (True, True)])
def test_debug_build_is_clean_and_identical(D, T, causal, drop):
    rel, dbg = _load("libattn.so"), _load("libattn_debug.so")
    inp = random_qkv(1000 + T + D, 2, 3, T, D, dtype=torch.bfloat16, do_std=1e-2)
    s1, r1 = _run(rel, inp, causal, drop)
    s2, r2 = _run(dbg, inp, causal, drop)
    assert s1 == 0 and s2 == 0, (s1, s2)  # -11: a device-side bounds check failed
    for n in ("o", "lse", "dk", "dv"):
        assert torch.equal(r1[n], r2[n]), n
    assert torch.allclose(r1["dq"].float(), r2["dq"].float(), rtol=1e-2, atol=1e-6)
    if not drop:
        cpu = lambda t: t.detach().to("cpu", torch.float64).numpy()
        parity.assert_close({n: cpu(t) for n, t in r2.items()}, parity.run_oracle(inp, causal=causal),
                            torch.bfloat16, f"debug build D={D} T={T} causal={causal}")


def test_debug_build_decode_is_clean():
    dbg = _load("libattn_debug.so")
    from workloads import WORKLOADS, make_decode_inputs
    w = WORKLOADS["gpt2_124m"]
    di = make_decode_inputs(w, 3, seed=5, layer=0)
    dev = torch.device("cuda", 0)
    q, k, v = (di[n].to(dev) for n in ("q", "k", "v"))
    dbg.attn_decode(q, k, v)
    assert dbg._lib.attn_device_error(None) == 0


def test_failed_check_is_reported():
    """One check that cannot hold is recorded by the debug build and read back
    as ATTN_ERR_DEVICE_CHECK (the release build compiles it away)."""
    dbg, rel = _load("libattn_debug.so"), _load("libattn.so")
    assert dbg._lib.attn_selftest_device_check(None) == 0
    assert dbg._lib.attn_device_error(None) == -11
    assert dbg._lib.attn_device_error(None) == 0  # read and cleared
    assert rel._lib.attn_selftest_device_check(None) == 0
    assert rel._lib.attn_device_error(None) == 0
