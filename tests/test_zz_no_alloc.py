"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (C hosts without a device allocator, plug-ins whose host framework owns
all device memory and forbids cudaMalloc, latency-critical loops that cannot
afford cudaMalloc's possible device synchronisation).  Its scratch is a fixed
array inside the library instead of a caller-supplied workspace.

The GPU tests call it through the C ABI and check every result both against
the regular attn_bwd on the same inputs and against the double-precision
oracle (all heads of the small cases, a seeded sample of whole heads of the
GPT-2 layer), within the bf16 parity tolerance every other test uses (max-abs
<= 2e-2, rel-L2 <= 1e-2).  The array keeps the previous call's contents, so
one test runs a full-size call, then a ragged smaller one, then the full-size
one again: every region a call reads must have been rewritten by that call.
This file is named to be collected last, and passes alone in a fresh process
as well as after the rest of the suite."""
import numpy as np
import pytest
import torch

from tests import parity
from workloads import WORKLOADS, make_inputs, random_qkv

E_NULL, E_SCALE, E_WS = -1, -9, -7
P = 1 << 20


def _case(name):
    if name == "gpt2_124m":
        w = WORKLOADS["gpt2_124m"]
        inp = make_inputs(w, seed=3)
        return inp, parity.sample_heads(w.B, w.H, 6, seed=3)
    if name == "ragged":
        return random_qkv(17, 2, 3, 333, 32, dtype=torch.bfloat16, do_std=1e-2), None
    return random_qkv(29, 1, 4, 1000, 64, dtype=torch.bfloat16, do_std=1e-2), None


def _check_call(A, inp, heads, label):
    """attn_bwd_noalloc against attn_bwd and against the oracle on one case."""
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = A.attn_fwd(q, k, v)
    ref_gpu = [t.double().cpu().numpy() for t in A.attn_bwd(q, k, v, o, lse, do)]
    got = A.attn_bwd_noalloc(q, k, v, o, lse, do)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    got = {n: t.double().cpu().numpy() for n, t in zip(("dq", "dk", "dv"), got)}
    B, H = q.shape[0], q.shape[1]
    ref = parity.run_oracle(inp, heads=heads)
    for i, name in enumerate(("dq", "dk", "dv")):
        g = got[name]
        assert np.all(np.isfinite(g)), f"{label} {name}: non-finite"
        ma, rel = parity.errors(g, ref_gpu[i])
        assert ma <= parity.BF16_TOL["max_abs"], f"{label} {name} vs attn_bwd: max-abs {ma:.3e}"
        assert rel is None or rel <= parity.BF16_TOL["rel_l2"], f"{label} {name} vs attn_bwd: rel-L2 {rel}"
        gs = parity.select_heads({name: g}, heads, B, H)[name]
        ma, rel = parity.errors(gs, ref[name])
        assert ma <= parity.BF16_TOL["max_abs"], f"{label} {name} vs oracle: max-abs {ma:.3e}"
        assert rel is None or rel <= parity.BF16_TOL["rel_l2"], f"{label} {name} vs oracle: rel-L2 {rel}"


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["gpt2_124m", "ragged"])
def test_noalloc_matches_attn_bwd_and_oracle_on_two_calls(case):
    import decoder_only_transformer_sdpa_b200 as A
    torch.cuda.set_device(0)
    inp, heads = _case(case)
    for call in range(2):
        _check_call(A, inp, heads, f"{case} call {call}")


@pytest.mark.gpu
def test_noalloc_large_then_ragged_then_large():
    """The shared array holds the previous call's dQ accumulator, lse and
    Delta: a smaller ragged call after a full-size one, and the full-size one
    again after it, must each read only what they wrote themselves."""
    import decoder_only_transformer_sdpa_b200 as A
    torch.cuda.set_device(0)
    for name in ("gpt2_124m", "ragged", "mid", "gpt2_124m"):
        inp, heads = _case(name)
        _check_call(A, inp, heads, name)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """A shape whose scratch would exceed the built-in array is refused before
    any work is enqueued (the pointers here are never touched)."""
    import decoder_only_transformer_sdpa_b200 as A
    lib = A.lib()
    B, H, T, D = 64, 16, 4096, 64
    assert A.attn_bwd_workspace_bytes(B, H, T, D) > 64 * 1024 * 1024
    assert lib.attn_bwd_noalloc(*([P] * 9), B, H, T, D, 0.125, None) == E_WS


def test_noalloc_argument_errors_come_first():
    """The statuses and their order are attn_bwd's: a NULL pointer or a bad
    scale is reported as such even when the shape is also too large for the
    built-in scratch."""
    import decoder_only_transformer_sdpa_b200 as A
    lib = A.lib()
    B, H, T, D = 64, 16, 4096, 64
    ptrs = [P] * 9
    ptrs[3] = None
    assert lib.attn_bwd_noalloc(*ptrs, B, H, T, D, 0.125, None) == E_NULL
    assert lib.attn_bwd_noalloc(*([P] * 9), B, H, T, D, -1.0, None) == E_SCALE
