"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (C hosts without a device allocator, plug-ins whose host framework owns
all device memory and forbids cudaMalloc, latency-critical loops that cannot
afford cudaMalloc's possible device synchronisation).  Its scratch is a fixed
array inside the library instead of a caller-supplied workspace.

The GPU test calls it through the C ABI twice in a row and checks each result
against the regular attn_bwd on the same inputs, within the bf16 parity
tolerance every other test uses (max-abs <= 2e-2, rel-L2 <= 1e-2).  This file
is named to be collected last, and passes alone in a fresh process as well as
after the rest of the suite (the array keeps the previous call's contents, and
each call must clear what it needs cleared)."""
import numpy as np
import pytest
import torch

from tests import parity
from workloads import WORKLOADS, make_inputs, random_qkv

E_WS = -7
P = 1 << 20


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["gpt2_124m", "ragged"])
def test_noalloc_matches_attn_bwd_on_two_calls(case):
    import decoder_only_transformer_sdpa_b200 as A
    torch.cuda.set_device(0)
    if case == "gpt2_124m":
        inp = make_inputs(WORKLOADS["gpt2_124m"], seed=3)
    else:
        inp = random_qkv(17, 2, 3, 333, 32, dtype=torch.bfloat16, do_std=1e-2)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = A.attn_fwd(q, k, v)
    ref = [t.double().cpu().numpy() for t in A.attn_bwd(q, k, v, o, lse, do)]
    for call in range(2):
        got = A.attn_bwd_noalloc(q, k, v, o, lse, do)
        torch.cuda.synchronize()
        assert A.attn_device_error() == 0
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            g = g.double().cpu().numpy()
            assert np.all(np.isfinite(g))
            ma, rel = parity.errors(g, r)
            assert ma <= parity.BF16_TOL["max_abs"], f"call {call} {name}: max-abs {ma:.3e}"
            assert rel is None or rel <= parity.BF16_TOL["rel_l2"], f"call {call} {name}: rel-L2 {rel}"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """A shape whose scratch would exceed the built-in array is refused before
    any work is enqueued (the pointers here are never touched)."""
    import decoder_only_transformer_sdpa_b200 as A
    lib = A.lib()
    B, H, T, D = 64, 16, 4096, 64
    assert A.attn_bwd_workspace_bytes(B, H, T, D) > 64 * 1024 * 1024
    assert lib.attn_bwd_noalloc(*([P] * 9), B, H, T, D, 0.125, None) == E_WS
