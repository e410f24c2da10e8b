"""The C ABI inside a captured CUDA graph.

A forward + backward (and a decode call) are captured once into a graph
on static buffers, then the graph is replayed on two different inputs copied
into those buffers.  Each replay must match the oracle: the launches keep no
host-side state that a replay would reuse wrongly, allocate nothing at run
time, and their programmatic dependent launches become graph edges that still
order every kernel after the one before it."""
import numpy as np
import pytest
import torch

from tests import parity
from workloads import random_qkv

pytestmark = pytest.mark.gpu


def _cpu(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("D", [64, 128])
def test_training_step_replayed_from_a_graph(D):
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    B, H, T = 2, 3, 300
    inps = [random_qkv(700 + 11 * n + D, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2) for n in range(2)]
    st = {n: a.to(dev) for n, a in inps[0].items()}
    # One eager call first: the library's one-time set-up (kernel attributes,
    # the launch-configuration check) happens outside the capture.
    o, lse = A.attn_fwd(st["q"], st["k"], st["v"])
    A.attn_bwd(st["q"], st["k"], st["v"], o, lse, st["do"])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        o, lse = A.attn_fwd(st["q"], st["k"], st["v"])
        dq, dk, dv = A.attn_bwd(st["q"], st["k"], st["v"], o, lse, st["do"])
    for n, inp in enumerate(inps):
        for name in ("q", "k", "v", "do"):
            st[name].copy_(inp[name].to(dev))
        g.replay()
        torch.cuda.synchronize()
        assert A.attn_device_error() == 0
        got = dict(o=_cpu(o), lse=_cpu(lse), dq=_cpu(dq), dk=_cpu(dk), dv=_cpu(dv))
        parity.assert_close(got, parity.run_oracle(inp), torch.bfloat16, f"graph D={D} replay {n}")
    del g


def test_decode_replayed_from_a_graph():
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    B, H, Tk, Tq, D = 2, 3, 333, 2, 64
    inps = [random_qkv(900 + n, B, H, Tk, D, dtype=torch.bfloat16) for n in range(2)]
    q = torch.empty(B, H, Tq, D, dtype=torch.bfloat16, device=dev)
    k = torch.empty(B, H, Tk, D, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    q.copy_(inps[0]["q"][:, :, -Tq:].to(dev))
    k.copy_(inps[0]["k"].to(dev))
    v.copy_(inps[0]["v"].to(dev))
    ref_eager = [None, None]
    A.attn_decode(q, k, v)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        o, lse = A.attn_decode(q, k, v)
    for n, inp in enumerate(inps):
        q.copy_(inp["q"][:, :, -Tq:].to(dev))
        k.copy_(inp["k"].to(dev))
        v.copy_(inp["v"].to(dev))
        g.replay()
        torch.cuda.synchronize()
        assert A.attn_device_error() == 0
        # The same call made eagerly on the same bytes gives the same bits.
        oe, lsee = A.attn_decode(q, k, v)
        torch.cuda.synchronize()
        assert torch.equal(o, oe) and torch.equal(lse, lsee), f"decode replay {n}"
        ref_eager[n] = _cpu(oe)
    assert not np.array_equal(ref_eager[0], ref_eager[1])
    del g
