"""Back-to-back calls on one stream with no host synchronisation between them.

Each training-path kernel may begin its prologue while the previous kernel in
the stream drains (programmatic dependent launch), and waits for that kernel
before it touches global memory.  These tests enqueue chains whose later calls
overwrite buffers that earlier calls still read (the shared backward workspace,
O and lse), or read what earlier calls wrote, and check every result against
the oracle: a kernel that ran ahead of its predecessor would read zeroed or
foreign data."""
import pytest
import torch

from tests import parity
from workloads import random_qkv

pytestmark = pytest.mark.gpu


def _cpu(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("D", [32, 64, 128])
def test_chained_calls_share_workspace_and_outputs(D):
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    B, H, T = 2, 3, 300
    inps = [random_qkv(900 + 7 * n + D, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
            for n in range(3)]
    ws = torch.empty(A.attn_bwd_workspace_bytes(B, H, T, D), dtype=torch.uint8, device=dev)
    o = torch.empty(B, H, T, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, T, dtype=torch.float32, device=dev)
    dev_inps = [{n: a.to(dev) for n, a in inp.items()} for inp in inps]
    torch.cuda.synchronize()
    grads, outs = [], []
    for x in dev_inps:
        # O and lse are rewritten by the next forward while this backward's
        # prep may still be reading them; the workspace's dQ accumulator is
        # zeroed by the next backward while this one's post kernel reads it.
        A.attn_fwd(x["q"], x["k"], x["v"], o=o, lse=lse)
        grads.append(A.attn_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], workspace=ws))
        outs.append((o.clone(), lse.clone()))
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    for n, (inp, (dq, dk, dv), (on, ln)) in enumerate(zip(inps, grads, outs)):
        got = dict(o=_cpu(on), lse=_cpu(ln), dq=_cpu(dq), dk=_cpu(dk), dv=_cpu(dv))
        parity.assert_close(got, parity.run_oracle(inp), torch.bfloat16, f"chain D={D} call {n}")


def test_chained_decode_after_training_calls():
    """A decode call enqueued right after a backward that writes the keys it
    reads (dK written into the buffer then passed as K)."""
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    B, H, T, D = 2, 3, 257, 64
    inp = random_qkv(77, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
    x = {n: a.to(dev) for n, a in inp.items()}
    kbuf = torch.empty(B, H, T, D, dtype=torch.bfloat16, device=dev)
    vbuf = torch.empty_like(kbuf)
    qd = x["q"][:, :, -4:].contiguous()
    o, lse = A.attn_fwd(x["q"], x["k"], x["v"])
    # The backward writes dK, dV into kbuf, vbuf; the decode reads them at once.
    A.attn_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], dk=kbuf, dv=vbuf)
    od, lsed = A.attn_decode(qd, kbuf, vbuf)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    kk, vv = kbuf.clone(), vbuf.clone()
    ref_o, ref_lse = A.attn_decode(qd, kk, vv)
    torch.cuda.synchronize()
    assert torch.equal(od, ref_o) and torch.equal(lsed, ref_lse)
