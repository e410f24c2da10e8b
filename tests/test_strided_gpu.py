"""GPU parity of the strided entry points: q, k, v read as slices of the c_attn
output [B, T, 3C], O written as [B, T, C], dO read as [B, T, C] and dq, dk, dv
written into one [B, T, 3C] buffer ("nanoGPT — 架构与原理", section 7 code
map: CausalSelfAttention splits the c_attn projection and feeds c_proj)."""
import numpy as np
import pytest
import torch

from tests import parity
from workloads import WORKLOADS, make_inputs_packed, packed_views, random_qkv

pytestmark = pytest.mark.gpu


def _run_packed(qkv, do_packed, H):
    """Forward + backward on packed layouts; returns float64 [B,H,T,D] arrays."""
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    qkv, do_packed = qkv.to(dev), do_packed.to(dev)
    B, T, C3 = qkv.shape
    D = C3 // 3 // H
    q, k, v = packed_views(qkv, H)
    do = do_packed.view(B, T, H, D).permute(0, 2, 1, 3)
    o, lse = A.attn_fwd_strided(q, k, v)
    dqkv = torch.full_like(qkv, float("nan"))
    dq, dk, dv = packed_views(dqkv, H)
    A.attn_bwd_strided(q, k, v, o, lse, do, dq, dk, dv)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    assert o.stride() == (T * H * D, D, H * D, 1)        # written token-major
    cpu = lambda t: t.detach().to("cpu", torch.float64).contiguous().numpy()
    return dict(o=cpu(o), lse=cpu(lse), dq=cpu(dq), dk=cpu(dk), dv=cpu(dv)), dqkv


@pytest.mark.parametrize("name", ["char_gpt", "gpt2_124m"])
def test_packed_layout_against_oracle(name):
    w = WORKLOADS[name]
    inp = make_inputs_packed(w, seed=5)
    got, dqkv = _run_packed(inp["qkv"], inp["do_packed"], w.H)
    assert torch.isfinite(dqkv.float()).all(), "every slot of the dq|dk|dv buffer is written"
    heads = None if name == "char_gpt" else parity.sample_heads(w.B, w.H, 6, seed=5)
    ref = parity.run_oracle(inp, heads=heads)
    parity.assert_close(parity.select_heads(got, heads, w.B, w.H), ref, torch.bfloat16,
                        f"{name} packed")


@pytest.mark.parametrize("T,D", [(333, 32), (129, 64), (1, 64)])
def test_packed_ragged_against_oracle(T, D):
    B, H = 2, 3
    inp = random_qkv(31 + T, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
    tm = lambda t: t.permute(0, 2, 1, 3).reshape(B, T, H * D)
    qkv = torch.cat([tm(inp["q"]), tm(inp["k"]), tm(inp["v"])], dim=2).contiguous()
    got, _ = _run_packed(qkv, tm(inp["do"]).contiguous(), H)
    parity.assert_close(got, parity.run_oracle(inp), torch.bfloat16, f"packed T={T} D={D}")


def test_strided_equals_contiguous():
    """The strided path runs the same kernels: identical O, lse, dK, dV; dQ
    equal up to the order of its float32 reduce-adds."""
    import decoder_only_transformer_sdpa_b200 as A
    w = WORKLOADS["char_gpt"]
    inp = make_inputs_packed(w, seed=9)
    got, _ = _run_packed(inp["qkv"], inp["do_packed"], w.H)
    dev = torch.device("cuda", 0)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = A.attn_fwd(q, k, v)
    dq, dk, dv = A.attn_bwd(q, k, v, o, lse, do)
    torch.cuda.synchronize()
    cpu = lambda t: t.detach().to("cpu", torch.float64).numpy()
    for n, t in (("o", o), ("lse", lse), ("dk", dk), ("dv", dv)):
        assert np.array_equal(got[n], cpu(t)), f"{n} differs between strided and contiguous"
    np.testing.assert_allclose(got["dq"], cpu(dq), rtol=0, atol=1e-4)


def test_packed_outputs_stay_in_their_slices():
    """Writing O into a [B, T, C] buffer and dq|dk|dv into [B, T, 3C] touches
    exactly those elements: NaN guard rows before and after stay NaN."""
    import decoder_only_transformer_sdpa_b200 as A
    B, H, T, D = 2, 2, 200, 64
    inp = random_qkv(77, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
    dev = torch.device("cuda", 0)
    tm = lambda t: t.permute(0, 2, 1, 3).reshape(B, T, H * D)
    qkv = torch.cat([tm(inp["q"]), tm(inp["k"]), tm(inp["v"])], dim=2).contiguous().to(dev)
    q, k, v = packed_views(qkv, H)
    pad = 512
    obuf = torch.full((B * T * H * D + 2 * pad,), float("nan"), dtype=torch.bfloat16, device=dev)
    o = obuf[pad:pad + B * T * H * D].view(B, T, H, D).permute(0, 2, 1, 3)
    o, lse = A.attn_fwd_strided(q, k, v, o=o)
    torch.cuda.synchronize()
    assert torch.isnan(obuf[:pad].float()).all() and torch.isnan(obuf[-pad:].float()).all()
    assert torch.isfinite(o.float()).all()
