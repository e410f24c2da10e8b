"""GPU parity of decode attention (the Tq newest queries against the kept
keys and values of Tk tokens) against the oracle's decode rows, on the same
seeded inputs: O within the bf16 tolerances of tests/parity.py, lse within
1e-3."""
import numpy as np
import pytest
import torch

import oracle
from tests import parity
from workloads import WORKLOADS, make_decode_inputs, random_qkv

pytestmark = pytest.mark.gpu


def _gpu_decode(q, k, v):
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    o, lse = A.attn_decode(q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def _check(got_o, got_lse, q, k, v, label):
    ref_o, ref_lse = oracle.attn_decode(q, k, v)
    assert np.all(np.isfinite(got_o)), label
    ma, rel = parity.errors(got_o, ref_o)
    assert ma <= parity.BF16_TOL["max_abs"], f"{label} O max-abs {ma:.3e}"
    assert rel is None or rel <= parity.BF16_TOL["rel_l2"], f"{label} O rel-L2 {rel:.3e}"
    ml, _ = parity.errors(got_lse, ref_lse)
    assert ml <= parity.LSE_BF16_MAX_ABS, f"{label} lse max-abs {ml:.3e}"


@pytest.mark.parametrize("tq", [1, 4])
def test_gpt2_decode_workload(tq):
    """GPT-2 124M heads (B=12, H=12, D=64) over a full 1024-token cache."""
    inp = make_decode_inputs(WORKLOADS["gpt2_124m"], tq, seed=6)
    _check(*_gpu_decode(inp["q"], inp["k"], inp["v"]), inp["q"], inp["k"], inp["v"], f"gpt2 tq={tq}")


@pytest.mark.parametrize("Tk", [1, 16, 127, 128, 129, 1000, 4097])
@pytest.mark.parametrize("tq", [1, 2, 5, 16])
@pytest.mark.parametrize("D", [32, 64])
def test_decode_lengths(Tk, tq, D):
    if tq > Tk:
        pytest.skip("Tq <= Tk")
    inp = random_qkv(17 * Tk + tq + D, 2, 3, Tk, D, dtype=torch.bfloat16)
    q = inp["q"][:, :, Tk - tq:].contiguous()
    _check(*_gpu_decode(q, inp["k"], inp["v"]), q, inp["k"], inp["v"], f"Tk={Tk} tq={tq} D={D}")


@pytest.mark.parametrize("B,H,Tk", [(1, 1, 2000), (1, 2, 16384), (64, 16, 300)])
def test_decode_cluster_extremes(B, H, Tk):
    """One head over many tiles (cluster of 8, several tiles per CTA), a long
    cache, and many heads (one CTA per head)."""
    inp = random_qkv(B * 1000 + Tk, B, H, Tk, 64, dtype=torch.bfloat16)
    q = inp["q"][:, :, Tk - 3:].contiguous()
    _check(*_gpu_decode(q, inp["k"], inp["v"]), q, inp["k"], inp["v"], f"B={B} H={H} Tk={Tk}")


def test_decode_on_a_cache_of_larger_capacity():
    """k, v are the first Tk rows of [B, H, Tmax, D] caches and of a
    token-major [B, Tmax, H, D] cache; q and o are token-major views."""
    B, H, Tmax, Tk, D, tq = 2, 4, 2048, 777, 64, 3
    dev = torch.device("cuda", 0)
    g = torch.Generator().manual_seed(12)
    cache_k = torch.randn(B, H, Tmax, D, generator=g).to(torch.bfloat16)
    cache_v = torch.randn(B, H, Tmax, D, generator=g).to(torch.bfloat16)
    q_tm = torch.randn(B, tq, H, D, generator=g).to(torch.bfloat16)
    k, v, q = cache_k[:, :, :Tk], cache_v[:, :, :Tk], q_tm.permute(0, 2, 1, 3)
    import decoder_only_transformer_sdpa_b200 as A
    o_buf = torch.full((B, tq, H, D), float("nan"), dtype=torch.bfloat16, device=dev)
    o, lse = A.attn_decode(q.to(dev), cache_k.to(dev)[:, :, :Tk], cache_v.to(dev)[:, :, :Tk],
                           o=o_buf.permute(0, 2, 1, 3))
    torch.cuda.synchronize()
    assert torch.isfinite(o_buf.float()).all()
    _check(o.double().cpu().numpy(), lse.double().cpu().numpy(), q.contiguous(), k.contiguous(),
           v.contiguous(), "capacity cache")
    # the same keys/values in a token-major cache
    ktm = cache_k.permute(0, 2, 1, 3).contiguous().to(dev)
    vtm = cache_v.permute(0, 2, 1, 3).contiguous().to(dev)
    o2, lse2 = A.attn_decode(q.to(dev), ktm[:, :Tk].permute(0, 2, 1, 3), vtm[:, :Tk].permute(0, 2, 1, 3))
    torch.cuda.synchronize()
    assert torch.equal(o2, o) and torch.equal(lse2, lse), "layout must not change the result"


def test_decode_uniform_closed_form():
    """Q = 0: query r averages the values of keys 0 .. Tk - Tq + r."""
    B, H, Tk, D, tq = 2, 2, 555, 64, 5
    inp = random_qkv(3, B, H, Tk, D, dtype=torch.bfloat16)
    q = torch.zeros(B, H, tq, D, dtype=torch.bfloat16)
    o, lse = _gpu_decode(q, inp["k"], inp["v"])
    v = inp["v"].double().numpy()
    for r in range(tq):
        n = Tk - tq + r + 1
        ma, rel = parity.errors(o[:, :, r], v[:, :, :n].mean(axis=2))
        assert ma <= 2e-2 and rel <= 1e-2, (r, ma, rel)
        np.testing.assert_allclose(lse[:, :, r], np.log(n), atol=1e-4)


def test_decode_matches_causal_forward_rows():
    """The decode rows agree with the same rows of the full causal forward
    kernel (two different kernels, both within the oracle's tolerance)."""
    import decoder_only_transformer_sdpa_b200 as A
    inp = random_qkv(44, 2, 3, 700, 64, dtype=torch.bfloat16)
    dev = torch.device("cuda", 0)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    of, lf = A.attn_fwd(q, k, v)
    od, ld = A.attn_decode(q[:, :, -8:].contiguous(), k, v)
    torch.cuda.synchronize()
    torch.testing.assert_close(od.float(), of[:, :, -8:].float(), rtol=0, atol=2e-2)
    torch.testing.assert_close(ld, lf[:, :, -8:], rtol=0, atol=1e-4)
