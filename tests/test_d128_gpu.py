"""GPU parity at head_dim 128 (the forward with two 64-column slabs per tile,
the backward main kernel with 64-query sub-tiles and a transposed dQ) against
the oracle, with the tolerances of tests/parity.py: causal and not, dropout,
ragged lengths around both tile sizes (64 and 128), packed c_attn layouts."""
import numpy as np
import pytest
import torch

from tests import parity
from workloads import random_qkv

pytestmark = pytest.mark.gpu

D = 128


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129, 200, 300, 1025])
@pytest.mark.parametrize("causal", [True, False])
def test_d128_ragged(T, causal):
    inp = random_qkv(61 * T + int(causal), 2, 3, T, D, dtype=torch.bfloat16, do_std=1e-2)
    got = parity.run_gpu(inp, causal=causal)
    parity.assert_close(got, parity.run_oracle(inp, causal=causal), torch.bfloat16,
                        f"D=128 T={T} causal={causal}")


def test_d128_wide_shape_sampled_heads():
    """C = 768 split into 6 heads of 128 at the GPT-2 124M batch and context
    (B = 12, T = 1024), in the launch configuration the bench times."""
    B, H, T = 12, 6, 1024
    inp = random_qkv(128, B, H, T, D, dtype=torch.bfloat16, std=0.55, do_std=1e-2)
    got = parity.run_gpu(inp)
    heads = parity.sample_heads(B, H, 6, seed=1)
    parity.assert_close(parity.select_heads(got, heads, B, H), parity.run_oracle(inp, heads=heads),
                        torch.bfloat16, "D=128 B=12 H=6 T=1024")


@pytest.mark.parametrize("causal", [True, False])
def test_d128_dropout(causal):
    inp = random_qkv(7, 2, 2, 333, D, dtype=torch.bfloat16, do_std=1e-2)
    kw = dict(dropout_p=0.1, seed=21, offset=4)
    got = parity.run_gpu(inp, causal=causal, **kw)
    parity.assert_close(got, parity.run_oracle(inp, causal=causal, **kw), torch.bfloat16,
                        f"D=128 dropout causal={causal}")


def test_d128_causality_and_averaging():
    """Tokens after t leave O and lse at rows <= t bit-identical; Q = 0 gives
    the prefix mean of V and dK = 0 exactly."""
    T = 300
    inp = random_qkv(12, 1, 2, T, D, dtype=torch.bfloat16, do_std=1e-2)
    base = parity.run_gpu(inp)
    for t in (0, 63, 64, 200):
        pert = {n: a.clone() for n, a in inp.items()}
        g = torch.Generator().manual_seed(t)
        for n in pert:
            tail = pert[n][:, :, t + 1:]
            tail += (3.0 * torch.randn(tail.shape, generator=g)).to(tail.dtype)
        got = parity.run_gpu(pert)
        for n in ("o", "lse"):
            assert np.array_equal(got[n][:, :, :t + 1], base[n][:, :, :t + 1]), f"{n} at t={t}"
    zq = dict(inp, q=torch.zeros_like(inp["q"]))
    got = parity.run_gpu(zq)
    v = inp["v"].to(torch.float64).numpy()
    prefix = np.cumsum(v, axis=2) / np.arange(1, T + 1)[:, None]
    ma, rel = parity.errors(got["o"], prefix)
    assert ma <= 2e-2 and rel <= 1e-2, (ma, rel)
    assert np.all(got["dk"] == 0.0)


def test_d128_packed_layout():
    """q, k, v slices of a [B, T, 3C] c_attn output (C = 4 * 128), O written
    as [B, T, C], gradients into one [B, T, 3C] buffer."""
    import decoder_only_transformer_sdpa_b200 as A
    from workloads import packed_views
    B, H, T = 2, 4, 257
    inp = random_qkv(99, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
    dev = torch.device("cuda", 0)
    tm = lambda t: t.permute(0, 2, 1, 3).reshape(B, T, H * D)
    qkv = torch.cat([tm(inp["q"]), tm(inp["k"]), tm(inp["v"])], dim=2).contiguous().to(dev)
    q, k, v = packed_views(qkv, H)
    do = tm(inp["do"]).contiguous().to(dev).view(B, T, H, D).permute(0, 2, 1, 3)
    o, lse = A.attn_fwd_strided(q, k, v)
    dqkv = torch.full_like(qkv, float("nan"))
    dq, dk, dv = packed_views(dqkv, H)
    A.attn_bwd_strided(q, k, v, o, lse, do, dq, dk, dv)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    assert torch.isfinite(dqkv.float()).all()
    cpu = lambda t: t.detach().to("cpu", torch.float64).contiguous().numpy()
    got = dict(o=cpu(o), lse=cpu(lse), dq=cpu(dq), dk=cpu(dk), dv=cpu(dv))
    parity.assert_close(got, parity.run_oracle(inp), torch.bfloat16, "D=128 packed")


@pytest.mark.parametrize("causal,dropout_p", [(True, 0.0), (False, 0.0), (True, 0.1)])
def test_d128_many_items_per_cta(causal, dropout_p):
    """768 (key tile, head) items, about five waves of CTAs on 148 SMs, with
    every head checked."""
    B, H, T = 16, 24, 130
    inp = random_qkv(4242 + int(causal), B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
    kw = dict(dropout_p=dropout_p, seed=5, offset=0) if dropout_p else {}
    got = parity.run_gpu(inp, causal=causal, **kw)
    parity.assert_close(got, parity.run_oracle(inp, causal=causal, **kw), torch.bfloat16,
                        f"D=128 B={B} H={H} T={T} causal={causal} p={dropout_p}")
