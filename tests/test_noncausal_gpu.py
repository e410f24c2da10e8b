"""GPU parity of the non-causal variant (no -inf triangle: every query sees
all T keys) against the oracle's non-causal entry points, on the same seeded
inputs and with the same tolerances as the causal path (tests/parity.py)."""
import numpy as np
import pytest
import torch

from tests import parity
from workloads import WORKLOADS, make_inputs, make_inputs_packed, packed_views, random_qkv

pytestmark = pytest.mark.gpu


def test_tiny_f32_workload_noncausal():
    inp = make_inputs(WORKLOADS["tiny_f32"], seed=0)
    got = parity.run_gpu(inp, dtype=torch.float32, causal=False)
    parity.assert_close(got, parity.run_oracle(inp, causal=False), torch.float32, "tiny_f32 nc")


@pytest.mark.parametrize("B,H,T,D", [(1, 1, 1, 1), (2, 3, 7, 3), (1, 2, 65, 13), (1, 2, 200, 128)])
def test_f32_odd_shapes_noncausal(B, H, T, D):
    inp = random_qkv(300 + T + D, B, H, T, D)
    got = parity.run_gpu(inp, dtype=torch.float32, causal=False)
    parity.assert_close(got, parity.run_oracle(inp, causal=False), torch.float32, f"f32 nc {T},{D}")


@pytest.mark.parametrize("name", ["char_gpt", "small_head"])
def test_bf16_workload_all_heads_noncausal(name):
    inp = make_inputs(WORKLOADS[name], seed=1)
    got = parity.run_gpu(inp, causal=False)
    parity.assert_close(got, parity.run_oracle(inp, causal=False), torch.bfloat16, f"{name} nc")


def test_bf16_gpt2_sampled_heads_noncausal():
    """The GPT-2 124M shape in the launch configuration the bench times."""
    w = WORKLOADS["gpt2_124m"]
    inp = make_inputs(w, seed=2)
    got = parity.run_gpu(inp, causal=False)
    heads = parity.sample_heads(w.B, w.H, 6, seed=2)
    ref = parity.run_oracle(inp, heads=heads, causal=False)
    parity.assert_close(parity.select_heads(got, heads, w.B, w.H), ref, torch.bfloat16, "gpt2 nc")


@pytest.mark.parametrize("T", [1, 2, 17, 127, 128, 129, 300, 1025])
@pytest.mark.parametrize("D", [32, 64])
def test_bf16_ragged_lengths_noncausal(T, D):
    inp = random_qkv(9 * T + D, 2, 3, T, D, dtype=torch.bfloat16, do_std=1e-2)
    got = parity.run_gpu(inp, causal=False)
    parity.assert_close(got, parity.run_oracle(inp, causal=False), torch.bfloat16, f"nc T={T} D={D}")


@pytest.mark.parametrize("D", [32, 64])
def test_bf16_averaging_noncausal(D):
    """Q = 0 without the mask: every row is the mean of all values, lse = ln T,
    and dK = 0 exactly."""
    T = 333
    inp = random_qkv(6, 2, 2, T, D, dtype=torch.bfloat16, do_std=1e-2)
    inp["q"] = torch.zeros_like(inp["q"])
    got = parity.run_gpu(inp, causal=False)
    v = inp["v"].to(torch.float64).numpy()
    mean = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
    ma, rel = parity.errors(got["o"], mean)
    assert ma <= 2e-2 and rel <= 1e-2, (ma, rel)
    np.testing.assert_allclose(got["lse"], np.log(T), atol=1e-4)
    assert np.all(got["dk"] == 0.0), "Q = 0 must give dK = 0 exactly"


@pytest.mark.parametrize("T,D", [(700, 64), (256, 32), (129, 64)])
def test_bf16_last_row_matches_causal(T, D):
    """The causal last row already attends to every key: both variants run the
    same tiles with the same mask there, so O and lse of row T - 1 agree
    bit for bit."""
    inp = random_qkv(40 + T, 2, 2, T, D, dtype=torch.bfloat16, do_std=1e-2)
    c = parity.run_gpu(inp)
    nc = parity.run_gpu(inp, causal=False)
    assert np.array_equal(nc["o"][:, :, -1], c["o"][:, :, -1])
    assert np.array_equal(nc["lse"][:, :, -1], c["lse"][:, :, -1])
    assert not np.array_equal(nc["o"][:, :, 0], c["o"][:, :, 0])


def test_bf16_packed_layout_noncausal():
    """Non-causal attention on the c_attn layout (strided views) through the
    same _ex entry points."""
    import decoder_only_transformer_sdpa_b200 as A
    w = WORKLOADS["char_gpt"]
    inp = make_inputs_packed(w, seed=4)
    dev = torch.device("cuda", 0)
    qkv = inp["qkv"].to(dev)
    B, T, C3 = qkv.shape
    D = C3 // 3 // w.H
    q, k, v = packed_views(qkv, w.H)
    do = inp["do_packed"].to(dev).view(B, T, w.H, D).permute(0, 2, 1, 3)
    o, lse = A.attn_fwd_ex(q, k, v, causal=False)
    dq, dk, dv = A.attn_bwd_ex(q, k, v, o, lse, do, causal=False)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    assert o.stride() == (T * C3 // 3, D, C3 // 3, 1)
    cpu = lambda t: t.detach().to("cpu", torch.float64).contiguous().numpy()
    got = dict(o=cpu(o), lse=cpu(lse), dq=cpu(dq), dk=cpu(dk), dv=cpu(dv))
    heads = parity.sample_heads(w.B, w.H, 8, seed=4)
    ref = parity.run_oracle(inp, heads=heads, causal=False)
    parity.assert_close(parity.select_heads(got, heads, w.B, w.H), ref, torch.bfloat16, "packed nc")
