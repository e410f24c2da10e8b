"""GPU parity of attention dropout: the keep mask the kernels draw (forward
and backward) equals the oracle's bit for bit, and forward/backward with
dropout match the oracle's dropout attention on the same seeded inputs with
the tolerances of tests/parity.py."""
import numpy as np
import pytest
import torch

import oracle
from tests import parity
from workloads import WORKLOADS, make_inputs, random_qkv

pytestmark = pytest.mark.gpu


def _keep_scale(p):
    t = int(np.floor(p * 65536.0 + 0.5))
    return 65536.0 / (65536.0 - t)


def _masks_from_gpu(B, H, T, D, causal, p, seed, offset, dtype):
    """Reads the keep mask out of the GPU forward (O) and backward (dV).

    With Q = 0 every visible weight is equal and positive, so with V one-hot
    over a 64-key chunk, O[i, d] > 0 exactly when key 64 c + d is kept for
    query i; with dO one-hot over a 64-query chunk, dV[j, d] > 0 exactly when
    key j is kept for query 64 c + d."""
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    fwd = A.attn_fwd_ex if dtype == torch.bfloat16 else A.attn_fwd_f32_ex
    bwd = A.attn_bwd_ex if dtype == torch.bfloat16 else A.attn_bwd_f32_ex
    q = torch.zeros(B, H, T, D, dtype=dtype, device=dev)
    k = torch.randn(B, H, T, D, generator=torch.Generator().manual_seed(1)).to(dtype).to(dev)
    m_fwd = np.zeros((B, H, T, T), dtype=np.uint8)
    m_bwd = np.zeros((B, H, T, T), dtype=np.uint8)
    kw = dict(causal=causal, dropout_p=p, seed=seed, offset=offset)
    for c in range((T + D - 1) // D):
        onehot = torch.zeros(B, H, T, D, dtype=dtype, device=dev)
        rows = torch.arange(c * D, min(T, (c + 1) * D), device=dev)
        onehot[:, :, rows, rows - c * D] = 1
        o, lse = fwd(q, k, onehot, **kw)
        # backward with V = one-hot too (any V works for dV), dO = one-hot
        dq, dk, dv = bwd(q, k, onehot, o, lse, onehot, **kw)
        torch.cuda.synchronize()
        n = len(rows)
        m_fwd[:, :, :, c * D:c * D + n] = (o[..., :n].float() > 0).cpu().numpy()
        m_bwd[:, :, c * D:c * D + n, :] = (dv[..., :n].float() > 0).cpu().numpy().transpose(0, 1, 3, 2)
    assert A.attn_device_error() == 0
    return m_fwd, m_bwd


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("T", [64, 300])
def test_keep_mask_bit_exact(dtype, causal, T):
    B, H, D, p, seed, offset = 2, 3, 64, 0.3, 0x5EED0123456789, 7
    m_fwd, m_bwd = _masks_from_gpu(B, H, T, D, causal, p, seed, offset, dtype)
    ref = oracle.dropout_mask(B, H, T, p, seed, offset)
    if causal:
        ref = ref * np.tril(np.ones((T, T), dtype=np.uint8))
    assert np.array_equal(m_fwd, ref), f"forward mask: {np.sum(m_fwd != ref)} of {ref.size} bits differ"
    assert np.array_equal(m_bwd, ref), f"backward mask: {np.sum(m_bwd != ref)} of {ref.size} bits differ"


def test_tiny_f32_workload_dropout():
    inp = make_inputs(WORKLOADS["tiny_f32"], seed=0)
    for causal in (True, False):
        kw = dict(dropout_p=0.2, seed=3, offset=1)
        got = parity.run_gpu(inp, dtype=torch.float32, causal=causal, **kw)
        ref = parity.run_oracle(inp, causal=causal, **kw)
        parity.assert_close(got, ref, torch.float32, f"tiny f32 dropout causal={causal}")


@pytest.mark.parametrize("B,H,T,D", [(1, 1, 1, 1), (2, 3, 7, 3), (1, 2, 65, 13), (1, 2, 200, 128)])
def test_f32_odd_shapes_dropout(B, H, T, D):
    inp = random_qkv(500 + T + D, B, H, T, D)
    kw = dict(dropout_p=0.25, seed=T, offset=D)
    for causal in (True, False):
        got = parity.run_gpu(inp, dtype=torch.float32, causal=causal, **kw)
        parity.assert_close(got, parity.run_oracle(inp, causal=causal, **kw), torch.float32,
                            f"f32 dropout {T},{D} causal={causal}")


def test_bf16_char_gpt_dropout_all_heads():
    """The character-level GPT shape, all heads, at a second rate (0.2)."""
    inp = make_inputs(WORKLOADS["char_gpt"], seed=3)
    kw = dict(dropout_p=0.2, seed=1234, offset=5)
    got = parity.run_gpu(inp, **kw)
    parity.assert_close(got, parity.run_oracle(inp, **kw), torch.bfloat16, "char_gpt dropout")


@pytest.mark.parametrize("causal", [True, False])
def test_bf16_gpt2_dropout_sampled_heads(causal):
    """GPT-2 124M shape, rate 0.1, in the launch configuration the bench times."""
    w = WORKLOADS["gpt2_124m"]
    inp = make_inputs(w, seed=4)
    kw = dict(dropout_p=0.1, seed=99, offset=11)
    got = parity.run_gpu(inp, causal=causal, **kw)
    heads = parity.sample_heads(w.B, w.H, 5, seed=4)
    ref = parity.run_oracle(inp, heads=heads, causal=causal, **kw)
    parity.assert_close(parity.select_heads(got, heads, w.B, w.H), ref, torch.bfloat16,
                        f"gpt2 dropout causal={causal}")


@pytest.mark.parametrize("T", [1, 17, 129, 300])
@pytest.mark.parametrize("D", [32, 64])
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_ragged_dropout(T, D, causal):
    inp = random_qkv(13 * T + D, 2, 3, T, D, dtype=torch.bfloat16, do_std=1e-2)
    kw = dict(dropout_p=0.1, seed=T * 7 + D, offset=2)
    got = parity.run_gpu(inp, causal=causal, **kw)
    parity.assert_close(got, parity.run_oracle(inp, causal=causal, **kw), torch.bfloat16,
                        f"dropout T={T} D={D} causal={causal}")


def test_bf16_dropout_determinism_and_fresh_masks():
    """Same (seed, offset): identical O, lse, dK, dV; another offset or seed:
    different O; lse never depends on the mask."""
    inp = random_qkv(8, 2, 2, 256, 64, dtype=torch.bfloat16, do_std=1e-2)
    a = parity.run_gpu(inp, dropout_p=0.1, seed=1, offset=0)
    b = parity.run_gpu(inp, dropout_p=0.1, seed=1, offset=0)
    for n in ("o", "lse", "dk", "dv"):
        assert np.array_equal(a[n], b[n]), n
    c = parity.run_gpu(inp, dropout_p=0.1, seed=1, offset=1)
    d = parity.run_gpu(inp, dropout_p=0.1, seed=2, offset=0)
    assert not np.array_equal(a["o"], c["o"]) and not np.array_equal(a["o"], d["o"])
    assert np.array_equal(a["lse"], c["lse"]) and np.array_equal(a["lse"], d["lse"])
    plain = parity.run_gpu(inp)
    assert np.array_equal(a["lse"], plain["lse"])


def test_bf16_zero_threshold_is_plain():
    """p below 1/131072 rounds to threshold 0: the kernels without dropout run
    and the result is bit-identical to the plain entry points."""
    inp = random_qkv(9, 2, 2, 200, 64, dtype=torch.bfloat16, do_std=1e-2)
    a = parity.run_gpu(inp, dropout_p=1e-6, seed=1, offset=0)
    b = parity.run_gpu(inp)
    for n in ("o", "lse", "dk", "dv"):
        assert np.array_equal(a[n], b[n]), n


def _unpack_kept_mask(buf, B, H, T):
    """The [B, H, T, T] keep bits of a kept dropout mask buffer (layout of
    include/attn.h: byte (query i, key group g) of head bh at
    (bh * Tp + i) * Tp/8 + g, bit e = key 8 g + e)."""
    tp = (T + 127) // 128 * 128
    by = buf.cpu().numpy().reshape(B * H, tp, tp // 8)           # [bh, i, g]
    bits = np.unpackbits(by[..., None], axis=-1, bitorder="little")  # [bh, i, g, e]
    m = bits.reshape(B * H, tp, tp)                              # [bh, i, 8 g + e]
    return m[:, :T, :T].reshape(B, H, T, T)


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_kept_mask_bits_equal_oracle(D, causal):
    """The forward call stores exactly the oracle's keep bits for every tile
    the kernels visit (with the mask, the tiles at or below the diagonal)."""
    import decoder_only_transformer_sdpa_b200 as A
    B, H, T, p, seed, offset = 2, 3, 300, 0.3, 0x5EED0123456789, 9
    inp = random_qkv(71 + D, B, H, T, D, dtype=torch.bfloat16)
    dev = torch.device("cuda", 0)
    buf = torch.full((A.attn_dropout_mask_bytes(B, H, T),), 0xA5, dtype=torch.uint8, device=dev)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    A.attn_fwd_ex(q, k, v, causal=causal, dropout_p=p, seed=seed, offset=offset, dropout_mask=buf)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    got = _unpack_kept_mask(buf, B, H, T)
    ref = oracle.dropout_mask(B, H, T, p, seed, offset)
    drawn = np.ones((T, T), dtype=bool)
    if causal:  # tiles of 128 x 128 at or below the diagonal
        tq = np.arange(T)[:, None] // 128
        tk = np.arange(T)[None, :] // 128
        drawn = tk <= tq
    assert np.array_equal(got[..., drawn], ref[..., drawn]), \
        f"{np.sum(got[..., drawn] != ref[..., drawn])} kept bits differ from the oracle's"


@pytest.mark.parametrize("D,T", [(64, 333), (64, 1024), (128, 333), (32, 200)])
@pytest.mark.parametrize("causal", [True, False])
def test_kept_mask_backward_matches_redraw(D, T, causal):
    """The backward that reads the forward's kept mask gives what the one that
    draws the mask again gives (dK, dV bit for bit; dQ, summed by float32
    reduce-adds in whatever order they land, within its rounding), and both
    match the oracle."""
    import decoder_only_transformer_sdpa_b200 as A
    B, H = 2, 2
    inp = random_qkv(900 + T + D, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
    dev = torch.device("cuda", 0)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    kw = dict(causal=causal, dropout_p=0.1, seed=123, offset=4)
    buf = torch.zeros(A.attn_dropout_mask_bytes(B, H, T), dtype=torch.uint8, device=dev)
    o1, lse1 = A.attn_fwd_ex(q, k, v, dropout_mask=buf, **kw)
    g1 = A.attn_bwd_ex(q, k, v, o1, lse1, do, dropout_mask=buf, **kw)
    o0, lse0 = A.attn_fwd_ex(q, k, v, **kw)
    g0 = A.attn_bwd_ex(q, k, v, o0, lse0, do, **kw)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    assert torch.equal(o1, o0) and torch.equal(lse1, lse0)
    assert torch.equal(g1[1], g0[1]) and torch.equal(g1[2], g0[2])
    assert torch.allclose(g1[0].float(), g0[0].float(), rtol=1e-2, atol=1e-6)
    cpu = lambda t: t.detach().to("cpu", torch.float64).numpy()
    got = dict(o=cpu(o1), lse=cpu(lse1), dq=cpu(g1[0]), dk=cpu(g1[1]), dv=cpu(g1[2]))
    parity.assert_close(got, parity.run_oracle(inp, causal=causal, dropout_p=0.1, seed=123, offset=4),
                        torch.bfloat16, f"kept mask D={D} T={T} causal={causal}")
