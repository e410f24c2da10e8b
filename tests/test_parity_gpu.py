"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs, element by element (tolerances in tests/parity.py)."""
import numpy as np
import pytest
import torch

from tests import parity
from workloads import WORKLOADS, make_inputs, random_qkv

pytestmark = pytest.mark.gpu


def test_tiny_f32_workload():
    w = WORKLOADS["tiny_f32"]
    inp = make_inputs(w, seed=0)
    got = parity.run_gpu(inp, dtype=torch.float32)
    ref = parity.run_oracle(inp)
    parity.assert_close(got, ref, torch.float32, "tiny_f32")


@pytest.mark.parametrize("B,H,T,D", [(1, 1, 1, 1), (2, 3, 7, 3), (1, 2, 65, 13), (1, 1, 130, 100),
                                     (1, 2, 200, 128), (3, 1, 64, 64), (1, 1, 1, 128)])
def test_f32_odd_shapes(B, H, T, D):
    inp = random_qkv(100 + T + D, B, H, T, D)
    got = parity.run_gpu(inp, dtype=torch.float32)
    ref = parity.run_oracle(inp)
    parity.assert_close(got, ref, torch.float32, f"f32 {B},{H},{T},{D}")


@pytest.mark.parametrize("name", ["char_gpt", "small_head"])
def test_bf16_workload_all_heads(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0)
    got = parity.run_gpu(inp)
    ref = parity.run_oracle(inp)
    parity.assert_close(got, ref, torch.bfloat16, name)


@pytest.mark.parametrize("name,layer", [("gpt2_124m", 0), ("gpt2_124m", 11), ("gpt2_xl", 0)])
def test_bf16_full_size_sampled_heads(name, layer):
    """Full-size workload on the GPU (the bench's launch configuration); the
    oracle recomputes a seeded sample of whole heads exactly."""
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0, layer=layer)
    got = parity.run_gpu(inp)
    heads = parity.sample_heads(w.B, w.H, 8, seed=layer)
    ref = parity.run_oracle(inp, heads=heads)
    parity.assert_close(parity.select_heads(got, heads, w.B, w.H), ref, torch.bfloat16,
                        f"{name} layer {layer}")


@pytest.mark.parametrize("T", [1, 2, 17, 127, 128, 129, 255, 300, 1000, 1025])
@pytest.mark.parametrize("D", [32, 64])
def test_bf16_ragged_lengths(T, D):
    inp = random_qkv(7 * T + D, 2, 3, T, D, dtype=torch.bfloat16, do_std=1e-2)
    got = parity.run_gpu(inp)
    ref = parity.run_oracle(inp)
    parity.assert_close(got, ref, torch.bfloat16, f"T={T} D={D}")


@pytest.mark.parametrize("D", [32, 64])
def test_bf16_single_head_long(D):
    inp = random_qkv(11 + D, 1, 1, 2048, D, dtype=torch.bfloat16, do_std=1e-2)
    got = parity.run_gpu(inp)
    ref = parity.run_oracle(inp)
    parity.assert_close(got, ref, torch.bfloat16, f"B*H=1 T=2048 D={D}")


@pytest.mark.parametrize("D", [32, 64])
def test_bf16_averaging_trick(D):
    """Q = 0: every row is the prefix mean of V (the pages' averaging trick)."""
    inp = random_qkv(5, 2, 2, 333, D, dtype=torch.bfloat16, do_std=1e-2)
    inp["q"] = torch.zeros_like(inp["q"])
    got = parity.run_gpu(inp)
    v = inp["v"].to(torch.float64).numpy()
    n = np.arange(1, v.shape[2] + 1, dtype=np.float64)
    prefix = np.cumsum(v, axis=2) / n[:, None]
    ma, rel = parity.errors(got["o"], prefix)
    assert ma <= 2e-2 and rel <= 1e-2, (ma, rel)
    np.testing.assert_allclose(got["lse"], np.broadcast_to(np.log(n), got["lse"].shape), atol=1e-4)
    assert np.all(got["dk"] == 0.0), "Q = 0 must give dK = 0 exactly"


@pytest.mark.parametrize("D", [32, 64])
def test_bf16_causality(D):
    """Changing tokens after t leaves O and lse at rows <= t bit-identical and
    dQ there unchanged up to the accumulation order of its float32 sums."""
    T = 700
    inp = random_qkv(21, 1, 2, T, D, dtype=torch.bfloat16, do_std=1e-2)
    base = parity.run_gpu(inp)
    for t in (0, 127, 128, 450):
        pert = {n: a.clone() for n, a in inp.items()}
        g = torch.Generator().manual_seed(t)
        for n in pert:
            tail = pert[n][:, :, t + 1:]
            tail += (3.0 * torch.randn(tail.shape, generator=g)).to(tail.dtype)
        got = parity.run_gpu(pert)
        for n in ("o", "lse"):
            assert np.array_equal(got[n][:, :, :t + 1], base[n][:, :, :t + 1]), f"{n} at t={t}"
        np.testing.assert_allclose(got["dq"][:, :, :t + 1], base["dq"][:, :, :t + 1], rtol=0,
                                   atol=1e-4, err_msg=f"dq at t={t}")


def test_bf16_guard_bands_and_determinism():
    """Outputs written exactly in place (NaN guard bands around every output
    stay untouched) and repeated runs give identical O, lse, dK, dV."""
    import decoder_only_transformer_sdpa_b200 as A
    B, H, T, D = 2, 3, 333, 64
    dev = torch.device("cuda", 0)
    inp = random_qkv(3, B, H, T, D, dtype=torch.bfloat16, do_std=1e-2)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    n = B * H * T * D
    pad = 4096

    def guarded(numel, dtype):
        buf = torch.full((numel + 2 * pad,), float("nan"), dtype=dtype, device=dev)
        return buf, buf[pad:pad + numel]

    results = []
    for _ in range(2):
        bo, o = guarded(n, torch.bfloat16)
        bl, lse = guarded(B * H * T, torch.float32)
        grads = [guarded(n, torch.bfloat16) for _ in range(3)]
        A.attn_fwd(q, k, v, o.view(B, H, T, D), lse.view(B, H, T))
        A.attn_bwd(q, k, v, o.view(B, H, T, D), lse.view(B, H, T), do,
                   *(g[1].view(B, H, T, D) for g in grads))
        torch.cuda.synchronize()
        for buf in [bo, bl] + [g[0] for g in grads]:
            assert torch.isnan(buf[:pad].float()).all() and torch.isnan(buf[-pad:].float()).all()
        for t in [o, lse] + [g[1] for g in grads]:
            assert torch.isfinite(t.float()).all()
        results.append([t.clone() for t in [o, lse] + [g[1] for g in grads]])
    names = ["o", "lse", "dq", "dk", "dv"]
    for name, a, b in zip(names, results[0], results[1]):
        if name == "dq":
            torch.testing.assert_close(a.float(), b.float(), rtol=0, atol=1e-3)
        else:
            assert torch.equal(a, b), f"{name} differs between identical runs"


def test_bf16_o_error_by_magnitude_band():
    """bf16 O against the oracle, broken out by |O| band (< 1, 1-4, >= 4), on
    the GPT-2 XL workload, whose outlier keys (1% of K rows x8) concentrate a
    row's attention on single value rows so that |O| reaches the range where
    bf16's own half-ulp (2^-7 on [2, 4), 2^-6 on [4, 8)) takes much of the 2e-2
    budget.  Every band must meet the bound, and every element must be within
    the error the bf16 path can have: half an ulp of its exact value (the final
    rounding) plus the rounding of the weights P to bf16 before P V, which moves
    O by at most 2^-9 max|v| (2^-8 max|v| is allowed, which also covers the
    float32 normalisation).  The band table is printed as the headroom report."""
    w = WORKLOADS["gpt2_xl"]
    inp = make_inputs(w, seed=0)
    got = parity.run_gpu(inp)
    heads = parity.sample_heads(w.B, w.H, 10, seed=5)
    ref = parity.run_oracle(inp, heads=heads)
    o = parity.select_heads(got, heads, w.B, w.H)["o"]
    r = ref["o"]
    v = inp["v"].to(torch.float64).numpy().reshape(w.B * w.H, w.T, w.D)[heads][None]
    vmax = np.max(np.abs(v), axis=(2, 3), keepdims=True)          # per head
    a = np.abs(r)
    half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.maximum(a, 1e-30))) - 8), 0.0)
    bound = half_ulp + 2.0 ** -8 * vmax
    err = np.abs(o - r)
    report, failures = [], []
    for lo, hi in ((0.0, 1.0), (1.0, 4.0), (4.0, np.inf)):
        m = (a >= lo) & (a < hi)
        if not m.any():
            report.append(f"|O| in [{lo},{hi}): empty")
            continue
        ma = float(np.max(err[m]))
        slack = float(np.min((bound - err)[m]))
        report.append(f"|O| in [{lo},{hi}): n={int(m.sum())} max-abs {ma:.3e} (headroom to 2e-2: "
                      f"{2e-2 - ma:.3e}; smallest slack to the bf16 bound: {slack:.3e})")
        if ma > parity.BF16_TOL["max_abs"] or slack < 0:
            failures.append(report[-1])
    print("O error by |O| band (gpt2_xl):\n  " + "\n  ".join(report))
    assert not failures, failures
