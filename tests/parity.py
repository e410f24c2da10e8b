"""Helpers for the GPU-vs-oracle parity tests: run the CUDA path through the
C ABI binding, run the oracle on the same bytes (all heads, or a seeded
sample of heads for the full-size workloads), and compare element by element.

Tolerances (written here, used by every parity test):

* float32 path: max-abs <= 1e-5 on O, lse, dQ, dK, dV.
* bf16 path: rel-L2 <= 1e-2 and max-abs <= 2e-2 on O, dQ, dK, dV; the fp32
  lse output (computed from exact bf16 inputs with fp32 accumulation) must be
  within 1e-3 absolute.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

F32_TOL = dict(max_abs=1e-5)
BF16_TOL = dict(max_abs=2e-2, rel_l2=1e-2)
LSE_BF16_MAX_ABS = 1e-3


def run_gpu(inp, scale=None, dtype=torch.bfloat16, causal=True):
    """Forward + backward through the C ABI (the plain entry points for the
    causal attention, the _ex ones with causal=False otherwise).  Returns CPU
    float64 numpy arrays."""
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    if not causal and dtype == torch.bfloat16:
        o, lse = A.attn_fwd_ex(q, k, v, scale=scale, causal=False)
        dq, dk, dv = A.attn_bwd_ex(q, k, v, o, lse, do, scale=scale, causal=False)
    elif not causal:
        o, lse = A.attn_fwd_f32_ex(q, k, v, scale=scale, causal=False)
        dq, dk, dv = A.attn_bwd_f32_ex(q, k, v, o, lse, do, scale=scale, causal=False)
    elif dtype == torch.bfloat16:
        o, lse = A.attn_fwd(q, k, v, scale=scale)
        dq, dk, dv = A.attn_bwd(q, k, v, o, lse, do, scale=scale)
    else:
        o, lse = A.attn_fwd_f32(q, k, v, scale=scale)
        dq, dk, dv = A.attn_bwd_f32(q, k, v, o, lse, do, scale=scale)
    torch.cuda.synchronize()
    assert A.attn_device_error() == 0
    cpu = lambda t: t.detach().to("cpu", torch.float64).numpy()
    return dict(o=cpu(o), lse=cpu(lse), dq=cpu(dq), dk=cpu(dk), dv=cpu(dv))


def sample_heads(B: int, H: int, n: int, seed: int):
    """A seeded sample of flat head indices b*H + h (always the first and last)."""
    total = B * H
    if n >= total:
        return np.arange(total)
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(total, size=n - 2, replace=False).tolist()) | {0, total - 1}
    return np.array(sorted(pick))


def run_oracle(inp, heads=None, scale=None, causal=True):
    """Oracle outputs on all heads, or only the flat head indices `heads`
    (heads are independent, so a subset is computed exactly)."""
    arrs = {n: inp[n].to(torch.float64).numpy() for n in ("q", "k", "v", "do")}
    B, H, T, D = arrs["q"].shape
    if heads is not None:
        arrs = {n: a.reshape(B * H, T, D)[heads][None] for n, a in arrs.items()}
    o, lse = oracle.attn_fwd(arrs["q"], arrs["k"], arrs["v"], scale, causal=causal)
    dq, dk, dv = oracle.attn_bwd(arrs["q"], arrs["k"], arrs["v"], arrs["do"], scale, causal=causal)
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def select_heads(out, heads, B, H):
    if heads is None:
        return out
    res = {}
    for n, a in out.items():
        if a.ndim == 4:
            res[n] = a.reshape(B * H, *a.shape[2:])[heads][None]
        else:
            res[n] = a.reshape(B * H, a.shape[2])[heads][None]
    return res


def errors(got: np.ndarray, ref: np.ndarray):
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / denom if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, ref, dtype, label=""):
    report = {}
    assert np.all(np.isfinite(got["o"])), f"{label}: non-finite O"
    for n in ("o", "dq", "dk", "dv"):
        assert np.all(np.isfinite(got[n])), f"{label}: non-finite {n}"
        ma, rel = errors(got[n], ref[n])
        report[n] = (ma, rel)
        if dtype == torch.float32:
            assert ma <= F32_TOL["max_abs"], f"{label} {n}: max-abs {ma:.3e} > 1e-5"
        else:
            assert ma <= BF16_TOL["max_abs"], f"{label} {n}: max-abs {ma:.3e} > 2e-2"
            assert rel <= BF16_TOL["rel_l2"], f"{label} {n}: rel-L2 {rel:.3e} > 1e-2"
    ma, _ = errors(got["lse"], ref["lse"])
    report["lse"] = (ma, None)
    lim = F32_TOL["max_abs"] if dtype == torch.float32 else LSE_BF16_MAX_ABS
    assert ma <= lim, f"{label} lse: max-abs {ma:.3e} > {lim}"
    return report
