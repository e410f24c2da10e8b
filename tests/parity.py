"""Helpers for the GPU-vs-oracle parity tests: run the CUDA path through the
C ABI binding, run the oracle on the same bytes (all heads, or a seeded
sample of heads for the full-size workloads), and compare element by element.

Tolerances (written here, used by every parity test):

* float32 path: max-abs <= 1e-5 on O, lse, dQ, dK, dV.
* bf16 path: rel-L2 <= 1e-2 and max-abs <= 2e-2 on O, dQ, dK, dV; the fp32
  lse output (computed from exact bf16 inputs with fp32 accumulation) must be
  within 1e-3 absolute.  rel-L2 applies where the oracle's output has an RMS
  above 1e-6; below that the exact output is zero up to the oracle's own
  rounding (e.g. dQ = dK = 0 for a single token), rel-L2 would divide by that
  rounding, and max-abs alone applies.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

F32_TOL = dict(max_abs=1e-5)
BF16_TOL = dict(max_abs=2e-2, rel_l2=1e-2)
LSE_BF16_MAX_ABS = 1e-3


def run_gpu(inp, scale=None, dtype=torch.bfloat16, causal=True, **drop):
    """Forward + backward through the C ABI (the plain entry points for the
    causal attention without dropout, the _ex ones otherwise; ``drop`` takes
    dropout_p, seed, offset).  Returns CPU float64 numpy arrays."""
    import decoder_only_transformer_sdpa_b200 as A
    dev = torch.device("cuda", 0)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    if (not causal or drop) and dtype == torch.bfloat16:
        o, lse = A.attn_fwd_ex(q, k, v, scale=scale, causal=causal, **drop)
        dq, dk, dv = A.attn_bwd_ex(q, k, v, o, lse, do, scale=scale, causal=causal, **drop)
    elif not causal or drop:
        o, lse = A.attn_fwd_f32_ex(q, k, v, scale=scale, causal=causal, **drop)
        dq, dk, dv = A.attn_bwd_f32_ex(q, k, v, o, lse, do, scale=scale, causal=causal, **drop)
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


def run_oracle(inp, heads=None, scale=None, causal=True, **drop):
    """Oracle outputs on all heads, or only the flat head indices `heads`
    (heads are independent, so a subset is computed exactly)."""
    arrs = {n: inp[n].to(torch.float64).numpy() for n in ("q", "k", "v", "do")}
    B, H, T, D = arrs["q"].shape
    if heads is not None and drop:
        # the keep mask depends on the flat head index: run the oracle per head
        # as a one-head problem whose mask is that head's (seed, offset) mask
        outs = [run_oracle({n: inp[n].reshape(B * H, T, D)[h][None, None]
                            for n in ("q", "k", "v", "do")}, None, scale, causal,
                           **{**drop, "head0": int(h)}) for h in heads]
        return {n: np.concatenate([o[n] for o in outs], axis=1) for n in outs[0]}
    if heads is not None:
        arrs = {n: a.reshape(B * H, T, D)[heads][None] for n, a in arrs.items()}
    o, lse = oracle.attn_fwd(arrs["q"], arrs["k"], arrs["v"], scale, causal=causal, **drop)
    dq, dk, dv = oracle.attn_bwd(arrs["q"], arrs["k"], arrs["v"], arrs["do"], scale, causal=causal,
                                 **drop)
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


REL_L2_MIN_RMS = 1e-6


def errors(got: np.ndarray, ref: np.ndarray):
    """(max-abs, rel-L2) of got against ref; rel-L2 is None when ref's RMS is
    at most REL_L2_MIN_RMS (an exactly-zero result up to rounding)."""
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    if diff.size == 0 or denom <= REL_L2_MIN_RMS * np.sqrt(diff.size):
        return max_abs, None
    return max_abs, float(np.linalg.norm(diff)) / denom


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
            assert rel is None or rel <= BF16_TOL["rel_l2"], f"{label} {n}: rel-L2 {rel:.3e} > 1e-2"
    ma, _ = errors(got["lse"], ref["lse"])
    report["lse"] = (ma, None)
    lim = F32_TOL["max_abs"] if dtype == torch.float32 else LSE_BF16_MAX_ABS
    assert ma <= lim, f"{label} lse: max-abs {ma:.3e} > {lim}"
    return report
