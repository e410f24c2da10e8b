"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each check takes an oracle implementation (an object with ``attn_fwd``,
``attn_bwd`` and ``attn_probs``) and raises AssertionError on a violation, so
that the same checks run on the committed oracle and on deliberately broken
variants of it (see test_oracle_mutations.py).

What pins what:

* rows of P sum to 1 and P is zero above the diagonal -- the softmax replaces
  the row-normalised lower-triangular matrix ("How Andrej Karpathy built GPT
  from 200 lines of code", section "Self-Attention: the mathematical trick",
  [51:04] and [55:20]);
* Q = 0 (or K = 0) turns causal attention into the averaging trick: every
  token gets the mean of the values of the tokens up to it (same section,
  [43:56]-[51:04]); closed forms follow for O, lse, dV, dK and dQ;
* perturbing tokens after t leaves O, lse and dQ at rows <= t bit-identical
  (the -inf upper triangle, [55:20]);
* T = 1 returns V exactly and lse = scale * <q, k>;
* adding one vector u to every key leaves P, O, dV, dK, dQ unchanged and adds
  scale * <q_i, u> to lse_i (softmax shift invariance);
* central finite differences of L = sum(O * dO) match dQ, dK, dV;
* torch's float64 CPU ``scaled_dot_product_attention(is_causal=True)`` and its
  autograd, a library routine used as an independent witness;
* small hand-derived golden examples under tests/golden/.

The non-causal variant (``causal=False``: no -inf triangle, every token sees
every token) has pins of its own: rows of P sum to 1 with every entry positive;
Q = 0 gives the mean of all values and lse = ln T; relabelling the tokens by a
permutation relabels every output the same way (nothing depends on position);
its last row equals the causal last row (both see all T keys); shift
invariance, finite differences, torch's ``is_causal=False`` witness and a
hand-derived golden example.

Dropout on the attention weights (keep mask drawn by Philox4x32-10) is pinned
by: the generator against cuRAND's host Philox4x32-10 generator (a library
routine, run on the CPU), word by word and as the whole keep mask of a head;
the keep rate within binomial bounds and distinct masks per head, offset and
seed; p below 1/131072 (threshold 0) giving back the plain attention bit for
bit; the uniform-weight closed form; unbiasedness of O and dV over seeds;
finite differences with the mask held fixed; and torch float64 autograd of
the same dropped-weight attention.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def check_probs_rows(impl, seed=1):
    r = _rng(seed)
    B, H, T, D = 2, 3, 17, 5
    q, k = r.standard_normal((B, H, T, D)), r.standard_normal((B, H, T, D)) * 3.0
    p = impl.attn_probs(q, k)
    assert np.all(np.abs(p.sum(-1) - 1.0) <= 1e-14), "rows of P must sum to 1"
    upper = np.triu(np.ones((T, T), dtype=bool), 1)
    assert np.all(p[..., upper] == 0.0), "P must be zero above the diagonal"
    assert np.all(p[..., ~upper] > 0.0), "P must be positive on and below the diagonal"


def check_averaging_trick(impl, seed=2):
    """Q = 0 (then K = 0): all scores equal, so P is the row-normalised tril."""
    r = _rng(seed)
    B, H, T, D = 2, 2, 11, 6
    k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(3))
    scale = 1.0 / math.sqrt(D)
    n = np.arange(1, T + 1, dtype=np.float64)              # i + 1
    prefix_mean = np.cumsum(v, axis=2) / n[:, None]

    zero = np.zeros_like(k)
    o, lse = impl.attn_fwd(zero, k, v)
    np.testing.assert_allclose(o, prefix_mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(n), lse.shape), rtol=0, atol=1e-14)

    dq, dk, dv = impl.attn_bwd(zero, k, v, do)
    # dV_j = sum_{i >= j} dO_i / (i + 1): a reversed cumulative sum
    w = do / n[:, None]
    dv_ref = np.flip(np.cumsum(np.flip(w, axis=2), axis=2), axis=2)
    np.testing.assert_allclose(dv, dv_ref, rtol=0, atol=1e-13)
    assert np.all(dk == 0.0), "Q = 0 must give dK = 0 exactly"
    # dQ_i = scale/(i+1) * sum_{j<=i} (<dO_i, v_j> - <dO_i, O_i>) k_j
    g = np.einsum("bhid,bhjd->bhij", do, v)                # <dO_i, v_j>
    delta = np.einsum("bhid,bhid->bhi", do, prefix_mean)
    tril = np.tril(np.ones((T, T)))
    ds = (g - delta[..., None]) * tril / n[:, None]
    dq_ref = scale * np.einsum("bhij,bhjd->bhid", ds, k)
    np.testing.assert_allclose(dq, dq_ref, rtol=0, atol=1e-13)

    # K = 0: the same uniform weights; dQ = 0 exactly, dK by the transposed sum
    q = r.standard_normal((B, H, T, D))
    o2, lse2 = impl.attn_fwd(q, zero, v)
    np.testing.assert_allclose(o2, prefix_mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, np.broadcast_to(np.log(n), lse2.shape), rtol=0, atol=1e-14)
    dq2, dk2, dv2 = impl.attn_bwd(q, zero, v, do)
    assert np.all(dq2 == 0.0), "K = 0 must give dQ = 0 exactly"
    np.testing.assert_allclose(dv2, dv_ref, rtol=0, atol=1e-13)
    dk_ref = scale * np.einsum("bhij,bhid->bhjd", ds, q)
    np.testing.assert_allclose(dk2, dk_ref, rtol=0, atol=1e-13)


def check_causality(impl, seed=3):
    r = _rng(seed)
    B, H, T, D = 1, 3, 13, 4
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    o, lse = impl.attn_fwd(q, k, v)
    dq, _, _ = impl.attn_bwd(q, k, v, do)
    for t in (0, 5, T - 2):
        q2, k2, v2, do2 = (a.copy() for a in (q, k, v, do))
        for a in (q2, k2, v2, do2):
            a[:, :, t + 1:] += 10.0 * r.standard_normal(a[:, :, t + 1:].shape)
        o2, lse2 = impl.attn_fwd(q2, k2, v2)
        dq2, _, _ = impl.attn_bwd(q2, k2, v2, do2)
        assert np.array_equal(o2[:, :, :t + 1], o[:, :, :t + 1]), f"O_<= {t} saw the future"
        assert np.array_equal(lse2[:, :, :t + 1], lse[:, :, :t + 1]), f"lse_<= {t} saw the future"
        assert np.array_equal(dq2[:, :, :t + 1], dq[:, :, :t + 1]), f"dQ_<= {t} saw the future"
        assert not np.array_equal(o2[:, :, t + 1:], o[:, :, t + 1:])


def check_single_token(impl, seed=4):
    r = _rng(seed)
    B, H, T, D = 3, 2, 1, 7
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    scale = 1.0 / math.sqrt(D)
    o, lse = impl.attn_fwd(q, k, v)
    assert np.array_equal(o, v), "T = 1 must return V exactly"
    np.testing.assert_allclose(lse, scale * np.sum(q * k, -1), rtol=1e-15, atol=1e-15)
    dq, dk, dv = impl.attn_bwd(q, k, v, do)
    assert np.array_equal(dv, do), "T = 1 must give dV = dO"
    np.testing.assert_allclose(dq, 0.0, atol=1e-15)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)


def check_shift_invariance(impl, seed=5):
    r = _rng(seed)
    B, H, T, D = 2, 2, 9, 5
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    u = 4.0 * r.standard_normal((B, H, 1, D))
    scale = 1.0 / math.sqrt(D)
    o, lse = impl.attn_fwd(q, k, v)
    o2, lse2 = impl.attn_fwd(q, k + u, v)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse + scale * np.sum(q * u, -1), rtol=0, atol=1e-12)
    g, g2 = impl.attn_bwd(q, k, v, do), impl.attn_bwd(q, k + u, v, do)
    for a, b in zip(g, g2):
        np.testing.assert_allclose(b, a, rtol=0, atol=1e-12)


def check_finite_differences(impl, seed=6):
    r = _rng(seed)
    B, H, T, D = 1, 2, 5, 3
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    dq, dk, dv = impl.attn_bwd(q, k, v, do)

    def loss(q_, k_, v_):
        return float(np.sum(impl.attn_fwd(q_, k_, v_)[0] * do))

    h = 1e-6
    for which, grad in (("q", dq), ("k", dk), ("v", dv)):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[which][idx] += h
            lp = loss(args["q"], args["k"], args["v"])
            args[which][idx] -= 2 * h
            lm = loss(args["q"], args["k"], args["v"])
            fd[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(fd - grad) / max(np.linalg.norm(grad), 1e-300)
        assert err <= 1e-7, f"d{which}: finite differences disagree (rel {err:.2e})"


def check_torch_witness(impl, seed=7):
    import torch
    r = _rng(seed)
    B, H, T, D = 2, 3, 33, 16
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    to.backward(torch.tensor(do))
    o, lse = impl.attn_fwd(q, k, v)
    dq, dk, dv = impl.attn_bwd(q, k, v, do)
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=0, atol=1e-12)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)
    s = torch.tensor(q) @ torch.tensor(k).transpose(-1, -2) / math.sqrt(D)
    s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def check_golden(impl):
    for name in sorted(os.listdir(GOLDEN)):
        if not name.endswith(".json"):
            continue
        with open(os.path.join(GOLDEN, name)) as f:
            g = json.load(f)
        arr = lambda key: np.asarray(g[key], dtype=np.float64)[None, None]
        q, k, v = arr("q"), arr("k"), arr("v")
        causal = g.get("causal", True)
        o, lse = impl.attn_fwd(q, k, v, g.get("scale"), causal=causal)
        np.testing.assert_allclose(o[0, 0], np.asarray(g["o"]), rtol=0, atol=g["atol"], err_msg=name)
        np.testing.assert_allclose(lse[0, 0], np.asarray(g["lse"]), rtol=0, atol=g["atol"], err_msg=name)
        if "do" in g:
            dq, dk, dv = impl.attn_bwd(q, k, v, arr("do"), g.get("scale"), causal=causal)
            for key, got in (("dq", dq), ("dk", dk), ("dv", dv)):
                np.testing.assert_allclose(got[0, 0], np.asarray(g[key]), rtol=0, atol=g["atol"],
                                           err_msg=f"{name}:{key}")


def check_nc_probs_rows(impl, seed=11):
    r = _rng(seed)
    B, H, T, D = 2, 3, 17, 5
    q, k = r.standard_normal((B, H, T, D)), r.standard_normal((B, H, T, D)) * 3.0
    p = impl.attn_probs(q, k, causal=False)
    assert np.all(np.abs(p.sum(-1) - 1.0) <= 1e-14), "rows of P must sum to 1"
    assert np.all(p > 0.0), "without the mask every key gets a positive weight"


def check_nc_averaging(impl, seed=12):
    """Q = 0 (then K = 0) without the mask: uniform weights 1/T over all keys."""
    r = _rng(seed)
    B, H, T, D = 2, 2, 11, 6
    k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(3))
    scale = 1.0 / math.sqrt(D)
    mean = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
    zero = np.zeros_like(k)
    o, lse = impl.attn_fwd(zero, k, v, causal=False)
    np.testing.assert_allclose(o, mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, np.full(lse.shape, math.log(T)), rtol=0, atol=1e-14)
    dq, dk, dv = impl.attn_bwd(zero, k, v, do, causal=False)
    dv_ref = np.broadcast_to(do.sum(axis=2, keepdims=True) / T, dv.shape)
    np.testing.assert_allclose(dv, dv_ref, rtol=0, atol=1e-13)
    assert np.all(dk == 0.0), "Q = 0 must give dK = 0 exactly"
    g = np.einsum("bhid,bhjd->bhij", do, v)
    delta = np.einsum("bhid,bhid->bhi", do, mean)
    ds = (g - delta[..., None]) / T
    np.testing.assert_allclose(dq, scale * np.einsum("bhij,bhjd->bhid", ds, k), rtol=0, atol=1e-13)
    q = r.standard_normal((B, H, T, D))
    o2, lse2 = impl.attn_fwd(q, zero, v, causal=False)
    np.testing.assert_allclose(o2, mean, rtol=0, atol=1e-13)
    dq2, dk2, dv2 = impl.attn_bwd(q, zero, v, do, causal=False)
    assert np.all(dq2 == 0.0), "K = 0 must give dQ = 0 exactly"
    np.testing.assert_allclose(dv2, dv_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk2, scale * np.einsum("bhij,bhid->bhjd", ds, q), rtol=0, atol=1e-13)


def check_nc_permutation(impl, seed=13):
    """Without the mask nothing depends on position: relabelling the tokens by
    a permutation relabels O, lse, dQ, dK and dV the same way, and permuting
    only the key/value pairs changes nothing."""
    r = _rng(seed)
    B, H, T, D = 1, 2, 10, 4
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    perm = r.permutation(T)
    o, lse = impl.attn_fwd(q, k, v, causal=False)
    grads = impl.attn_bwd(q, k, v, do, causal=False)
    pq, pk, pv, pdo = (a[:, :, perm] for a in (q, k, v, do))
    o2, lse2 = impl.attn_fwd(pq, pk, pv, causal=False)
    np.testing.assert_allclose(o2, o[:, :, perm], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse[:, :, perm], rtol=0, atol=1e-13)
    for a, b in zip(grads, impl.attn_bwd(pq, pk, pv, pdo, causal=False)):
        np.testing.assert_allclose(b, a[:, :, perm], rtol=0, atol=1e-13)
    o3, lse3 = impl.attn_fwd(q, pk, pv, causal=False)
    np.testing.assert_allclose(o3, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse3, lse, rtol=0, atol=1e-13)


def check_nc_last_row_and_single_token(impl, seed=14):
    """The causal last row already sees every key, so both variants agree
    there; at T = 1 they agree everywhere."""
    r = _rng(seed)
    B, H, T, D = 2, 2, 9, 5
    q, k, v = (r.standard_normal((B, H, T, D)) for _ in range(3))
    o, lse = impl.attn_fwd(q, k, v)
    onc, lsenc = impl.attn_fwd(q, k, v, causal=False)
    np.testing.assert_allclose(onc[:, :, -1], o[:, :, -1], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lsenc[:, :, -1], lse[:, :, -1], rtol=0, atol=1e-14)
    assert not np.allclose(onc[:, :, 0], o[:, :, 0]), "row 0 must see the later keys"
    q1, k1, v1, do1 = (r.standard_normal((B, H, 1, D)) for _ in range(4))
    o1, _ = impl.attn_fwd(q1, k1, v1, causal=False)
    assert np.array_equal(o1, v1), "T = 1 must return V exactly"
    assert np.array_equal(impl.attn_bwd(q1, k1, v1, do1, causal=False)[2], do1)


def check_nc_shift_invariance(impl, seed=15):
    r = _rng(seed)
    B, H, T, D = 2, 2, 9, 5
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    u = 4.0 * r.standard_normal((B, H, 1, D))
    scale = 1.0 / math.sqrt(D)
    o, lse = impl.attn_fwd(q, k, v, causal=False)
    o2, lse2 = impl.attn_fwd(q, k + u, v, causal=False)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse + scale * np.sum(q * u, -1), rtol=0, atol=1e-12)
    g, g2 = impl.attn_bwd(q, k, v, do, causal=False), impl.attn_bwd(q, k + u, v, do, causal=False)
    for a, b in zip(g, g2):
        np.testing.assert_allclose(b, a, rtol=0, atol=1e-12)


def check_nc_finite_differences(impl, seed=16):
    r = _rng(seed)
    B, H, T, D = 1, 2, 5, 3
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    dq, dk, dv = impl.attn_bwd(q, k, v, do, causal=False)

    def loss(q_, k_, v_):
        return float(np.sum(impl.attn_fwd(q_, k_, v_, causal=False)[0] * do))

    h = 1e-6
    for which, grad in (("q", dq), ("k", dk), ("v", dv)):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[which][idx] += h
            lp = loss(args["q"], args["k"], args["v"])
            args[which][idx] -= 2 * h
            lm = loss(args["q"], args["k"], args["v"])
            fd[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(fd - grad) / max(np.linalg.norm(grad), 1e-300)
        assert err <= 1e-7, f"d{which}: finite differences disagree (rel {err:.2e})"


def check_nc_torch_witness(impl, seed=17):
    import torch
    r = _rng(seed)
    B, H, T, D = 2, 3, 33, 16
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=False)
    to.backward(torch.tensor(do))
    o, lse = impl.attn_fwd(q, k, v, causal=False)
    dq, dk, dv = impl.attn_bwd(q, k, v, do, causal=False)
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=0, atol=1e-12)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)
    s = torch.tensor(q) @ torch.tensor(k).transpose(-1, -2) / math.sqrt(D)
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


ALL_PINS = [check_probs_rows, check_averaging_trick, check_causality, check_single_token,
            check_shift_invariance, check_finite_differences, check_torch_witness, check_golden,
            check_nc_probs_rows, check_nc_averaging, check_nc_permutation,
            check_nc_last_row_and_single_token, check_nc_shift_invariance,
            check_nc_finite_differences, check_nc_torch_witness]


# ---------------------------------------------------------------- dropout

def _curand():
    """cuRAND's host-side generator (runs on the CPU, no GPU needed), or None."""
    import ctypes
    import glob
    paths = sorted(glob.glob("/usr/local/cuda/lib64/libcurand.so*"))
    try:
        import nvidia.curand
        paths += sorted(glob.glob(os.path.join(os.path.dirname(nvidia.curand.__file__), "lib",
                                               "libcurand.so*")))
    except ImportError:
        pass
    for path in paths:
        try:
            return ctypes.CDLL(path)
        except OSError:
            continue
    return None


def curand_philox_block(seed: int, block: int):
    """Four 32-bit outputs of cuRAND's host PHILOX4_32_10 generator at output
    offset 4 * block, under key (seed low word, seed high word).  Its host
    generator places output block b at counter words (b div 2^16 over words 0
    and 1, b mod 2^16, 0); see curand_block_of."""
    import ctypes
    lib = _curand()
    assert lib is not None
    g = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(g), 161) == 0   # PHILOX4_32_10
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(g, ctypes.c_ulonglong(seed)) == 0
        assert lib.curandSetGeneratorOffset(g, ctypes.c_ulonglong(4 * block)) == 0
        buf = (ctypes.c_uint32 * 4)()
        assert lib.curandGenerate(g, buf, ctypes.c_size_t(4)) == 0
        return [int(x) for x in buf]
    finally:
        lib.curandDestroyGenerator(g)


def curand_block_of(c0: int, c1: int, c2: int) -> int:
    """The cuRAND host output block holding counter (c0, c1, c2, 0), c2 < 2^16."""
    assert 0 <= c2 < (1 << 16) and c1 < (1 << 14)
    return (((c1 << 32) | c0) << 16) | c2


def _threshold(p):
    return int(math.floor(p * 65536.0 + 0.5))


def check_philox_against_curand(impl):
    import pytest
    if _curand() is None:
        pytest.skip("libcurand not found")
    for seed in (0, 1, 0xFFFFFFFF, (5 << 32) + 17, 0x123456789ABCDEF0):
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for ctr in ((0, 0, 0), (0, 0, 1), (1, 0, 0), (0, 1, 0), (12345, 0, 65535),
                    (0xFFFFFFFF, 0x3FFF, 0xFFFF), (0xDEADBEEF, 0x1234, 0x0F0F)):
            want = curand_philox_block(seed, curand_block_of(*ctr))
            got = impl.philox4x32_10(list(ctr) + [0], key)
            assert got == want, f"Philox4x32-10 differs from cuRAND (seed {seed:#x}, ctr {ctr})"


def check_dropout_mask_against_curand(impl):
    """Head bh at offset 0 uses counters (i, j / 8, bh, 0): its whole keep
    mask follows from cuRAND's outputs and the 16-bit split of the words."""
    import pytest
    if _curand() is None:
        pytest.skip("libcurand not found")
    T, p, seed = 40, 0.3, 0xC0FFEE
    t = _threshold(p)
    masks = impl.dropout_mask(1, 3, T, p, seed, 0)[0]
    for bh in (0, 2):
        for i in range(T):
            for g in range((T + 7) // 8):
                words = curand_philox_block(seed, curand_block_of(i, g, bh))
                for e in range(8):
                    j = 8 * g + e
                    if j < T:
                        u = (words[e >> 1] >> (16 * (e & 1))) & 0xFFFF
                        assert masks[bh, i, j] == (1 if u >= t else 0), f"mask {bh} ({i},{j}) differs"


def check_dropout_mask_statistics(impl):
    B, H, T = 2, 3, 256
    for p in (0.1, 0.5):
        m = impl.dropout_mask(B, H, T, p, seed=11, offset=3)
        n = m.size
        keep = 1.0 - _threshold(p) / 65536.0
        sigma = math.sqrt(n * keep * (1 - keep))
        assert abs(int(m.sum()) - n * keep) <= 5 * sigma, f"keep rate off for p={p}"
        assert np.array_equal(m, impl.dropout_mask(B, H, T, p, seed=11, offset=3))
        flat = m.reshape(B * H, T * T).astype(np.float64)
        for a, b in ((0, 1), (0, B * H - 1)):
            assert not np.array_equal(flat[a], flat[b]), "heads must get different masks"
        # neighbouring elements (same 16-bit word and across words) uncorrelated
        x = m.reshape(-1, T).astype(np.float64)
        c = np.corrcoef(x[:, :-1].ravel(), x[:, 1:].ravel())[0, 1]
        assert abs(c) < 0.01, f"neighbouring keep bits correlated ({c:.3f})"
    base = impl.dropout_mask(1, 2, 64, 0.5, seed=11, offset=3)
    assert not np.array_equal(base, impl.dropout_mask(1, 2, 64, 0.5, seed=11, offset=4))
    assert not np.array_equal(base, impl.dropout_mask(1, 2, 64, 0.5, seed=12, offset=3))
    assert not np.array_equal(base, impl.dropout_mask(1, 2, 64, 0.5, seed=11 + (1 << 32), offset=3))


def check_dropout_zero_threshold_is_plain(impl, seed=21):
    """p < 1/131072 rounds to threshold 0: every weight kept with scale 1, so
    the dropout path must give back the plain attention bit for bit."""
    r = _rng(seed)
    B, H, T, D = 2, 2, 19, 4
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    for causal in (True, False):
        o, lse = impl.attn_fwd(q, k, v, causal=causal)
        o2, lse2 = impl.attn_fwd(q, k, v, causal=causal, dropout_p=1e-6, seed=5, offset=1)
        assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
        for a, b in zip(impl.attn_bwd(q, k, v, do, causal=causal),
                        impl.attn_bwd(q, k, v, do, causal=causal, dropout_p=1e-6, seed=5, offset=1)):
            assert np.array_equal(a, b)


def check_dropout_uniform_closed_form(impl, seed=22):
    """Q = 0: the weights are uniform over the visible keys, so O_i is the keep
    scale times the mean over the visible keys of M_ij v_j; lse is unchanged."""
    r = _rng(seed)
    B, H, T, D = 2, 2, 23, 5
    k, v = r.standard_normal((B, H, T, D)), r.standard_normal((B, H, T, D))
    zero = np.zeros_like(k)
    p, sd, off = 0.25, 99, 7
    c = 65536.0 / (65536.0 - _threshold(p))
    m = impl.dropout_mask(B, H, T, p, sd, off).astype(np.float64)
    for causal in (True, False):
        vis = np.tril(np.ones((T, T))) if causal else np.ones((T, T))
        n = vis.sum(-1)
        o, lse = impl.attn_fwd(zero, k, v, causal=causal, dropout_p=p, seed=sd, offset=off)
        ref = c * np.einsum("bhij,bhjd->bhid", m * vis, v) / n[:, None]
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, np.broadcast_to(np.log(n), lse.shape), rtol=0, atol=1e-14)


def check_dropout_unbiased(impl, seed=23):
    """Over many seeds the dropped output and dV average to the plain ones."""
    r = _rng(seed)
    B, H, T, D = 1, 1, 6, 3
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    o_ref, _ = impl.attn_fwd(q, k, v, causal=False)
    dv_ref = impl.attn_bwd(q, k, v, do, causal=False)[2]
    N = 600
    os_, dvs = [], []
    for s in range(N):
        os_.append(impl.attn_fwd(q, k, v, causal=False, dropout_p=0.5, seed=s)[0])
        dvs.append(impl.attn_bwd(q, k, v, do, causal=False, dropout_p=0.5, seed=s)[2])
    for samples, ref, name in ((np.array(os_), o_ref, "O"), (np.array(dvs), dv_ref, "dV")):
        mean, sd = samples.mean(0), samples.std(0) + 1e-12
        z = np.abs(mean - ref) / (sd / math.sqrt(N))
        assert np.all(z < 5.0), f"E[{name}] with dropout differs from {name} (max z {z.max():.1f})"


def check_dropout_finite_differences(impl, seed=24):
    r = _rng(seed)
    B, H, T, D = 1, 2, 6, 3
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    kw = dict(dropout_p=0.3, seed=77, offset=2)
    for causal in (True, False):
        dq, dk, dv = impl.attn_bwd(q, k, v, do, causal=causal, **kw)

        def loss(q_, k_, v_):
            return float(np.sum(impl.attn_fwd(q_, k_, v_, causal=causal, **kw)[0] * do))

        h = 1e-6
        for which, grad in (("q", dq), ("k", dk), ("v", dv)):
            fd = np.zeros_like(grad)
            for idx in np.ndindex(*grad.shape):
                args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
                args[which][idx] += h
                lp = loss(args["q"], args["k"], args["v"])
                args[which][idx] -= 2 * h
                lm = loss(args["q"], args["k"], args["v"])
                fd[idx] = (lp - lm) / (2 * h)
            err = np.linalg.norm(fd - grad) / max(np.linalg.norm(grad), 1e-300)
            assert err <= 1e-7, f"dropout d{which} (causal={causal}): rel {err:.2e}"


def check_dropout_torch_witness(impl, seed=25):
    """torch float64 autograd of softmax -> keep mask * scale -> @ V."""
    import torch
    r = _rng(seed)
    B, H, T, D = 2, 2, 37, 8
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    p, sd, off = 0.2, 1234, 5
    c = 65536.0 / (65536.0 - _threshold(p))
    m = torch.tensor(impl.dropout_mask(B, H, T, p, sd, off), dtype=torch.float64)
    for causal in (True, False):
        tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
        s = tq @ tk.transpose(-1, -2) / math.sqrt(D)
        if causal:
            s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
        lse_t = torch.logsumexp(s, -1)
        o_t = (torch.softmax(s, -1) * m * c) @ tv
        o_t.backward(torch.tensor(do))
        o, lse = impl.attn_fwd(q, k, v, causal=causal, dropout_p=p, seed=sd, offset=off)
        np.testing.assert_allclose(o, o_t.detach().numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_t.detach().numpy(), rtol=0, atol=1e-12)
        grads = impl.attn_bwd(q, k, v, do, causal=causal, dropout_p=p, seed=sd, offset=off)
        for mine, ref in zip(grads, (tq.grad, tk.grad, tv.grad)):
            np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)


def check_dropout_head_subset(impl, seed=26):
    """A single head computed alone with head0 = its flat index matches that
    head of the full call (so sampled heads can be checked one by one)."""
    r = _rng(seed)
    B, H, T, D = 2, 3, 21, 4
    q, k, v, do = (r.standard_normal((B, H, T, D)) for _ in range(4))
    kw = dict(dropout_p=0.3, seed=5, offset=9)
    o, lse = impl.attn_fwd(q, k, v, **kw)
    g = impl.attn_bwd(q, k, v, do, **kw)
    for h in (0, 4, 5):
        b, hh = divmod(h, H)
        sl = lambda a: a[b:b + 1, hh:hh + 1]
        o1, lse1 = impl.attn_fwd(sl(q), sl(k), sl(v), head0=h, **kw)
        assert np.array_equal(o1, sl(o)) and np.array_equal(lse1, sl(lse))
        for a, b1 in zip(g, impl.attn_bwd(sl(q), sl(k), sl(v), sl(do), head0=h, **kw)):
            assert np.array_equal(b1, sl(a))


DROPOUT_PINS = [check_philox_against_curand, check_dropout_mask_against_curand,
                check_dropout_mask_statistics, check_dropout_zero_threshold_is_plain,
                check_dropout_uniform_closed_form, check_dropout_unbiased,
                check_dropout_finite_differences, check_dropout_torch_witness,
                check_dropout_head_subset]
ALL_PINS = ALL_PINS + DROPOUT_PINS


# ---------------------------------------------------------------- decode

def check_decode_rows_of_causal(impl, seed=31):
    """The Tq newest queries over Tk cached keys are exactly the last Tq rows
    of the causal attention over all Tk tokens (bit for bit: the same row
    computation), for every Tq from 1 to Tk."""
    r = _rng(seed)
    B, H, Tk, D = 2, 3, 13, 5
    q, k, v = (r.standard_normal((B, H, Tk, D)) for _ in range(3))
    o, lse = impl.attn_fwd(q, k, v)
    for tq in (1, 2, 5, Tk):
        od, lsed = impl.attn_decode(q[:, :, Tk - tq:], k, v)
        assert np.array_equal(od, o[:, :, Tk - tq:]), f"decode Tq={tq} differs from causal rows"
        assert np.array_equal(lsed, lse[:, :, Tk - tq:])


def check_decode_uniform_closed_form(impl, seed=32):
    """Q = 0: query r averages the values of keys 0 .. Tk - Tq + r."""
    r = _rng(seed)
    B, H, Tk, D, tq = 2, 2, 17, 4, 3
    k, v = r.standard_normal((B, H, Tk, D)), r.standard_normal((B, H, Tk, D))
    o, lse = impl.attn_decode(np.zeros((B, H, tq, D)), k, v)
    for rr in range(tq):
        n = Tk - tq + rr + 1
        np.testing.assert_allclose(o[:, :, rr], v[:, :, :n].mean(axis=2), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, rr], math.log(n), rtol=0, atol=1e-14)


def check_decode_torch_witness(impl, seed=33):
    import torch
    r = _rng(seed)
    B, H, Tk, D, tq = 2, 2, 40, 8, 4
    q = r.standard_normal((B, H, tq, D))
    k, v = r.standard_normal((B, H, Tk, D)), r.standard_normal((B, H, Tk, D))
    allowed = torch.arange(Tk)[None, :] <= (Tk - tq + torch.arange(tq))[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), attn_mask=allowed)
    o, _ = impl.attn_decode(q, k, v)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


DECODE_PINS = [check_decode_rows_of_causal, check_decode_uniform_closed_form,
               check_decode_torch_witness]
ALL_PINS = ALL_PINS + DECODE_PINS
