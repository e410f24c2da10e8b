"""Seeded synthetic inputs for causal attention, shared by the tests, the bench
and the oracle's checks.

This module only draws random numbers and shapes them; it holds none of the
attention arithmetic.  Both the CUDA path and the oracle receive the very same
bytes from here (bf16 values are upcast to float64 for the oracle).

The five workloads are the model shapes the nanoGPT pages train:

* tiny fp32 causal attention (B=4, T=8, 4 heads of 8) -- a unit-test size;
* the character-level GPT: "Model Architecture Nanogpt" skill card, Workflow 1
  config block (n_layer 6, n_head 6, n_embd 384, block_size 256, batch 64);
* a small-head GPT with 12 heads of 32 on 384 channels: "GPT da zero",
  table "Come funziona" (context 256, embedding 384, 12 heads of dimension 32);
* GPT-2 124M: skill card, Workflow 2 config block (12 layers, 12 heads, n_embd
  768, block_size 1024, batch 12, dropout 0.0);
* GPT-2 XL (n_head 25, n_embd 1600, block 1024), the largest checkpoint the
  pages load with ``from_pretrained``.

Input recipe (no dataset or trained weight is used anywhere):

* "iid" workloads: Q, K, V ~ N(0, 1) independently.
* "proj" workloads: x ~ N(0, 1) of shape [B, T, C] is layer-normalised over C
  (no affine, eps 1e-5), multiplied by a c_attn weight W ~ N(0, 0.02) of shape
  [C, 3C] (no bias), split into q | k | v along the last dim, each viewed as
  [B, T, H, D] and permuted to [B, H, T, D] contiguous.
* GPT-2 XL additionally multiplies exactly round(0.01 * B*H*T) rows of K,
  drawn without replacement, by 8 (stresses the softmax max subtraction).
* dO ~ N(0, 1e-2) (standard deviation 1e-2), except the tiny workload where
  dO ~ N(0, 1).
* Everything is drawn in float32 from ``torch.Generator`` seeded with
  ``seed + 1000 * workload_index + layer`` and then rounded to the workload's
  dtype (bf16 or kept float32).
* Decode (``make_decode_inputs``): the same Q, K, V of a workload; the Tq
  newest tokens' queries are Q's last Tq rows, and K and V of all T tokens
  are the kept keys and values (T plays Tk).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int          # position in WORKLOADS (enters the seed)
    name: str
    B: int
    H: int
    T: int
    D: int
    dtype: str          # "f32" or "bf16"
    recipe: str         # "iid" or "proj"
    layers: int = 1     # independent instances per bench step
    do_std: float = 1e-2
    k_outlier_frac: float = 0.0
    k_outlier_scale: float = 1.0

    @property
    def n_embd(self) -> int:
        return self.H * self.D

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def causal_pairs(self) -> int:
        """Attended (i, j) pairs, j <= i, over all heads of one instance."""
        return self.B * self.H * self.T * (self.T + 1) // 2

    def flops(self) -> int:
        """Algorithmic fwd+bwd FLOPs of one instance: 12*D per attended pair.

        4*D in the forward (Q K^T and P V), 8*D in the backward (dV, dP, dK,
        dQ); the causal half of the 12*L*H*Q*T per-token attention term of
        ``estimate_mfu`` (nanoGPT -- architecture page, section 4).
        """
        return 12 * self.D * self.causal_pairs()

    def fwd_flops(self) -> int:
        return 4 * self.D * self.causal_pairs()


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload(0, "tiny_f32", B=4, H=4, T=8, D=8, dtype="f32", recipe="iid", do_std=1.0),
        Workload(1, "char_gpt", B=64, H=6, T=256, D=64, dtype="bf16", recipe="proj"),
        Workload(2, "small_head", B=8, H=12, T=256, D=32, dtype="bf16", recipe="iid"),
        Workload(3, "gpt2_124m", B=12, H=12, T=1024, D=64, dtype="bf16", recipe="proj", layers=12),
        Workload(4, "gpt2_xl", B=4, H=25, T=1024, D=64, dtype="bf16", recipe="iid",
                 k_outlier_frac=0.01, k_outlier_scale=8.0),
    ]
}


def _proj_qkv(g: torch.Generator, B: int, H: int, T: int, D: int):
    C = H * D
    x = torch.randn(B, T, C, generator=g, dtype=torch.float32)
    w = torch.randn(C, 3 * C, generator=g, dtype=torch.float32) * 0.02
    x = torch.nn.functional.layer_norm(x, (C,), eps=1e-5)
    qkv = x @ w
    q, k, v = qkv.split(C, dim=2)
    shape = lambda t: t.reshape(B, T, H, D).permute(0, 2, 1, 3).contiguous()
    return shape(q), shape(k), shape(v)


def make_inputs(w: Workload, seed: int = 0, layer: int = 0,
                B: Optional[int] = None, H: Optional[int] = None,
                T: Optional[int] = None, D: Optional[int] = None,
                dtype: Optional[torch.dtype] = None) -> Dict[str, torch.Tensor]:
    """Q, K, V, dO on the CPU as contiguous [B, H, T, D] tensors of the
    workload's dtype (override any shape field for parity cases)."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    T = w.T if T is None else T
    D = w.D if D is None else D
    dtype = w.torch_dtype if dtype is None else dtype
    g = torch.Generator().manual_seed(seed + 1000 * w.index + layer)
    if w.recipe == "proj":
        q, k, v = _proj_qkv(g, B, H, T, D)
    else:
        q = torch.randn(B, H, T, D, generator=g, dtype=torch.float32)
        k = torch.randn(B, H, T, D, generator=g, dtype=torch.float32)
        v = torch.randn(B, H, T, D, generator=g, dtype=torch.float32)
    if w.k_outlier_frac > 0:
        n_rows = B * H * T
        n_pick = int(round(w.k_outlier_frac * n_rows))
        pick = torch.randperm(n_rows, generator=g)[:n_pick]
        k.view(n_rows, D)[pick] *= w.k_outlier_scale
    do = torch.randn(B, H, T, D, generator=g, dtype=torch.float32) * w.do_std
    return {name: t.to(dtype).contiguous() for name, t in
            (("q", q), ("k", k), ("v", v), ("do", do))}


def make_inputs_packed(w: Workload, seed: int = 0, layer: int = 0) -> Dict[str, torch.Tensor]:
    """The same values as make_inputs, laid out the way nanoGPT's attention
    sees them: "qkv" [B, T, 3C] (the c_attn output, q | k | v along the last
    dim) and "do_packed" [B, T, C] (the gradient arriving from c_proj), next to
    make_inputs' contiguous [B, H, T, D] "q", "k", "v", "do"."""
    inp = make_inputs(w, seed=seed, layer=layer)
    tm = lambda t: t.permute(0, 2, 1, 3).reshape(t.shape[0], t.shape[2], -1)
    qkv = torch.cat([tm(inp["q"]), tm(inp["k"]), tm(inp["v"])], dim=2).contiguous()
    return {**inp, "qkv": qkv, "do_packed": tm(inp["do"]).contiguous()}


def packed_views(qkv: torch.Tensor, H: int):
    """[B, H, T, D] views of q, k, v inside a [B, T, 3C] tensor."""
    B, T, C3 = qkv.shape
    C = C3 // 3
    D = C // H
    return [qkv[:, :, i * C:(i + 1) * C].view(B, T, H, D).permute(0, 2, 1, 3) for i in range(3)]


def random_qkv(seed: int, B: int, H: int, T: int, D: int, dtype=torch.float32,
               std: float = 1.0, do_std: float = 1.0) -> Dict[str, torch.Tensor]:
    """Plain i.i.d. normal inputs of any shape (edge cases, ragged tails)."""
    g = torch.Generator().manual_seed(seed)
    out = {}
    for name, s in (("q", std), ("k", std), ("v", std), ("do", do_std)):
        out[name] = (torch.randn(B, H, T, D, generator=g, dtype=torch.float32) * s).to(dtype).contiguous()
    return out


def make_decode_inputs(w: Workload, tq: int, seed: int = 0, layer: int = 0) -> Dict[str, torch.Tensor]:
    """Decode inputs from the workload's Q, K, V: "q" [B, H, tq, D] = the last
    tq rows of Q (the newest tokens), "k", "v" [B, H, T, D] all T tokens."""
    inp = make_inputs(w, seed=seed, layer=layer)
    return {"q": inp["q"][:, :, w.T - tq:].contiguous(), "k": inp["k"], "v": inp["v"]}
