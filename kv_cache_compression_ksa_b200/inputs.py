"""Seeded synthetic inputs, shared by the tests, the smoke check and the
benchmark.  This module draws random tensors of the right shapes and nothing
else: it holds none of the attention arithmetic and imports neither the CUDA
binding nor the oracle.

Workloads (Qwen3-4B-class shapes, bf16, N(0, 1) times a scale):
  text Q/K/V   [sum n_b, H, d]     summary Q/K/V  [sum floor(n_b/k), H, d]
drawn in the order q_text, k_text, v_text, q_sum, k_sum, v_sum as fp32
standard normals from one torch.Generator, multiplied by `scale`, rounded to
bf16.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass
class PrefillInputs:
    seqlens: list
    k: int
    cu_seqlens: torch.Tensor   # int32 [B+1] (on `device`)
    q_text: torch.Tensor
    k_text: torch.Tensor
    v_text: torch.Tensor
    q_sum: torch.Tensor
    k_sum: torch.Tensor
    v_sum: torch.Tensor


def _randn(gen, shape, scale, device):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def prefill_inputs(seqlens, k, Hq, Hkv, d, seed=0, scale=1.0, device="cpu") -> PrefillInputs:
    """Packed text and per-chunk summary projections for a varlen batch.
    A sequence of n text tokens has floor(n/k) summary rows."""
    gen = torch.Generator(device=device).manual_seed(seed)
    nt = int(sum(seqlens))
    ns = int(sum(n // k for n in seqlens))
    qt = _randn(gen, (nt, Hq, d), scale, device)
    kt = _randn(gen, (nt, Hkv, d), scale, device)
    vt = _randn(gen, (nt, Hkv, d), scale, device)
    qs = _randn(gen, (ns, Hq, d), scale, device)
    ks = _randn(gen, (ns, Hkv, d), scale, device)
    vs = _randn(gen, (ns, Hkv, d), scale, device)
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    return PrefillInputs(list(seqlens), k, cu.to(device), qt, kt, vt, qs, ks, vs)


def token_stream(n_text, k, Hq, Hkv, d, seed=0, scale=1.0, device="cpu"):
    """Per-token decode inputs of one sequence: text q/k/v [n, H, d] and the
    summary q/k/v [floor(n/k), H, d] of each completed chunk."""
    p = prefill_inputs([n_text], k, Hq, Hkv, d, seed=seed, scale=scale, device=device)
    return p.q_text, p.k_text, p.v_text, p.q_sum, p.k_sum, p.v_sum


def uniform_ints(n, lo, hi, seed, device="cpu"):
    """n integers uniform on [lo, hi] (inclusive)."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randint(lo, hi + 1, (n,), generator=gen).to(device)


def fill_normal_(t: torch.Tensor, seed: int, scale: float = 1.0):
    """Fill a (possibly huge) bf16 device tensor with N(0,1)*scale in slabs."""
    gen = torch.Generator(device=t.device).manual_seed(seed)
    flat = t.view(-1)
    step = 1 << 26
    for i in range(0, flat.numel(), step):
        j = min(flat.numel(), i + step)
        x = torch.randn(j - i, generator=gen, dtype=torch.float32, device=t.device)
        if scale != 1.0:
            x.mul_(scale)
        flat[i:j].copy_(x)
    return t
