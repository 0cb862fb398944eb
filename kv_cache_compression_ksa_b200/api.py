"""Tensor-level convenience calls over the C ABI (allocation of outputs and
workspaces with torch; every computation runs in libksa.so).

prefill(...)      RoPE + interleave + KSA prefill attention for a packed batch
KSAAttention      the same as a torch.autograd.Function (backward through
                  ksa_prefill_bwd and ksa_interleave_rope_bwd)
DecodeCache       the contiguous decode cache plus append / decode / chunked
                  prefill steps
MlaCache          the latent (MLA) cache plus append / decode steps
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib as L


@dataclass
class PrefillOut:
    o_aug: torch.Tensor        # [aug_rows, Hq, d] bf16
    lse: torch.Tensor | None   # [aug_rows, Hq] fp32
    q_aug: torch.Tensor
    k_aug: torch.Tensor
    v_aug: torch.Tensor


def aug_rows(p: L.ksa_params, seqlens) -> int:
    return L.ksa_aug_rows(p, seqlens)


def prefill(p: L.ksa_params, seqlens, cu_seqlens, q_text, k_text, v_text, q_sum, k_sum, v_sum,
            want_lse: bool = True, stream=None) -> PrefillOut:
    """Run ksa_interleave_rope then ksa_prefill_fwd on device tensors.

    seqlens: host list of text lengths (sizes the outputs); cu_seqlens: the
    same as a device int32 prefix array [B+1]."""
    dev = q_text.device
    B = len(seqlens)
    total_text = int(sum(seqlens))
    total_sum = int(sum(n // p.k for n in seqlens))
    rows = aug_rows(p, seqlens)
    Hq, Hkv, d = p.num_q_heads, p.num_kv_heads, p.head_dim
    q_aug = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    k_aug = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    v_aug = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    o_aug = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev) if want_lse else None
    ws = torch.empty(L.ksa_prefill_workspace_size(p, B, total_text), dtype=torch.uint8, device=dev)
    L.ksa_interleave_rope(p, cu_seqlens, total_text, total_sum, rows, q_text, k_text, v_text,
                          q_sum, k_sum, v_sum, q_aug, k_aug, v_aug, ws, stream=stream)
    L.ksa_prefill_fwd(p, cu_seqlens, total_text, rows, q_aug, k_aug, v_aug, o_aug, lse, ws, stream=stream)
    return PrefillOut(o_aug, lse, q_aug, k_aug, v_aug)


class KSAAttention(torch.autograd.Function):
    """KSA prefill attention with autograd, for training.

    forward(p, seqlens, cu_seqlens, q_text, k_text, v_text, q_sum, k_sum,
    v_sum) -> o_aug [aug_rows, Hq, d] bf16 in the augmented layout
    (include/ksa.h): ksa_interleave_rope + ksa_prefill_fwd, keeping the
    rotated q/k/v, O and LSE for the backward.  backward: ksa_prefill_bwd
    then ksa_interleave_rope_bwd give the gradients of the six projections.
    Padding rows of o_aug are unspecified and their incoming gradient is
    ignored.  Use: o = KSAAttention.apply(p, seqlens, cu, qt, kt, vt, qs, ks, vs).
    """

    @staticmethod
    def forward(ctx, p, seqlens, cu_seqlens, q_text, k_text, v_text, q_sum, k_sum, v_sum):
        out = prefill(p, seqlens, cu_seqlens, q_text, k_text, v_text, q_sum, k_sum, v_sum, want_lse=True)
        ctx.p = p
        ctx.seqlens = [int(n) for n in seqlens]
        ctx.save_for_backward(cu_seqlens, out.q_aug, out.k_aug, out.v_aug, out.o_aug, out.lse)
        ctx.in_shapes = [tuple(t.shape) for t in (q_text, k_text, v_text, q_sum, k_sum, v_sum)]
        return out.o_aug

    @staticmethod
    def backward(ctx, do_aug):
        cu, qa, ka, va, oa, lse = ctx.saved_tensors
        p, seqlens = ctx.p, ctx.seqlens
        dev = qa.device
        B = len(seqlens)
        total_text = sum(seqlens)
        total_sum = sum(n // p.k for n in seqlens)
        rows = qa.shape[0]
        do = do_aug.to(torch.bfloat16).contiguous()
        dqa, dka, dva = torch.empty_like(qa), torch.empty_like(ka), torch.empty_like(va)
        wsb = torch.empty(L.ksa_prefill_bwd_workspace_size(p, B, rows), dtype=torch.uint8, device=dev)
        L.ksa_prefill_bwd(p, cu, total_text, rows, qa, ka, va, oa, lse, do, dqa, dka, dva, wsb)
        grads = [torch.empty(sh, dtype=torch.bfloat16, device=dev) for sh in ctx.in_shapes]
        ws = torch.empty(L.ksa_prefill_workspace_size(p, B, total_text), dtype=torch.uint8, device=dev)
        L.ksa_interleave_rope_bwd(p, cu, total_text, total_sum, rows, dqa, dka, dva, *grads, ws)
        return (None, None, None, *grads)


class DecodeCache:
    """K/V cache [B, Hkv, slots, d] bf16 + state [B, 4] int32 (slot map of
    the report's Figure 4; see include/ksa.h)."""

    def __init__(self, p: L.ksa_params, batch: int, cap: int, device="cuda"):
        """cap: summary-buffer capacity (chunks) of every sequence."""
        self.p = p
        self.batch = batch
        self.cap = cap
        self.slots = L.ksa_cache_slots(p, cap)
        shape = (batch, p.num_kv_heads, self.slots, p.head_dim)
        self.k = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.v = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.state = torch.zeros(batch, 4, dtype=torch.int32, device=device)
        self.desc = L.make_cache(self.k, self.v, self.state, cap)

    def append(self, kind, k_new, v_new, stream=None):
        L.ksa_cache_append(self.p, self.desc, kind, k_new, v_new, stream=stream)

    def from_prefill(self, cu_seqlens, total_text: int, k_aug, v_aug, workspace, stream=None):
        """Fill the cache with the state a prefill of these sequences leaves
        (k_aug / v_aug: the rotated augmented K/V of ksa_interleave_rope)."""
        L.ksa_cache_from_prefill(self.p, self.desc, cu_seqlens, total_text, k_aug.shape[0], k_aug, v_aug, workspace,
                                 stream=stream)

    def chunk_workspace(self, total_text: int, total_sum: int):
        n = L.ksa_prefill_chunk_workspace_size(self.p, self.batch, total_text, total_sum)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=self.k.device)

    def prefill_chunk(self, cu_text, total_text: int, cu_sum, total_sum: int, q_text, k_text, v_text,
                      q_sum, k_sum, v_sum, ws=None, want_lse=True, stream=None):
        """Chunked prefill: attend a block of new tokens per sequence against
        the cache, then append them (ksa_prefill_chunk).  Returns
        (o_text, o_sum, lse_text, lse_sum)."""
        p = self.p
        dev = self.k.device
        o_t = torch.empty(total_text, p.num_q_heads, p.head_dim, dtype=torch.bfloat16, device=dev)
        o_s = torch.empty(total_sum, p.num_q_heads, p.head_dim, dtype=torch.bfloat16, device=dev)
        l_t = torch.empty(total_text, p.num_q_heads, dtype=torch.float32, device=dev) if want_lse else None
        l_s = torch.empty(total_sum, p.num_q_heads, dtype=torch.float32, device=dev) if want_lse else None
        if ws is None:
            ws = self.chunk_workspace(total_text, total_sum)
        L.ksa_prefill_chunk(p, self.desc, cu_text, total_text, cu_sum, total_sum, q_text, k_text, v_text, q_sum,
                            k_sum, v_sum, o_t, o_s, l_t, l_s, ws, stream=stream)
        return o_t, o_s, l_t, l_s

    def workspace(self, max_text: int):
        n = L.ksa_decode_workspace_size(self.p, self.batch, max_text)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=self.k.device)

    def decode(self, kind, q, max_text, ws=None, want_lse=True, stream=None):
        p = self.p
        o = torch.empty(self.batch, p.num_q_heads, p.head_dim, dtype=torch.bfloat16, device=q.device)
        lse = torch.empty(self.batch, p.num_q_heads, dtype=torch.float32, device=q.device) if want_lse else None
        if ws is None:
            ws = self.workspace(max_text)
        L.ksa_decode(p, self.desc, kind, q, o, lse, max_text, ws, stream=stream)
        return o, lse


class MlaCache:
    """Latent (MLA) cache [B, slots, d_c + d_r] bf16 + state [B, 4] int32 under
    the same slot map (include/ksa.h, ksa_mla_*)."""

    def __init__(self, p: L.ksa_mla_params, batch: int, cap: int, device="cuda"):
        self.p = p
        self.batch = batch
        self.cap = cap
        self.slots = L.ksa_mla_cache_slots(p, cap)
        self.latent = torch.zeros(batch, self.slots, p.kv_lora_rank + p.rope_dim, dtype=torch.bfloat16,
                                  device=device)
        self.state = torch.zeros(batch, 4, dtype=torch.int32, device=device)
        self.desc = L.make_mla_cache(self.latent, self.state, cap)

    def append(self, kind, x, stream=None):
        L.ksa_mla_cache_append(self.p, self.desc, kind, x, stream=stream)

    def workspace(self, max_text: int):
        n = L.ksa_mla_decode_workspace_size(self.p, self.batch, max_text)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=self.latent.device)

    def decode(self, kind, q, max_text, ws=None, want_lse=True, stream=None):
        p = self.p
        o = torch.empty(self.batch, p.num_heads, p.kv_lora_rank, dtype=torch.bfloat16, device=q.device)
        lse = torch.empty(self.batch, p.num_heads, dtype=torch.float32, device=q.device) if want_lse else None
        if ws is None:
            ws = self.workspace(max_text)
        L.ksa_mla_decode(p, self.desc, kind, q, o, lse, max_text, ws, stream=stream)
        return o, lse
