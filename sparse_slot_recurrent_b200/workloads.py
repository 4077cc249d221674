"""Seeded synthetic inputs for the RAM-Net layer core.

This module is the one piece shared by the CUDA path's tests/bench and the CPU oracle:
it only draws random tensors.  It holds none of the method's arithmetic (no address
decoding, no update, no normalisation), so neither side can borrow the other's.

Shapes stand in for the RAM-Net pages' 340M and 1.3B layers (M = 1024 slots, d_v = 128
per head; Top-8/16/32 as in the results paragraph of the project page) and for a batched
decode step.  No dataset is involved.

Draw order for one call (fp32, from a single ``torch.Generator`` seeded with ``seed``):
k_logits, q_logits, v, gamma_pre, z_pre, then (mixed-logit workloads only) the per
token-head peaked/flat mask, then (decode workloads only) the initial state S0, m0.
Gates are sigmoid(N(0,1)); the write gate goes in as the activated g in [0,1].
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

__all__ = ["Workload", "WORKLOADS", "generate", "generate_decode_state"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int                  # tokens per sequence (prefill) or decode steps (decode)
    d_p: int
    U: int
    K: int
    d_v: int
    in_dtype: torch.dtype   # dtype of logits / v / g / z as handed to the layer
    cape: bool              # CAPE on for every head
    logit_std: float = 1.0
    mixed_p: float = 0.0    # >0: Bernoulli(mixed_p) per token-head picks peaked_std, else flat_std
    peaked_std: float = 4.0
    flat_std: float = 0.1
    decode: bool = False    # one token per (b,h) per step, state resident in HBM
    ring: int = 16          # decode: number of distinct pre-generated input steps

    @property
    def M(self) -> int:
        return self.d_p ** self.U

    @property
    def L(self) -> int:
        return self.d_p * self.U

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # all-fp32 parity case
    "tiny": Workload("tiny", B=1, H=1, T=256, d_p=4, U=5, K=8, d_v=16,
                     in_dtype=torch.float32, cape=True, logit_std=1.0),
    # 340M-like layer, Top-8 prefill
    "prefill_340m_top8": Workload("prefill_340m_top8", B=8, H=8, T=4096, d_p=4, U=5, K=8, d_v=128,
                                  in_dtype=torch.bfloat16, cape=False, logit_std=1.5),
    # 340M-like layer, Top-32 prefill with 70% peaked / 30% near-flat logits (ties, collisions)
    "prefill_340m_top32": Workload("prefill_340m_top32", B=8, H=8, T=8192, d_p=4, U=5, K=32,
                                   d_v=128, in_dtype=torch.bfloat16, cape=False, mixed_p=0.7),
    # 1.3B-like layer, Top-16 long-context prefill
    "prefill_1p3b_top16": Workload("prefill_1p3b_top16", B=4, H=16, T=16384, d_p=4, U=5, K=16,
                                   d_v=128, in_dtype=torch.bfloat16, cape=True, logit_std=1.5),
    # batched decode step, state pre-filled and resident in HBM, 1024 consecutive steps
    "decode_b256": Workload("decode_b256", B=256, H=16, T=1024, d_p=8, U=4, K=16, d_v=128,
                            in_dtype=torch.bfloat16, cape=True, logit_std=1.5, decode=True),
}


def generate(w: Workload, seed: int = 0, device: str | torch.device = "cpu") -> dict:
    """Per-token inputs of a workload.

    Prefill: k_logits, q_logits [B,T,H,L]; v, z [B,T,H,d_v]; g [B,T,H].
    Decode: the same with T replaced by the ring length (steps cycle through the ring).
    Also returns cape_mask [H] uint8 and pos0 [B] int32 (zeros).  All tensors are
    contiguous, in ``w.in_dtype`` (masks/positions excepted), on ``device``.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T = w.ring if w.decode else w.T
    shp_l = (w.B, T, w.H, w.L)
    shp_v = (w.B, T, w.H, w.d_v)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    k = torch.randn(shp_l, **f32)
    q = torch.randn(shp_l, **f32)
    v = torch.randn(shp_v, **f32)
    gamma = torch.randn((w.B, T, w.H), **f32)
    zpre = torch.randn(shp_v, **f32)
    if w.mixed_p > 0:
        peaked = torch.rand((w.B, T, w.H, 1), **f32) < w.mixed_p
        std = torch.where(peaked, torch.tensor(w.peaked_std, device=device),
                          torch.tensor(w.flat_std, device=device))
        k = k * std
        q = q * std
    else:
        k = k * w.logit_std
        q = q * w.logit_std
    out = dict(
        k_logits=k.to(w.in_dtype).contiguous(),
        q_logits=q.to(w.in_dtype).contiguous(),
        v=v.to(w.in_dtype).contiguous(),
        g=torch.sigmoid(gamma).to(w.in_dtype).contiguous(),
        z=torch.sigmoid(zpre).to(w.in_dtype).contiguous(),
        cape_mask=torch.full((w.H,), 1 if w.cape else 0, dtype=torch.uint8, device=device),
        pos0=torch.zeros((w.B,), dtype=torch.int32, device=device),
    )
    out["_gen"] = gen
    return out


def generate_decode_state(w: Workload, gen: torch.Generator, device="cpu"):
    """Initial decode state: S0 ~ N(0,1) [B,H,M,d_v] fp32 and m0 ~ U[0.5, 2] [B,H,M] fp32,
    drawn after the per-token inputs from the same generator."""
    S0 = torch.randn((w.B, w.H, w.M, w.d_v), dtype=torch.float32, device=device, generator=gen)
    m0 = torch.rand((w.B, w.H, w.M), dtype=torch.float32, device=device, generator=gen) * 1.5 + 0.5
    return S0, m0
