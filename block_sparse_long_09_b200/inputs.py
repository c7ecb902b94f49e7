"""Seeded synthetic inputs for one QSA layer (prefill and decode).

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle
consume what it returns, so it is the one piece of code they share.

Recipe (fixed draw order from one ``torch.Generator`` seeded with ``seed``):
q, k, v, q_idx, k_idx, w, then (only where the workload has them) per-block
offsets.  Activations are drawn in fp32 from N(0, 1) and cast to bf16 with
round-to-nearest-even; w is fp32 from U(0, 1).  Shapes follow the model table
of the Qwen3.8-Flash-Next reading notes (papers.chlience.com, "Model Summary":
24 query heads, 2 KV heads, head dim 256; indexer 4 query heads, 1 key head,
head dim 128; compression ratio 4, budget 512 micro-blocks).

The "peaked" variant adds one scalar c_b ~ N(0, 0.5^2) per micro-block of each
sequence to all r tokens x 128 dims of k_idx before the bf16 cast, so that
whole blocks score high or low together.

Decode inputs are packed caches: k/v ``[sum L_s, 2, 256]``, raw indexer keys
``[sum L_s, 128]`` and one query per sequence.  The lengths fix every shape, so
they come first, uniform on ``[len_lo, len_hi]`` from a CPU generator seeded
with ``seed``; the tensors then follow in the order above from a generator
seeded with ``seed + 1``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

N_HEADS_Q = 24
N_HEADS_KV = 2
HEAD_DIM = 256
N_HEADS_IDX = 4
IDX_DIM = 128
R = 4
BUDGET_BLOCKS = 512


@dataclasses.dataclass
class PrefillInputs:
    q: torch.Tensor          # [total_q, 24, 256] bf16
    k: torch.Tensor          # [total_k, 2, 256] bf16
    v: torch.Tensor          # [total_k, 2, 256] bf16
    q_idx: torch.Tensor      # [total_q, 4, 128] bf16
    k_idx: torch.Tensor      # [total_k, 128] bf16
    w: torch.Tensor          # [total_q, 4] fp32
    seqlens: list            # per sequence length (L_q = L_k for prefill)
    cu_seqlens: torch.Tensor  # int32 [B+1]
    cu_blocks: torch.Tensor   # int32 [B+1], prefix sums of floor(L_s / r)
    r: int = R


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor          # [B, 24, 256] bf16 (one new token per sequence), [B, next_n, 24, 256] for next_n > 1
    k_cache: torch.Tensor    # [sum L_s, 2, 256] bf16, the new token's row included
    v_cache: torch.Tensor    # [sum L_s, 2, 256] bf16
    q_idx: torch.Tensor      # [B, 4, 128] bf16
    k_idx: torch.Tensor      # [sum L_s, 128] bf16 (raw indexer keys of the cache)
    w: torch.Tensor          # [B, 4] fp32
    seqlens: list
    cu_seqlens_k: torch.Tensor  # int32 [B+1]
    cu_blocks: torch.Tensor     # int32 [B+1]
    r: int = R


def _randn_bf16(g: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


def _cu(lengths, device) -> torch.Tensor:
    out = [0]
    for L in lengths:
        out.append(out[-1] + int(L))
    return torch.tensor(out, dtype=torch.int32, device=device)


def make_prefill(seqlens, seed: int = 0, peaked: bool = False, device: str = "cpu",
                 r: int = R) -> PrefillInputs:
    """Prefill inputs for sequences of the given lengths (L_q = L_k = L_s)."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    total = int(sum(seqlens))
    q = _randn_bf16(g, (total, N_HEADS_Q, HEAD_DIM), device)
    k = _randn_bf16(g, (total, N_HEADS_KV, HEAD_DIM), device)
    v = _randn_bf16(g, (total, N_HEADS_KV, HEAD_DIM), device)
    q_idx = _randn_bf16(g, (total, N_HEADS_IDX, IDX_DIM), device)
    k_idx32 = torch.randn((total, IDX_DIM), generator=g, dtype=torch.float32, device=device)
    w = torch.rand((total, N_HEADS_IDX), generator=g, dtype=torch.float32, device=device)
    if peaked:
        start = 0
        for L in seqlens:
            nblk = (int(L) + r - 1) // r
            c = torch.randn((nblk,), generator=g, dtype=torch.float32, device=device) * 0.5
            off = c.repeat_interleave(r)[: int(L)]
            k_idx32[start:start + int(L)] += off[:, None]
            start += int(L)
    k_idx = k_idx32.to(torch.bfloat16)
    return PrefillInputs(q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx, w=w,
                         seqlens=[int(L) for L in seqlens],
                         cu_seqlens=_cu(seqlens, device),
                         cu_blocks=_cu([int(L) // r for L in seqlens], device), r=r)


def draw_decode_lengths(batch: int, len_lo: int, len_hi: int, seed: int) -> list:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return [int(x) for x in torch.randint(len_lo, len_hi + 1, (batch,), generator=g)]


def make_decode(batch: int, len_lo: int, len_hi: Optional[int] = None, seed: int = 0,
                device: str = "cpu", r: int = R, next_n: int = 1) -> DecodeInputs:
    """Decode inputs: one new query per sequence against packed bf16 caches (next_n > 1:
    q holds next_n new queries per sequence, [batch, next_n, 24, 256], the last of them
    the one whose indexer query q_idx and weights w are drawn).

    Lengths are U{len_lo..len_hi} (fixed length when len_hi is None or equal)."""
    if len_hi is None or len_hi == len_lo:
        seqlens = [int(len_lo)] * batch
    else:
        seqlens = draw_decode_lengths(batch, len_lo, len_hi, seed)
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed + 1)
    total = int(sum(seqlens))
    q = _randn_bf16(g, (batch, N_HEADS_Q, HEAD_DIM) if next_n == 1 else (batch, next_n, N_HEADS_Q, HEAD_DIM),
                    device)
    k = _randn_bf16(g, (total, N_HEADS_KV, HEAD_DIM), device)
    v = _randn_bf16(g, (total, N_HEADS_KV, HEAD_DIM), device)
    q_idx = _randn_bf16(g, (batch, N_HEADS_IDX, IDX_DIM), device)
    k_idx = _randn_bf16(g, (total, IDX_DIM), device)
    w = torch.rand((batch, N_HEADS_IDX), generator=g, dtype=torch.float32, device=device)
    return DecodeInputs(q=q, k_cache=k, v_cache=v, q_idx=q_idx, k_idx=k_idx, w=w,
                        seqlens=seqlens, cu_seqlens_k=_cu(seqlens, device),
                        cu_blocks=_cu([L // r for L in seqlens], device), r=r)
