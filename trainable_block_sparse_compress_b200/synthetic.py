"""Seeded synthetic inputs shaped like the long-context workloads of InfLLM v2.

This module only draws random numbers; it holds none of the method's arithmetic, so the
CPU oracle and the CUDA library can both be fed from it.

Recipe (one ``torch.Generator`` seeded with ``seed``, draws in this order):
  1. Q       ~ N(0, 1)                      prefill [B, L, Hq, d], decode [B, Hq, d]
  2. K noise ~ N(0, 1)                      [B, Hkv, Lmax, d]
  3. K block offsets ~ N(0, 0.5^2)          [B, Hkv, ceil(Lmax/64), d], one d-vector per
     (sequence, kv-head, 64-token block), added to every key row of its block
  4. V       ~ N(0, 1)                      [B, Hkv, Lmax, d]
  5. lens    ~ U{lo, ..., hi} (ragged decode only), [B] int32
Every float tensor is drawn in fp32 and rounded to bf16 (nearest even) once.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str  # "prefill" or "decode"
    batch: int
    seq_len: int  # prefill length, or the KV-cache capacity Lmax for decode
    num_q_heads: int
    num_kv_heads: int
    topk: int
    head_dim: int = 128
    block_size: int = 64
    kernel_size: int = 32
    kernel_stride: int = 16
    n_init: int = 1
    n_local: int = 2
    ragged: Optional[tuple] = None  # decode: (lo, hi) inclusive bounds of lens[b]
    offset_std: float = 0.5

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the long-context benchmark (block 64, kernel 32 / stride 16,
# 1 initial + 2 local blocks counted inside top-k).
WORKLOADS = {
    "prefill_2k": Workload("prefill_2k", "prefill", 1, 2048, 8, 1, 16),
    "decode_32k": Workload("decode_32k", "decode", 8, 32768, 32, 2, 96),
    "prefill_32k": Workload("prefill_32k", "prefill", 1, 32768, 32, 2, 96),
    "prefill_128k": Workload("prefill_128k", "prefill", 1, 131072, 32, 2, 96),
    "decode_ragged_128k": Workload("decode_ragged_128k", "decode", 32, 131072, 32, 2, 96,
                                   ragged=(65536, 131072)),
}


@dataclass
class Inputs:
    wl: Workload
    q: torch.Tensor  # bf16, CPU
    k: torch.Tensor
    v: torch.Tensor
    lens: Optional[torch.Tensor]  # int32 [B] for decode, None for prefill
    extra: dict = field(default_factory=dict)


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def make_inputs(wl: Workload, seed: int = 0) -> Inputs:
    g = torch.Generator().manual_seed(seed)
    B, L, Hq, Hkv, d = wl.batch, wl.seq_len, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
    if wl.mode == "prefill":
        q = _bf16(torch.randn((B, L, Hq, d), generator=g))
    else:
        q = _bf16(torch.randn((B, Hq, d), generator=g))
    nb = (L + wl.block_size - 1) // wl.block_size
    k = torch.randn((B, Hkv, L, d), generator=g)
    off = torch.randn((B, Hkv, nb, d), generator=g) * wl.offset_std
    k = k.view(B, Hkv, -1, d)
    k += off.repeat_interleave(wl.block_size, dim=2)[:, :, :L]
    k = _bf16(k)
    del off
    v = _bf16(torch.randn((B, Hkv, L, d), generator=g))
    lens = None
    if wl.mode == "decode":
        if wl.ragged is not None:
            lo, hi = wl.ragged
            lens = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
        else:
            lens = torch.full((B,), L, dtype=torch.int32)
    return Inputs(wl, q, k, v, lens)


def as_u16(t: torch.Tensor):
    """bf16 CPU tensor -> numpy uint16 bit patterns (no copy)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
