"""Seeded synthetic workloads: the five reference shapes and generic cases.

This module only draws numbers.  It holds none of the attention arithmetic, so
both the CUDA path and the float64 oracle can take their inputs from it.

Recipe (the same for every workload):
* one CPU ``torch.Generator`` seeded with ``seed`` (1000 + workload index for
  the named workloads);
* draw order: cached lengths (workloads with a cached prefix only), cache K,
  cache V, prompt (or chunk) q, k, v, then q, k, v of each decode step;
* values ``torch.randn`` in float32, rounded to bfloat16 (round-to-nearest-even);
  cached lengths ``randint(lo, hi + 1)``;
* cache capacity Lmax = the longest sequence the workload reaches, rounded up
  to a multiple of 128; every cache slot at or beyond a sequence's valid length
  holds the bfloat16 quiet-NaN pattern 0x7FC0, so a kernel that reads past the
  valid length poisons its output.

Shapes follow the models the pages describe: a 12-layer / 768-hidden / 8-head
decoder (head_dim 96), the 3.8B Llama-style model (24 query heads, 8 KV heads,
QK-norm, head_dim 128), and a 512-token prompt followed by 100 generated tokens.
A workload with both a cached prefix and T > 0 is a continuation chunk: T new
tokens per sequence starting at position lens[b].
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

BF16_QNAN_BITS = 0x7FC0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    Hq: int
    Hkv: int
    D: int
    T: int                      # new tokens: a prompt from 0, or a chunk after the cache
    decode_steps: int           # single-token steps after the prompt
    qk_norm: bool
    cached_len_range: Optional[tuple] = None   # cached prefix: lens ~ U[lo, hi]
    rope_base: float = 10000.0
    eps: float = 1e-6

    def __post_init__(self):
        # Configuration assertions before any run (page "750美元从零训练3个LLM",
        # item "用断言检查配置": the query-head count must divide into KV groups).
        assert self.Hkv >= 1 and self.Hq % self.Hkv == 0, "Hq must be a multiple of Hkv"
        assert self.D in (64, 96, 128), "head_dim must be 64, 96 or 128"
        assert self.B >= 1 and self.T >= 0 and self.decode_steps >= 0

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def max_len(self) -> int:
        if self.cached_len_range is not None:
            return self.cached_len_range[1] + self.T + self.decode_steps
        return self.T + self.decode_steps

    @property
    def Lmax(self) -> int:
        return round_up(self.max_len, 128)


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


WORKLOADS = [
    Workload("tiny_gqa", 0, B=1, Hq=4, Hkv=2, D=64, T=128, decode_steps=16, qk_norm=False),
    Workload("mha_prefill", 1, B=8, Hq=8, Hkv=8, D=96, T=1024, decode_steps=0, qk_norm=False),
    Workload("generation", 2, B=1, Hq=16, Hkv=4, D=64, T=512, decode_steps=100, qk_norm=False),
    Workload("prefill_3p8b", 3, B=8, Hq=24, Hkv=8, D=128, T=2048, decode_steps=0, qk_norm=True),
    Workload("batched_decode", 4, B=64, Hq=24, Hkv=8, D=128, T=0, decode_steps=1, qk_norm=True,
             cached_len_range=(256, 2048)),
    # continuation chunk: 1024 new tokens after cached prefixes of 512 .. 1536
    Workload("chunked_prefill_3p8b", 5, B=8, Hq=24, Hkv=8, D=128, T=1024, decode_steps=0,
             qk_norm=True, cached_len_range=(512, 1536)),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def _randn_bf16(g: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(w: Workload, decode_steps: Optional[int] = None, seed: Optional[int] = None,
                Lmax: Optional[int] = None) -> dict:
    """Draw one workload's inputs on the CPU (bfloat16 unless noted).

    Returns a dict with
      lens     int32 [B]   cached lengths (workloads with a prefix) or None
      k_cache, v_cache     [B, Hkv, Lmax, D]: random in slots < lens, NaN after
      q, k, v              prompt projections [B, T, H, D] (None when T == 0)
      steps                list of (q [B, Hq, D], k [B, Hkv, D], v [B, Hkv, D])
    """
    steps_n = w.decode_steps if decode_steps is None else decode_steps
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    L = w.Lmax if Lmax is None else Lmax
    out = {"lens": None, "q": None, "k": None, "v": None, "steps": []}
    if w.cached_len_range is not None:
        lo, hi = w.cached_len_range
        lens = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
        kc = _randn_bf16(g, w.B, w.Hkv, L, w.D)
        vc = _randn_bf16(g, w.B, w.Hkv, L, w.D)
        slot = torch.arange(L).view(1, 1, L, 1)
        dead = slot >= lens.view(-1, 1, 1, 1).to(torch.int64)
        kc.masked_fill_(dead, float("nan"))
        vc.masked_fill_(dead, float("nan"))
        out["lens"] = lens
    else:
        kc = torch.full((w.B, w.Hkv, L, w.D), float("nan"), dtype=torch.bfloat16)
        vc = torch.full((w.B, w.Hkv, L, w.D), float("nan"), dtype=torch.bfloat16)
    out["k_cache"], out["v_cache"] = kc, vc
    if w.T > 0:
        out["q"] = _randn_bf16(g, w.B, w.T, w.Hq, w.D)
        out["k"] = _randn_bf16(g, w.B, w.T, w.Hkv, w.D)
        out["v"] = _randn_bf16(g, w.B, w.T, w.Hkv, w.D)
    for _ in range(steps_n):
        out["steps"].append((_randn_bf16(g, w.B, w.Hq, w.D),
                             _randn_bf16(g, w.B, w.Hkv, w.D),
                             _randn_bf16(g, w.B, w.Hkv, w.D)))
    return out


def custom(name: str, B: int, Hq: int, Hkv: int, D: int, T: int = 0, decode_steps: int = 0,
           qk_norm: bool = False, cached_len_range=None, seed_index: int = 50) -> Workload:
    """A workload of arbitrary shape for parity cases (ragged tails, edge cases)."""
    return Workload(name, seed_index, B=B, Hq=Hq, Hkv=Hkv, D=D, T=T,
                    decode_steps=decode_steps, qk_norm=qk_norm,
                    cached_len_range=cached_len_range)


def packed_doc_ids(B: int, T: int, mean_len: float, seed: int) -> torch.Tensor:
    """Document ids [B, T] (int32, non-decreasing along each row) of documents
    packed back to back, lengths 1 + an exponential draw of the given mean (the
    last document cut at T): many short documents and a few long ones."""
    g = torch.Generator().manual_seed(seed)
    ids = torch.empty(B, T, dtype=torch.int32)
    for b in range(B):
        t, d = 0, 0
        while t < T:
            n = 1 + int(torch.empty(1).exponential_(1.0 / mean_len, generator=g).item())
            ids[b, t:t + n] = d
            t += n
            d += 1
    return ids


def bits(t: torch.Tensor):
    """bfloat16 tensor -> numpy uint16 bit patterns (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
