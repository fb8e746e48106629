"""Seeded synthetic inputs for Dynamic Bifocal RoPE attention.

This module draws random numbers and nothing else: it holds no part of the
attention method (no RoPE, no position map, no softmax). Both the CUDA path and
the CPU oracle receive tensors made here.

Input recipe
------------
The attention entry points take Q and K *already rotated by standard RoPE at
their absolute position* (the form a model's KV cache stores them in), and an
unrotated V.  A standard RoPE rotation is orthogonal, so if the raw projections
are i.i.d. N(0, 1) then so are their rotated images.  The synthetic inputs are
therefore drawn directly in the rotated frame: Q~, K~ and V are i.i.d. N(0, 1)
float32 draws from a seeded CPU ``torch.Generator``, then rounded to the run's
dtype (bf16 by round-to-nearest-even, or kept as fp32).

Seeds: Q~ = 1000 + w, K~ = 2000 + w, V = 3000 + w where w is the workload id
below; the decode query of step t uses seed 4000 + t.

Workloads (Qwen3 attention shapes, packed "thd" layout):

====================  =====================================================
name                  shape
====================  =====================================================
tiny_fp32             1 seq, L=1024, Hq=2, Hkv=1, D=64, w_pre=256 (G=4),
                      w0=64, theta=1e4, fp32
prefill_32k_g1        1 seq, L=32768, 16/8 heads, D=128, w_pre=32768 (G=1),
                      w0=4096, theta=1e6, bf16
prefill_128k_g4       1 seq, L=131072, 32/8 heads, D=128, w_pre=32768 (G=4),
                      w0=4096, theta=1e6, bf16
decode_128k           1 seq, cache of 131072 (+255) tokens, 32/8 heads,
                      D=128, 256 steps with L = 131072 + t, bf16
varlen_4seq           4 seqs {16384, 40000, 65536, 100000}, 32/8 heads,
                      D=128, w_pre=32768 (G = 1, 2, 2, 4), bf16
====================  =====================================================
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    seqlens: tuple
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    w_pretrained: int
    w0: int
    rope_theta: float
    dtype: str  # "bf16" | "fp32"
    decode_steps: int = 0  # > 0: a decode workload over a cache of seqlens[0] tokens

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def cu_seqlens(self) -> torch.Tensor:
        cu = [0]
        for s in self.seqlens:
            cu.append(cu[-1] + int(s))
        return torch.tensor(cu, dtype=torch.int32)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny_fp32", 1, (1024,), 2, 1, 64, 256, 64, 1.0e4, "fp32"),
        Workload("prefill_32k_g1", 2, (32768,), 16, 8, 128, 32768, 4096, 1.0e6, "bf16"),
        Workload("prefill_128k_g4", 3, (131072,), 32, 8, 128, 32768, 4096, 1.0e6, "bf16"),
        Workload("decode_128k", 4, (131072,), 32, 8, 128, 32768, 4096, 1.0e6, "bf16",
                 decode_steps=256),
        Workload("varlen_4seq", 5, (16384, 40000, 65536, 100000), 32, 8, 128, 32768, 4096,
                 1.0e6, "bf16"),
    )
}


def normal(shape, seed: int, dtype=torch.float32) -> torch.Tensor:
    """i.i.d. N(0,1) float32 draws from a CPU generator seeded with ``seed``,
    rounded to ``dtype``."""
    g = torch.Generator("cpu")
    g.manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    return x if dtype == torch.float32 else x.to(dtype)


def prefill_inputs(w: Workload, wid: int | None = None):
    """Packed prefill inputs (CPU tensors): q [T,Hq,D], k [T,Hkv,D], v [T,Hkv,D],
    cu_seqlens int32 [B+1]."""
    wid = w.wid if wid is None else wid
    T, D = w.total_tokens, w.head_dim
    q = normal((T, w.n_q_heads, D), 1000 + wid, w.torch_dtype)
    k = normal((T, w.n_kv_heads, D), 2000 + wid, w.torch_dtype)
    v = normal((T, w.n_kv_heads, D), 3000 + wid, w.torch_dtype)
    return q, k, v, w.cu_seqlens()


def decode_cache(w: Workload, batch: int = 1, wid: int | None = None):
    """Decode KV cache (CPU tensors) [B, Lcap, Hkv, D] with Lcap = seqlens[0] +
    decode_steps - 1, so that every step's new token is already in place."""
    wid = w.wid if wid is None else wid
    cap = w.seqlens[0] + max(w.decode_steps, 1) - 1
    shape = (batch, cap, w.n_kv_heads, w.head_dim)
    k = normal(shape, 2000 + wid, w.torch_dtype)
    v = normal(shape, 3000 + wid, w.torch_dtype)
    return k, v


def decode_query(w: Workload, step: int, batch: int = 1) -> torch.Tensor:
    """Decode query of step ``step``: [B, Hq, D]."""
    return normal((batch, w.n_q_heads, w.head_dim), 4000 + step, w.torch_dtype)


def random_case(seed: int, seqlens, n_q_heads: int, n_kv_heads: int, head_dim: int,
                dtype=torch.float32):
    """Small packed case with its own seed (for edge-case tests)."""
    T = int(sum(seqlens))
    q = normal((T, n_q_heads, head_dim), seed * 7 + 1, dtype)
    k = normal((T, n_kv_heads, head_dim), seed * 7 + 2, dtype)
    v = normal((T, n_kv_heads, head_dim), seed * 7 + 3, dtype)
    cu = [0]
    for s in seqlens:
        cu.append(cu[-1] + int(s))
    return q, k, v, torch.tensor(cu, dtype=torch.int32)
