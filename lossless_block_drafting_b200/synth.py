"""Seeded synthetic inputs for the decode-step hot path.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic (no attention, no logits, no consensus).  Both the CUDA
path's tests/benchmark and the CPU oracle read inputs made here, so they see
the same bits.  All draws happen on the CPU from explicit seeds: fp32 normals
from a ``torch.Generator`` rounded to bf16, integers from numpy's PCG64.

Shapes follow Qwen3-8B's attention and LM head (32 query / 8 KV heads,
head_dim 128, hidden 4096, vocab 151936) because the pages evaluate Orthrus on
the Qwen3 family; no trained weights are used or needed.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

QWEN3_8B = dict(n_q_heads=32, n_kv_heads=8, head_dim=128, hidden=4096, vocab=151936,
                layers=36)


def normal_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from a seeded CPU generator, rounded to bf16."""
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def normal_f32(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    return x.mul_(std) if std != 1.0 else x


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(int(seed))


def ctx_lens_uniform(B: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """B committed lengths uniform on the integers [lo, hi]."""
    return rng(seed).integers(lo, hi + 1, size=B).astype(np.int32)


def accept_geometric(n: int, p: float, cap: int, seed: int) -> np.ndarray:
    """a = min(G - 1, cap), G ~ Geometric(p) on {1, 2, ...} (mean about 1/p - 1)."""
    g = rng(seed).geometric(p, size=n)
    return np.minimum(g - 1, cap).astype(np.int32)


def accept_uniform(n: int, K: int, seed: int) -> np.ndarray:
    """a uniform on {0, ..., K}."""
    return rng(seed).integers(0, K + 1, size=n).astype(np.int32)


def plant_draft(target: np.ndarray, accept: np.ndarray, vocab: int, seed: int) -> np.ndarray:
    """Draft tokens that agree with ``target`` on exactly the first accept[b] slots.

    target [B, K] int token ids.  Slot a (if a < K) gets a different token,
    (target + 1 + U{0..vocab-2}) mod vocab; later slots are uniform random.
    """
    target = np.asarray(target, np.int64)
    B, K = target.shape
    r = rng(seed)
    draft = r.integers(0, vocab, size=(B, K))
    for b in range(B):
        a = int(accept[b])
        draft[b, :a] = target[b, :a]
        if a < K:
            draft[b, a] = (target[b, a] + 1 + r.integers(0, vocab - 1)) % vocab
    return draft.astype(np.int32)


@dataclass
class AttnCase:
    """One block-attention problem: Q [B,K,Hq,d], caches [B,Hkv,cap,d], lengths [B]."""
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    ctx_lens: np.ndarray
    K: int

    @property
    def shape(self):
        B, K, Hq, d = self.q.shape
        return dict(B=B, K=K, Hq=Hq, Hkv=self.k_cache.shape[1], cap=self.k_cache.shape[2], d=d)


def attn_case(B: int, K: int, Hq: int, Hkv: int, d: int, ctx_lens, cap: int | None = None,
              seed: int = 0, poison: float | None = float("nan")) -> AttnCase:
    """Q and K/V caches ~ N(0,1) in bf16; cache slots at or beyond L_b + K hold ``poison``.

    Poisoning the unused tail (NaN by default) makes any read past the valid key
    range visible in the output.
    """
    ctx = np.asarray(ctx_lens, np.int32).reshape(B)
    need = int(ctx.max()) + K if B else K
    cap = need if cap is None else int(cap)
    if cap < need:
        raise ValueError("cap smaller than max(ctx_lens) + K")
    q = normal_bf16((B, K, Hq, d), seed * 1000 + 1)
    kc = normal_bf16((B, Hkv, cap, d), seed * 1000 + 2)
    vc = normal_bf16((B, Hkv, cap, d), seed * 1000 + 3)
    if poison is not None:
        for b in range(B):
            kc[b, :, int(ctx[b]) + K:, :] = poison
            vc[b, :, int(ctx[b]) + K:, :] = poison
    return AttnCase(q, kc, vc, ctx, K)


def lmhead_case(R: int, H: int, V: int, seed: int = 0, w_std: float = 0.02):
    """Hidden states h ~ N(0,1) [R,H] and LM-head weights W ~ N(0, w_std^2) [V,H], bf16."""
    h = normal_bf16((R, H), seed * 1000 + 11)
    W = normal_bf16((V, H), seed * 1000 + 12, std=w_std)
    return h, W
