"""Random-weight fp64 toy transformer for the losslessness check of block drafting.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The gist.science summary of "Orthrus: Memory-Efficient Parallel Token Generation
via Dual-View Diffusion" (technical summary §2.1-2.3) describes a frozen AR
transformer plus an injected diffusion attention module whose q/k/v projections
are separate (the Hacker News thread "Orthrus-Qwen3: ..." post #26 names them
q/k/v/o_proj_diff) and which reads the same KV cache.  Inference per step:

1. diffusion pass over [anchor, <mask> x (K-1)] with the M_diff block mask
   (prefix + bidirectional block) -> K drafted tokens;
2. AR pass over [anchor, draft_0 .. draft_{K-2}] with the causal mask -> the
   AR greedy token at each of the K positions;
3. exact consensus: keep the longest prefix where draft == AR greedy, append
   the AR correction token, shorten the cache (move the length pointer).

The claim to check is losslessness (summary §2.3 item 3, §3; abstract): the
emitted tokens equal token-by-token greedy AR decoding, for any drafter.  This
module builds both decoders on one random-weight model in fp64 and lets the
tests compare them.  All attention, greedy choice, consensus and commit calls go
through the oracle's C functions; the model's own projections are numpy, applied
one row at a time so a row's arithmetic does not depend on how many rows are
processed together.

Readings where the pages are silent: block row i (position L+i) predicts the
token at position L+i+1; the new anchor is the last emitted token and is not
yet cached; the committed length advances by min(a+1, K).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import MASK_AR, MASK_DIFF, block_attn, kv_commit, row_argmax, verify


def _rows(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """x @ w computed one row at a time (row results independent of batch size)."""
    return np.stack([x[i] @ w for i in range(x.shape[0])]) if x.shape[0] else \
        np.zeros((0, w.shape[1]))


@dataclass
class ToyConfig:
    vocab: int = 64
    hidden: int = 32
    layers: int = 2
    n_q_heads: int = 2
    n_kv_heads: int = 1
    head_dim: int = 16
    max_pos: int = 512
    seed: int = 0


@dataclass
class ToyModel:
    cfg: ToyConfig
    p: dict = field(default_factory=dict)

    @classmethod
    def random(cls, cfg: ToyConfig) -> "ToyModel":
        rng = np.random.default_rng(cfg.seed)
        D, V = cfg.hidden, cfg.vocab
        qd = cfg.n_q_heads * cfg.head_dim
        kd = cfg.n_kv_heads * cfg.head_dim
        s = 1.0 / np.sqrt(D)
        p = {
            # one extra embedding row: the <mask> token id == vocab
            "emb": rng.normal(0, 1, (V + 1, D)),
            "pos": rng.normal(0, 0.5, (cfg.max_pos, D)),
            "lm": rng.normal(0, 1, (V, D)),
        }
        for li in range(cfg.layers):
            for view in ("ar", "diff"):
                p[f"{view}.wq.{li}"] = rng.normal(0, s, (D, qd))
                p[f"{view}.wk.{li}"] = rng.normal(0, s, (D, kd))
                p[f"{view}.wv.{li}"] = rng.normal(0, s, (D, kd))
                p[f"{view}.wo.{li}"] = rng.normal(0, 1.0 / np.sqrt(qd), (qd, D))
            p[f"w1.{li}"] = rng.normal(0, s, (D, 2 * D))
            p[f"w2.{li}"] = rng.normal(0, 1.0 / np.sqrt(2 * D), (2 * D, D))
        return cls(cfg, p)

    @property
    def mask_id(self) -> int:
        return self.cfg.vocab

    def new_cache(self, cap: int):
        c = self.cfg
        shape = (c.layers, 1, c.n_kv_heads, cap, c.head_dim)
        return np.zeros(shape), np.zeros(shape)

    def forward_block(self, tokens, L: int, kc, vc, view: str, mask_mode: int) -> np.ndarray:
        """Run len(tokens) block rows at positions L.. through every layer.

        Each layer writes the block's K/V (projected by ``view``'s weights) into
        the shared cache slots [L, L+n) and then runs block attention over the
        cache with ``mask_mode``.  Returns the final hidden states [n, D].
        """
        c = self.cfg
        n = len(tokens)
        x = self.p["emb"][np.asarray(tokens)] + self.p["pos"][L:L + n]
        ctx = np.array([L], np.int32)
        for li in range(c.layers):
            q = _rows(x, self.p[f"{view}.wq.{li}"]).reshape(1, n, c.n_q_heads, c.head_dim)
            k = _rows(x, self.p[f"{view}.wk.{li}"]).reshape(n, c.n_kv_heads, c.head_dim)
            v = _rows(x, self.p[f"{view}.wv.{li}"]).reshape(n, c.n_kv_heads, c.head_dim)
            kc[li, 0, :, L:L + n, :] = k.transpose(1, 0, 2)
            vc[li, 0, :, L:L + n, :] = v.transpose(1, 0, 2)
            a = block_attn(q, kc[li], vc[li], ctx, mask_mode)
            x = x + _rows(a.reshape(n, -1), self.p[f"{view}.wo.{li}"])
            x = x + _rows(np.tanh(_rows(x, self.p[f"w1.{li}"])), self.p[f"w2.{li}"])
        return x

    def greedy(self, hidden: np.ndarray) -> np.ndarray:
        logits = _rows(hidden, self.p["lm"].T)
        return row_argmax(logits)[0]


def sequential_decode(model: ToyModel, prompt, n_new: int, cap: int = 256):
    """Token-by-token greedy AR decoding (the reference behaviour).

    The prompt's tokens except the last are cached one at a time; the last
    prompt token is the first anchor.  Returns (emitted tokens, kc, vc, L).
    """
    kc, vc = model.new_cache(cap)
    L = 0
    for t in prompt[:-1]:
        model.forward_block([t], L, kc, vc, "ar", MASK_AR)
        L += 1
    anchor = prompt[-1]
    out = []
    while len(out) < n_new:
        h = model.forward_block([anchor], L, kc, vc, "ar", MASK_AR)
        tok = int(model.greedy(h)[0])
        L += 1
        out.append(tok)
        anchor = tok
    return out, kc, vc, L


def diffusion_drafter(model: ToyModel, anchor: int, L: int, K: int, kc, vc):
    """Draft K tokens with the diffusion view: [anchor, <mask> x (K-1)], M_diff mask."""
    h = model.forward_block([anchor] + [model.mask_id] * (K - 1), L, kc, vc, "diff",
                            MASK_DIFF)
    return [int(t) for t in model.greedy(h)]


def block_decode(model: ToyModel, prompt, n_new: int, K: int, drafter=None, cap: int = 256,
                 trace: list | None = None, verify_fn=verify, commit_fn=kv_commit):
    """Orthrus-style block decoding: draft -> AR verify -> consensus -> commit.

    ``drafter(anchor, L, K, kc, vc, emitted)`` returns K token ids; by default
    the diffusion view drafts.  Returns (emitted tokens, kc, vc, L).  If
    ``trace`` is a list, per-step (L, accept_len, next_tok) tuples are appended.
    ``verify_fn`` / ``commit_fn`` default to the oracle's; tests swap in
    deliberately wrong variants to show the losslessness check catches them.
    """
    kc, vc = model.new_cache(cap)
    L = 0
    for t in prompt[:-1]:
        model.forward_block([t], L, kc, vc, "ar", MASK_AR)
        L += 1
    anchor = prompt[-1]
    out: list[int] = []
    while len(out) < n_new:
        if drafter is None:
            draft = diffusion_drafter(model, anchor, L, K, kc, vc)
        else:
            draft = [int(t) for t in drafter(anchor, L, K, kc, vc, list(out))]
        h = model.forward_block([anchor] + draft[:K - 1], L, kc, vc, "ar", MASK_AR)
        am = model.greedy(h)
        acc, nxt = verify_fn(np.asarray([am]), np.asarray([draft]))
        a, nt = int(acc[0]), int(nxt[0])
        emitted = draft[:a] + ([nt] if a < K else [])
        new_l, st = commit_fn(np.array([L], np.int32), acc, K, cap)
        if st != 0:
            raise RuntimeError("cache capacity exceeded in toy decode")
        if trace is not None:
            trace.append((L, a, nt))
        L = int(new_l[0])
        out.extend(emitted)
        anchor = nt
    return out[:n_new], kc, vc, L
