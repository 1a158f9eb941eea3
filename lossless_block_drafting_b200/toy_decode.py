"""Block decoding on the GPU with a random-weight toy transformer.

This is the decode loop around the path's kernels, end to end on the device.
Orthrus (gist.science technical summary §2.1-2.3; Hacker News thread
"Orthrus-Qwen3: ..." posts #21 and #26) adds to a frozen AR transformer a
diffusion attention module with its own q/k/v/o projections that reads the same
KV cache. One decode step:

1. diffusion pass over [anchor, <mask> x (K-1)] at positions L..L+K-1 with the
   diffusion mask (committed prefix + bidirectional block) -> K greedy drafts;
2. AR pass over [anchor, draft_0 .. draft_{K-2}] with the causal mask -> the
   AR greedy token at each of the K positions;
3. exact consensus: keep the longest prefix where draft == AR greedy, emit the
   AR correction token, and move the length pointer by min(a + 1, K).

The emitted tokens must equal token-by-token greedy decoding with the AR view
(summary §2.3 item 3, §3) for any drafter.

The library's kernels do every step of the path: all attention goes through
``orthrus_block_attn`` (both masks), every greedy choice through
``orthrus_lmhead_argmax``, and consensus plus commit through
``orthrus_verify_commit`` (or ``orthrus_kv_commit`` for single-token steps).
The model's projections, MLP and cache writes are plain torch glue (fp32
residual stream). Positions and cache slots are gathered on the device from the
length pointer, so the loop never reads the lengths back. The block is always
written into the scratch slots [L, L+n), where the AR pass overwrites the
diffusion view's block K/V.

Readings where the pages are silent: block row i (position L+i) predicts the
token at position L+i+1; the new anchor is the last emitted token and is not yet
cached; the <mask> token is an extra embedding row with id == vocab; positions
are learned absolute embeddings (the toy has no RoPE).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import orthrus as ob


@dataclass
class ToyDims:
    vocab: int = 512
    hidden: int = 256
    layers: int = 2
    n_q_heads: int = 4
    n_kv_heads: int = 2
    head_dim: int = 64
    max_pos: int = 1024


def random_params(dims: ToyDims, seed: int = 0) -> dict:
    """Random weights (numpy fp64), laid out as [in, out] matrices per layer/view."""
    rng = np.random.default_rng(seed)
    D, V = dims.hidden, dims.vocab
    qd, kd = dims.n_q_heads * dims.head_dim, dims.n_kv_heads * dims.head_dim
    s = 1.0 / math.sqrt(D)
    p = {"emb": rng.normal(0, 1, (V + 1, D)),
         "pos": rng.normal(0, 0.5, (dims.max_pos, D)),
         "lm": rng.normal(0, 1, (V, D))}
    for li in range(dims.layers):
        for view in ("ar", "diff"):
            p[f"{view}.wq.{li}"] = rng.normal(0, s, (D, qd))
            p[f"{view}.wk.{li}"] = rng.normal(0, s, (D, kd))
            p[f"{view}.wv.{li}"] = rng.normal(0, s, (D, kd))
            p[f"{view}.wo.{li}"] = rng.normal(0, 1.0 / math.sqrt(qd), (qd, D))
        p[f"w1.{li}"] = rng.normal(0, s, (D, 2 * D))
        p[f"w2.{li}"] = rng.normal(0, 1.0 / math.sqrt(2 * D), (2 * D, D))
    return p


class GpuToyModel:
    """The toy transformer on one GPU; weights fp32 except the bf16 LM head."""

    def __init__(self, dims: ToyDims, params: dict, device="cuda"):
        if dims.head_dim not in (64, 128) or dims.hidden % 64:
            raise ValueError("head_dim must be 64 or 128 and hidden a multiple of 64")
        self.dims = dims
        self.device = torch.device(device)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.w = {k: torch.as_tensor(np.asarray(v), **f32) for k, v in params.items()
                  if k != "lm"}
        self.lm = torch.as_tensor(np.asarray(params["lm"]), **f32).to(torch.bfloat16).contiguous()
        self.mask_id = dims.vocab

    def new_cache(self, B: int, cap: int):
        d = self.dims
        shape = (d.layers, B, d.n_kv_heads, cap, d.head_dim)
        kc = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        vc = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        return kc, vc

    def forward_block(self, tokens: torch.Tensor, ctx_lens: torch.Tensor, kc, vc, view: str,
                      mask_mode: int) -> torch.Tensor:
        """Run the n tokens of each row of ``tokens`` [B, n] at positions
        ctx_lens[b] + i through every layer; each layer writes the block's K/V
        (``view``'s projections) into cache slots [L_b, L_b + n) and attends
        with ``mask_mode``. Returns the final hidden states, fp32 [B, n, D]."""
        d = self.dims
        B, n = tokens.shape
        ar = torch.arange(n, device=self.device)
        pos = ctx_lens.long()[:, None] + ar[None, :]                       # [B, n]
        x = self.w["emb"][tokens.long()] + self.w["pos"][pos]               # [B, n, D]
        bi = torch.arange(B, device=self.device)[:, None].expand(B, n)
        for li in range(d.layers):
            q = (x @ self.w[f"{view}.wq.{li}"]).view(B, n, d.n_q_heads, d.head_dim)
            k = (x @ self.w[f"{view}.wk.{li}"]).view(B, n, d.n_kv_heads, d.head_dim)
            v = (x @ self.w[f"{view}.wv.{li}"]).view(B, n, d.n_kv_heads, d.head_dim)
            kc[li][bi, :, pos] = k.to(torch.bfloat16)                       # slots [L, L+n)
            vc[li][bi, :, pos] = v.to(torch.bfloat16)
            a = ob.block_attn(q.to(torch.bfloat16).contiguous(), kc[li], vc[li], ctx_lens,
                              mask_mode)
            x = x + a.float().view(B, n, -1) @ self.w[f"{view}.wo.{li}"]
            x = x + torch.tanh(x @ self.w[f"w1.{li}"]) @ self.w[f"w2.{li}"]
        return x

    def greedy(self, hidden: torch.Tensor) -> torch.Tensor:
        """LM-head argmax per row (the library's fused kernel) -> int32 [B, n]."""
        B, n, D = hidden.shape
        h = hidden.reshape(B * n, D).to(torch.bfloat16).contiguous()
        return ob.lmhead_argmax(h, self.lm).view(B, n)

    def logit_gap(self, hidden: torch.Tensor) -> torch.Tensor:
        """Top-1 minus top-2 logit per row (fp32, diagnostics for near-ties)."""
        B, n, D = hidden.shape
        h = hidden.reshape(B * n, D).to(torch.bfloat16).float()
        top = torch.topk(h @ self.lm.float().T, 2, dim=1).values
        return (top[:, 0] - top[:, 1]).view(B, n)


def _prefill(model: GpuToyModel, prompts: torch.Tensor, K_max: int, cap: int):
    """Cache every prompt token but the last (the first anchor), K_max at a time."""
    B, P = prompts.shape
    kc, vc = model.new_cache(B, cap)
    ctx = torch.zeros(B, dtype=torch.int32, device=model.device)
    done = 0
    while done < P - 1:
        n = min(K_max, P - 1 - done)
        model.forward_block(prompts[:, done:done + n], ctx, kc, vc, "ar", ob.MASK_AR)
        # the whole chunk is committed: accept_len n - 1 advances by min(n, n)
        ob.kv_commit(ctx, torch.full((B,), n - 1, dtype=torch.int32, device=model.device), n,
                     cap)
        done += n
    return kc, vc, ctx


def sequential_decode(model: GpuToyModel, prompts: torch.Tensor, n_new: int, cap: int,
                      gaps: list | None = None) -> list[list[int]]:
    """Token-by-token greedy decoding with the AR view (the reference).

    ``prompts`` is int [B, P]. Returns B lists of n_new tokens; if ``gaps`` is a
    list, B lists holding the top-2 logit gap of each emitted token are appended.
    """
    B = prompts.shape[0]
    kc, vc, ctx = _prefill(model, prompts, 32, cap)
    anchor = prompts[:, -1:].to(torch.int32)
    zeros = torch.zeros(B, dtype=torch.int32, device=model.device)
    out, gap_steps = [], []
    for _ in range(n_new):
        h = model.forward_block(anchor, ctx, kc, vc, "ar", ob.MASK_AR)
        tok = model.greedy(h)                                   # [B, 1]
        if gaps is not None:
            gap_steps.append(model.logit_gap(h)[:, 0])
        ob.kv_commit(ctx, zeros, 1, cap)                        # the anchor is now cached
        out.append(tok)
        anchor = tok
    if gaps is not None:
        gaps.extend(torch.stack(gap_steps, dim=1).cpu().tolist())
    return torch.cat(out, dim=1).cpu().tolist()


def block_decode(model: GpuToyModel, prompts: torch.Tensor, n_new: int, K: int, cap: int,
                 drafter=None, trace: list | None = None) -> list[list[int]]:
    """Orthrus block decoding: diffusion draft -> AR verify -> consensus -> commit.

    ``drafter(anchor, ctx_lens, kc, vc)`` may replace the diffusion view; it
    returns int32 drafts [B, K] on the device. Returns B lists of n_new tokens;
    if ``trace`` is a list, per-step (accept_len, next_tok) host lists are appended.
    """
    B = prompts.shape[0]
    kc, vc, ctx = _prefill(model, prompts, 32, cap)
    anchor = prompts[:, -1:].to(torch.int32)
    masks = torch.full((B, K - 1), model.mask_id, dtype=torch.int32, device=model.device)
    out = [[] for _ in range(B)]
    while min(len(o) for o in out) < n_new:
        if drafter is None:
            h = model.forward_block(torch.cat([anchor, masks], dim=1), ctx, kc, vc, "diff",
                                    ob.MASK_DIFF)
            draft = model.greedy(h)                              # [B, K]
        else:
            draft = drafter(anchor, ctx, kc, vc).to(torch.int32).contiguous()
        h = model.forward_block(torch.cat([anchor, draft[:, :K - 1]], dim=1), ctx, kc, vc,
                                "ar", ob.MASK_AR)
        am = model.greedy(h)
        acc, nxt = ob.verify_commit(am, draft, ctx, cap)
        a_h, n_h, d_h = acc.cpu().tolist(), nxt.cpu().tolist(), draft.cpu().tolist()
        if trace is not None:
            trace.append((a_h, n_h))
        for b in range(B):
            out[b].extend(d_h[b][:a_h[b]] + ([n_h[b]] if a_h[b] < K else []))
        anchor = nxt.view(B, 1)
    return [o[:n_new] for o in out]
