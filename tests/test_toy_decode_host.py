"""The on-device decode loop's bookkeeping, checked on the CPU.

`toy_decode` drives the library's kernels; here, inside the test only, the
binding's calls are replaced by the fp64 oracle's (attention, greedy choice,
consensus, commit) and the model runs on CPU tensors. What is checked is the
loop itself: the block built from anchor + masks, drafts and AR rows aligned as
the method requires (gist.science summary §2.3 items 1-3), the tokens emitted
per step (accepted drafts + correction token, or all K drafts), the length
pointer, and that the result equals token-by-token decoding (exactly, since the
stand-ins are fp64 and row-independent).
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_block_drafting_b200 import toy_decode as td

DIMS = td.ToyDims(vocab=96, hidden=64, layers=2, n_q_heads=2, n_kv_heads=1, head_dim=64,
                  max_pos=256)


class OracleBinding:
    """Stand-ins for the binding functions toy_decode calls (CPU, fp64)."""
    MASK_DIFF, MASK_AR = oracle.MASK_DIFF, oracle.MASK_AR

    def __init__(self):
        self.calls = []

    def block_attn(self, q, kc, vc, ctx, mode):
        self.calls.append(("attn", mode, q.shape[1]))
        out = oracle.block_attn(q, kc, vc, ctx.numpy(), mode)
        return torch.from_numpy(out).to(torch.bfloat16)

    def lmhead_argmax(self, h, W):
        am, _, _ = oracle.lmhead_argmax(h, W)
        return torch.from_numpy(np.asarray(am, np.int32))

    def kv_commit(self, ctx, acc, K, cap):
        new, st = oracle.kv_commit(ctx.numpy(), acc.numpy(), K, cap)
        assert st == 0
        ctx.copy_(torch.from_numpy(np.asarray(new, np.int32)))

    def verify_commit(self, am, draft, ctx, cap):
        acc, nxt = oracle.verify(am.numpy(), draft.numpy())
        self.kv_commit(ctx, torch.from_numpy(np.asarray(acc, np.int32)), am.shape[1], cap)
        return (torch.from_numpy(np.asarray(acc, np.int32)),
                torch.from_numpy(np.asarray(nxt, np.int32)))


@pytest.fixture()
def cpu_model(monkeypatch):
    fake = OracleBinding()
    monkeypatch.setattr(td, "ob", fake)
    return td.GpuToyModel(DIMS, td.random_params(DIMS, seed=7), device="cpu"), fake


def prompts():
    g = torch.Generator().manual_seed(1)
    return torch.randint(0, DIMS.vocab, (2, 6), generator=g)


@pytest.mark.parametrize("K", [1, 3, 8])
def test_block_decode_equals_token_by_token(cpu_model, K):
    model, fake = cpu_model
    ref = td.sequential_decode(model, prompts(), 20, cap=64)
    trace = []
    got = td.block_decode(model, prompts(), 20, K, cap=64, trace=trace)
    assert got == ref
    # every step's diffusion pass attends K rows with the diffusion mask, and the
    # AR pass K rows with the causal mask
    modes = [(m, n) for kind, m, n in fake.calls if kind == "attn" and n == K]
    assert (oracle.MASK_DIFF, K) in modes and (oracle.MASK_AR, K) in modes
    for acc, nxt in trace:
        assert all(0 <= a <= K for a in acc)


def test_step_accounting_with_a_planted_error(cpu_model):
    model, _ = cpu_model
    K, j, n = 5, 2, 24
    ref = td.sequential_decode(model, prompts(), n + K, cap=96)
    P = prompts().shape[1]

    def planted(anchor, ctx, kc, vc):
        done = (ctx - (P - 1)).tolist()        # tokens emitted so far
        d = [list(ref[b][done[b]:done[b] + K]) for b in range(len(done))]
        for row in d:
            row[j] = (row[j] + 1) % DIMS.vocab
        return torch.tensor(d, dtype=torch.int32)

    trace = []
    got = td.block_decode(model, prompts(), n, K, cap=96, drafter=planted, trace=trace)
    assert got == [r[:n] for r in ref]
    # j drafts accepted and one correction token per step: j + 1 tokens per step
    assert all(a == j for acc, _ in trace for a in acc)
    assert len(trace) == -(-n // (j + 1))


def test_perfect_drafter_emits_whole_blocks(cpu_model):
    model, _ = cpu_model
    K, n = 4, 20
    ref = td.sequential_decode(model, prompts(), n + K, cap=96)
    P = prompts().shape[1]

    def perfect(anchor, ctx, kc, vc):
        done = (ctx - (P - 1)).tolist()
        return torch.tensor([ref[b][done[b]:done[b] + K] for b in range(len(done))],
                            dtype=torch.int32)

    trace = []
    got = td.block_decode(model, prompts(), n, K, cap=96, drafter=perfect, trace=trace)
    assert got == [r[:n] for r in ref]
    assert all(a == K for acc, _ in trace for a in acc)
    assert len(trace) == n // K
