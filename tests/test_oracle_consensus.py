"""Pins for the oracle's greedy choice, consensus and commit (CPU only).

Rules fixed by the pages (gist.science summary of "Orthrus: Memory-Efficient
Parallel Token Generation via Dual-View Diffusion", §2.3 item 3; Hacker News
thread "Orthrus-Qwen3: ..." post #21): strict left-to-right comparison, keep
the longest prefix that matches the AR greedy choice, append the AR
correction token at the first mismatch, shorten the cache.  Checked here by
exhaustive brute force over tiny vocabularies against the defining properties,
by hand-worked examples (tests/golden), and by torch float64 matmul/argmax for
the LM head.
"""
import itertools
import os

import numpy as np
import pytest
import torch

import oracle
from lossless_block_drafting_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_verify_exhaustive_tiny(K):
    """All 3^K x 3^K (argmax, draft) pairs: the defining properties hold."""
    seqs = np.array(list(itertools.product(range(3), repeat=K)), np.int32)
    am = np.repeat(seqs, len(seqs), axis=0)
    dr = np.tile(seqs, (len(seqs), 1))
    acc, nxt = oracle.verify(am, dr)
    for n in range(len(am)):
        a = int(acc[n])
        assert 0 <= a <= K
        assert (am[n, :a] == dr[n, :a]).all()          # accepted prefix matches
        if a < K:
            assert am[n, a] != dr[n, a]                 # ...and is the longest
            assert nxt[n] == am[n, a]                   # AR correction token
        else:
            assert nxt[n] == dr[n, K - 1]               # full accept: last draft


def test_verify_planted_prefixes():
    B, K, V = 64, 32, 151936
    target = np.random.default_rng(1).integers(0, V, size=(B, K)).astype(np.int32)
    a_true = synth.accept_uniform(B, K, seed=2)
    draft = synth.plant_draft(target, a_true, V, seed=3)
    acc, nxt = oracle.verify(target, draft)
    assert np.array_equal(acc, a_true)
    for b in range(B):
        assert nxt[b] == (target[b, a_true[b]] if a_true[b] < K else draft[b, K - 1])


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line)
    return rows


def test_verify_hand_worked_examples():
    """Examples worked by hand from the consensus rule (tests/golden/verify_hand.txt)."""
    n = 0
    for row in _read_golden("verify_hand.txt"):
        f = dict(kv.split("=") for kv in row.split())
        am = np.array([[int(x) for x in f["argmax"].split(",")]], np.int32)
        dr = np.array([[int(x) for x in f["draft"].split(",")]], np.int32)
        acc, nxt = oracle.verify(am, dr)
        assert int(acc[0]) == int(f["accept"]), row
        assert int(nxt[0]) == int(f["next"]), row
        cl, st = oracle.kv_commit(np.array([int(f["L"])], np.int32), acc, am.shape[1],
                                  int(f["cap"]))
        assert int(cl[0]) == int(f["L_after"]), row
        n += 1
    assert n >= 6


@pytest.mark.parametrize("K", [1, 2, 5, 32])
def test_commit_advance_rule_exhaustive(K):
    cap = 100
    for L in (0, 3, cap - K, cap - 1, cap):
        for a in range(-1, K + 2):
            cl, st = oracle.kv_commit(np.array([L], np.int32), np.array([a], np.int32), K, cap)
            if a < 0 or a > K:
                assert st == oracle.EINVAL and cl[0] == L
                continue
            adv = min(a + 1, K)
            if L + adv > cap:
                assert st == oracle.ECAPACITY and cl[0] == cap
            else:
                assert st == oracle.OK and cl[0] == L + adv


def test_commit_is_per_sequence():
    cl, st = oracle.kv_commit(np.array([5, 10, 20], np.int32), np.array([0, 4, 3], np.int32),
                              4, 64)
    assert st == 0 and list(cl) == [6, 14, 24]


def test_lmhead_matches_torch_float64_and_reports_gap():
    h, W = synth.lmhead_case(R=12, H=256, V=3000, seed=4)
    am, top1, gap = oracle.lmhead_argmax(h, W)
    logits = h.double() @ W.double().T
    t2 = torch.topk(logits, 2, dim=1)
    assert np.array_equal(am, torch.argmax(logits, 1).numpy().astype(np.int32))
    np.testing.assert_allclose(top1, t2.values[:, 0].numpy(), rtol=1e-12)
    np.testing.assert_allclose(gap, (t2.values[:, 0] - t2.values[:, 1]).numpy(), rtol=1e-9,
                               atol=1e-12)


def test_lmhead_planted_winner_and_lowest_index_tie_break():
    rng = np.random.default_rng(5)
    R, H, V = 4, 64, 500
    h = rng.normal(size=(R, H))
    W = rng.normal(scale=0.01, size=(V, H))
    winners = [7, 499, 0, 250]
    for r, v in enumerate(winners):
        W[v] = h[r] * 10.0                      # logit 10|h_r|^2, far above the rest
    am, _, gap = oracle.lmhead_argmax(h, W)
    assert list(am) == winners and (gap > 1.0).all()
    # exact tie between rows 250 and 300 for hidden row 3 -> lowest index wins
    W[300] = W[250]
    am, _, gap = oracle.lmhead_argmax(h, W)
    assert am[3] == 250 and gap[3] == 0.0


def test_lmhead_sensitive_to_transposed_weight():
    """Using W's columns instead of rows changes the answer (guards the layout)."""
    rng = np.random.default_rng(6)
    h = rng.normal(size=(3, 40))
    W = rng.normal(size=(40, 40))
    am, _, _ = oracle.lmhead_argmax(h, W)
    assert np.array_equal(am, np.argmax(h @ W.T, 1))
    assert not np.array_equal(am, np.argmax(h @ W, 1))


def test_row_argmax_f32_and_nan():
    logits = synth.normal_f32((8, 4096), seed=7)
    am, top1, gap = oracle.row_argmax(logits)
    assert np.array_equal(am, torch.argmax(logits, 1).numpy())
    x = np.array([[np.nan, 1.0, 3.0, 3.0, -np.inf]], np.float32)
    am, top1, gap = oracle.row_argmax(x)
    assert am[0] == 2 and top1[0] == 3.0 and gap[0] == 0.0
