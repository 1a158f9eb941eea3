"""Losslessness pin for the oracle: block drafting == token-by-token greedy decoding.

The pages claim Orthrus is strictly lossless: the emitted text equals what the
frozen AR model produces token by token, whatever the drafter proposes
(gist.science summary of "Orthrus: Memory-Efficient Parallel Token Generation
via Dual-View Diffusion", §2.3 item 3 and §3; the paper's abstract; Hacker News
thread "Orthrus-Qwen3: ...", post #21).  In fp64 with identical per-row
arithmetic this must hold exactly, and the committed cache slots must equal
the sequential decoder's cache.  Deliberately wrong consensus/commit variants
(planted in the oracle's call sites, on the CPU) must break it.
"""
import numpy as np
import pytest

import oracle
from oracle import toy_model as tm

PROMPT = [3, 17, 42, 8, 23]
N_NEW = 40


@pytest.fixture(scope="module")
def model():
    return tm.ToyModel.random(tm.ToyConfig(seed=11))


@pytest.fixture(scope="module")
def reference(model):
    return tm.sequential_decode(model, PROMPT, N_NEW + 40)


def _check(model, reference, K, drafter):
    ref_tokens, ref_k, ref_v, _ = reference
    trace = []
    toks, kc, vc, L = tm.block_decode(model, PROMPT, N_NEW, K, drafter=drafter, trace=trace)
    assert toks == ref_tokens[:N_NEW]
    # committed slots hold exactly the sequential decoder's K/V
    np.testing.assert_allclose(kc[:, :, :, :L], ref_k[:, :, :, :L], rtol=0, atol=1e-12)
    np.testing.assert_allclose(vc[:, :, :, :L], ref_v[:, :, :, :L], rtol=0, atol=1e-12)
    return trace


@pytest.mark.parametrize("K", [1, 2, 4, 8])
def test_diffusion_drafter_is_lossless(model, reference, K):
    _check(model, reference, K, None)


@pytest.mark.parametrize("K", [1, 4, 8])
def test_perfect_drafter_accepts_everything(model, reference, K):
    ref_tokens = reference[0]
    n_prompt = len(PROMPT)

    def perfect(anchor, L, K_, kc, vc, emitted):
        # the AR model's own continuation after `emitted`
        n = len(emitted)
        return ref_tokens[n:n + K_]

    trace = _check(model, reference, K, perfect)
    assert all(a == K for (_, a, _) in trace)
    assert trace[0][0] == n_prompt - 1


@pytest.mark.parametrize("K,err_at", [(4, 0), (4, 3), (8, 5)])
def test_planted_error_is_corrected(model, reference, K, err_at):
    ref_tokens = reference[0]

    def planted(anchor, L, K_, kc, vc, emitted):
        n = len(emitted)
        d = list(ref_tokens[n:n + K_])
        d[err_at] = (d[err_at] + 1) % model.cfg.vocab
        return d

    trace = _check(model, reference, K, planted)
    assert all(a == err_at for (_, a, _) in trace)


def test_random_drafter_is_lossless(model, reference):
    rng = np.random.default_rng(0)

    def rand(anchor, L, K_, kc, vc, emitted):
        return rng.integers(0, model.cfg.vocab, size=K_)

    _check(model, reference, 8, rand)


def test_wrong_commit_breaks_losslessness(model, reference):
    """Committing a+2 slots (caching an unverified token) must be detected."""
    def bad_commit(ctx_lens, accept_len, K, cap):
        cl, st = oracle.kv_commit(ctx_lens, accept_len, K, cap)
        return np.minimum(cl + 1, cap).astype(np.int32), st

    ref_tokens = reference[0]
    toks, *_ = tm.block_decode(model, PROMPT, N_NEW, 4, commit_fn=bad_commit)
    assert toks != ref_tokens[:N_NEW]


def test_wrong_correction_token_breaks_losslessness(model, reference):
    """Using the rejected draft instead of the AR correction token must be detected."""
    def bad_verify(argmax, draft):
        acc, nxt = oracle.verify(argmax, draft)
        a = int(acc[0])
        if a < draft.shape[1]:
            nxt = np.array([draft[0, a]], np.int32)
        return acc, nxt

    ref_tokens = reference[0]
    toks, *_ = tm.block_decode(model, PROMPT, N_NEW, 4, verify_fn=bad_verify)
    assert toks != ref_tokens[:N_NEW]


def test_wrong_alignment_breaks_losslessness(model, reference):
    """Comparing draft[i] with the AR choice of row i+1 (off by one) must be detected."""
    def shifted_verify(argmax, draft):
        am = np.concatenate([argmax[:, 1:], argmax[:, -1:]], axis=1)
        return oracle.verify(am, draft)

    ref_tokens = reference[0]
    toks, *_ = tm.block_decode(model, PROMPT, N_NEW, 4, verify_fn=shifted_verify)
    assert toks != ref_tokens[:N_NEW]
