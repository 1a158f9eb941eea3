"""Block decoding end to end on the GPU with a random-weight toy transformer.

The losslessness claim (gist.science technical summary §2.3 item 3, §3): the
tokens emitted by draft -> AR verify -> consensus -> commit equal token-by-token
greedy decoding, whatever the drafter. On the GPU both decoders run in bf16/fp32,
and the K-row AR pass and the one-row reference sum in different orders, so
equality is required up to near-ties: a divergence is accepted only where the
reference's top-1 minus top-2 logit gap is below GAP_TOL (logits are ~N(0, 20^2)
here, rounding noise is ~1e-2).
"""
import numpy as np
import pytest
import torch

from lossless_block_drafting_b200 import toy_decode as td
from oracle import toy_model as tm

pytestmark = pytest.mark.gpu

DIMS = td.ToyDims()
GAP_TOL = 0.5
N_NEW = 64
P = 9


def cap_for(K):
    return P + N_NEW + 2 * K + 8


@pytest.fixture(scope="module")
def model():
    return td.GpuToyModel(DIMS, td.random_params(DIMS, seed=3))


@pytest.fixture(scope="module")
def prompts():
    g = torch.Generator().manual_seed(5)
    return torch.randint(0, DIMS.vocab, (2, P), generator=g).cuda()


@pytest.fixture(scope="module")
def reference(model, prompts):
    gaps = []
    toks = td.sequential_decode(model, prompts, N_NEW + 40, cap_for(32) + 40, gaps=gaps)
    return toks, gaps


def assert_same_up_to_near_ties(got, ref, gaps, n=N_NEW):
    for b in range(len(got)):
        diff = [i for i in range(n) if got[b][i] != ref[b][i]]
        if diff:
            i = diff[0]
            assert gaps[b][i] < GAP_TOL, (b, i, got[b][i], ref[b][i], gaps[b][i])


def test_reference_is_not_degenerate(reference):
    toks, gaps = reference
    for b in range(len(toks)):
        assert len(set(toks[b])) > 8              # a varied continuation
    assert np.median(np.asarray(gaps)) > 5 * GAP_TOL  # near-ties are the exception


@pytest.mark.parametrize("K", [1, 4, 16, 32])
def test_diffusion_drafted_block_decode_equals_token_by_token(model, prompts, reference, K):
    trace = []
    got = td.block_decode(model, prompts, N_NEW, K, cap_for(K), trace=trace)
    ref, gaps = reference
    assert_same_up_to_near_ties(got, ref, gaps)
    for acc, _ in trace:
        assert all(0 <= a <= K for a in acc)


@pytest.mark.parametrize("K", [8, 32])
def test_perfect_drafter_accepts_whole_blocks(model, prompts, reference, K):
    ref, gaps = reference
    B = prompts.shape[0]

    def perfect(anchor, ctx, kc, vc):
        # tokens emitted so far = committed length - cached prompt tokens
        done = (ctx.cpu() - (P - 1)).tolist()
        return torch.tensor([ref[b][done[b]:done[b] + K] for b in range(B)],
                            dtype=torch.int32, device="cuda")

    trace = []
    got = td.block_decode(model, prompts, N_NEW, K, cap_for(K), drafter=perfect, trace=trace)
    assert_same_up_to_near_ties(got, ref, gaps)
    if got == [r[:N_NEW] for r in ref]:
        # every step before the end accepted all K drafts
        assert all(a == K for acc, _ in trace[:-1] for a in acc)
        assert len(trace) == -(-N_NEW // K)


def test_planted_error_is_corrected_every_block(model, prompts, reference):
    K, j = 8, 3
    ref, gaps = reference
    B = prompts.shape[0]

    def planted(anchor, ctx, kc, vc):
        done = (ctx.cpu() - (P - 1)).tolist()
        d = [list(ref[b][done[b]:done[b] + K]) for b in range(B)]
        for b in range(B):
            d[b][j] = (d[b][j] + 1) % DIMS.vocab
        return torch.tensor(d, dtype=torch.int32, device="cuda")

    trace = []
    got = td.block_decode(model, prompts, N_NEW, K, cap_for(K), drafter=planted, trace=trace)
    assert_same_up_to_near_ties(got, ref, gaps)
    if got == [r[:N_NEW] for r in ref]:
        # j drafts accepted, the AR token corrects the planted one: j + 1 per step
        assert all(a == j for acc, _ in trace for a in acc)


def test_gpu_toy_matches_fp64_oracle_toy(model, prompts, reference):
    """The GPU model computes the oracle's toy transformer (same weights)."""
    params = td.random_params(DIMS, seed=3)
    cfg = tm.ToyConfig(vocab=DIMS.vocab, hidden=DIMS.hidden, layers=DIMS.layers,
                       n_q_heads=DIMS.n_q_heads, n_kv_heads=DIMS.n_kv_heads,
                       head_dim=DIMS.head_dim, max_pos=DIMS.max_pos)
    ot = tm.ToyModel(cfg, params)
    n = 16
    ref, gaps = reference
    for b in range(prompts.shape[0]):
        want, *_ = tm.sequential_decode(ot, prompts[b].cpu().tolist(), n, cap=P + n + 4)
        diff = [i for i in range(n) if want[i] != ref[b][i]]
        if diff:
            assert gaps[b][diff[0]] < 2 * GAP_TOL, (b, diff[0], gaps[b][diff[0]])
