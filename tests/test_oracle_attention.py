"""Pins for the oracle's block attention (CPU only).

What the pages fix (gist.science summary of "Orthrus: Memory-Efficient Parallel
Token Generation via Dual-View Diffusion", §2.2 M_diff rules and §2.3 items 1-2):
the diffusion view sees the committed prefix plus the whole block in both
directions; the AR view sees the prefix plus the block causally.  The checks
below pin the oracle to things other than itself: torch's float64 SDPA with an
explicit boolean mask (a library special case), the K=1 reduction to ordinary
decode, row-by-row reductions, block-slot permutation invariance, and closed
forms.  A transposed head mapping, a wrong mask bound, a dropped scale or a
missing normaliser each fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from lossless_block_drafting_b200 import synth


def sdpa_reference(case: synth.AttnCase, mode: int):
    """torch float64 SDPA with an explicit boolean mask per sequence."""
    s = case.shape
    B, K, Hq, Hkv, d = s["B"], s["K"], s["Hq"], s["Hkv"], s["d"]
    G = Hq // Hkv
    out = torch.empty(B, K, Hq, d, dtype=torch.float64)
    for b in range(B):
        L = int(case.ctx_lens[b])
        e = L + K
        q = case.q[b].double().permute(1, 0, 2)                       # [Hq, K, d]
        k = case.k_cache[b, :, :e].double().repeat_interleave(G, 0)   # [Hq, e, d]
        v = case.v_cache[b, :, :e].double().repeat_interleave(G, 0)
        j = torch.arange(e)
        i = torch.arange(K)
        if mode == oracle.MASK_DIFF:
            mask = torch.ones(K, e, dtype=torch.bool)
        else:
            mask = j[None, :] < (L + i[:, None] + 1)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
        out[b] = o.permute(1, 0, 2)
    return out.numpy()


CASES = [
    # B, K, Hq, Hkv, d, ctx_lens
    (1, 8, 4, 2, 64, [512]),          # tiny oracle-check shape
    (1, 1, 4, 2, 64, [77]),           # K = 1
    (2, 5, 6, 3, 16, [0, 13]),        # empty prefix, ragged
    (3, 32, 8, 2, 32, [40, 1, 130]),  # K = 32, GQA 4
    (1, 4, 2, 2, 8, [3]),             # MHA (G = 1)
]


@pytest.mark.parametrize("mode", [oracle.MASK_DIFF, oracle.MASK_AR])
@pytest.mark.parametrize("B,K,Hq,Hkv,d,ctx", CASES)
def test_matches_torch_sdpa_float64(B, K, Hq, Hkv, d, ctx, mode):
    case = synth.attn_case(B, K, Hq, Hkv, d, ctx, cap=max(ctx) + K + 3, seed=B + K + d)
    got = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode)
    ref = sdpa_reference(case, mode)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_ar_row_equals_single_token_decode():
    """AR row i of a K-block equals K=1 AR decode of query i at context L+i."""
    B, K, Hq, Hkv, d, L = 1, 7, 4, 2, 32, 50
    case = synth.attn_case(B, K, Hq, Hkv, d, [L], seed=3)
    block = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, oracle.MASK_AR)
    for i in range(K):
        one = oracle.block_attn(case.q[:, i:i + 1], case.k_cache, case.v_cache,
                                np.array([L + i], np.int32), oracle.MASK_AR)
        assert np.array_equal(one[:, 0], block[:, i])


def test_diff_row_equals_full_range_decode():
    """DIFF row i equals K=1 decode of query i over all L+K keys."""
    B, K, Hq, Hkv, d, L = 1, 6, 4, 1, 16, 21
    case = synth.attn_case(B, K, Hq, Hkv, d, [L], seed=4)
    block = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens,
                              oracle.MASK_DIFF)
    for i in range(K):
        one = oracle.block_attn(case.q[:, i:i + 1], case.k_cache, case.v_cache,
                                np.array([L + K - 1], np.int32), oracle.MASK_AR)
        assert np.array_equal(one[:, 0], block[:, i])


def test_diff_last_row_equals_ar_last_row():
    """The last block row sees the same keys in both modes."""
    case = synth.attn_case(2, 9, 4, 2, 32, [5, 33], seed=5)
    a = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, oracle.MASK_AR)
    b = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, oracle.MASK_DIFF)
    assert np.array_equal(a[:, -1], b[:, -1])
    assert not np.allclose(a[:, 0], b[:, 0])


def test_diff_invariant_to_block_slot_permutation():
    """Bidirectional block: permuting the block's K/V slots changes no output."""
    B, K, Hq, Hkv, d, L = 1, 8, 4, 2, 32, 40
    case = synth.attn_case(B, K, Hq, Hkv, d, [L], seed=6)
    base = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens,
                             oracle.MASK_DIFF)
    perm = torch.randperm(K, generator=torch.Generator().manual_seed(0))
    kc, vc = case.k_cache.clone(), case.v_cache.clone()
    kc[:, :, L:L + K] = case.k_cache[:, :, L + perm]
    vc[:, :, L:L + K] = case.v_cache[:, :, L + perm]
    got = oracle.block_attn(case.q, kc, vc, case.ctx_lens, oracle.MASK_DIFF)
    np.testing.assert_allclose(got, base, rtol=1e-12, atol=1e-13)
    # the causal view is NOT invariant to the same permutation
    ar0 = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, oracle.MASK_AR)
    ar1 = oracle.block_attn(case.q, kc, vc, case.ctx_lens, oracle.MASK_AR)
    assert not np.allclose(ar0, ar1)


def test_two_key_closed_form():
    """One query, two keys: weights are a logistic of the score difference."""
    d = 4
    q = np.zeros((1, 1, 1, d)); q[0, 0, 0] = [1.0, 2.0, 0.0, -1.0]
    kc = np.zeros((1, 1, 2, d)); vc = np.zeros((1, 1, 2, d))
    kc[0, 0, 0] = [0.5, 0.0, 1.0, 0.0]; kc[0, 0, 1] = [0.0, 1.0, 0.0, 1.0]
    vc[0, 0, 0] = [1.0, 0.0, 3.0, -2.0]; vc[0, 0, 1] = [0.0, 1.0, -1.0, 4.0]
    # L = 1 committed key, block K = 1 at slot 1 -> both keys visible in AR mode
    out = oracle.block_attn(q, kc, vc, np.array([1], np.int32), oracle.MASK_AR)
    s0 = (1.0 * 0.5) / 2.0                       # (q.k0)/sqrt(4)
    s1 = (2.0 - 1.0) / 2.0                       # (q.k1)/sqrt(4)
    p0 = 1.0 / (1.0 + math.exp(s1 - s0))
    expect = p0 * vc[0, 0, 0] + (1 - p0) * vc[0, 0, 1]
    np.testing.assert_allclose(out[0, 0, 0], expect, rtol=1e-14, atol=1e-15)


def test_equal_keys_give_mean_of_values():
    """Identical keys -> uniform weights -> output is the mean of the visible values."""
    B, K, Hq, Hkv, d, L = 1, 4, 2, 1, 8, 10
    rng = np.random.default_rng(0)
    q = rng.normal(size=(B, K, Hq, d))
    kc = np.tile(rng.normal(size=(1, 1, 1, d)), (B, Hkv, L + K, 1))
    vc = rng.normal(size=(B, Hkv, L + K, d))
    ar = oracle.block_attn(q, kc, vc, np.array([L], np.int32), oracle.MASK_AR)
    df = oracle.block_attn(q, kc, vc, np.array([L], np.int32), oracle.MASK_DIFF)
    for i in range(K):
        np.testing.assert_allclose(ar[0, i, 0], vc[0, 0, :L + i + 1].mean(0), rtol=1e-12,
                                   atol=1e-13)
        np.testing.assert_allclose(df[0, i, 1], vc[0, 0, :L + K].mean(0), rtol=1e-12,
                                   atol=1e-13)


def test_dominant_key_selects_its_value_and_scale_is_inverse_sqrt_d():
    """A key aligned with the query and far larger than the rest picks its value."""
    d = 16
    q = np.zeros((1, 1, 1, d)); q[0, 0, 0, 3] = 1.0
    kc = np.zeros((1, 1, 6, d)); vc = np.arange(6 * d, dtype=np.float64).reshape(1, 1, 6, d)
    kc[0, 0, 2, 3] = 400.0                       # score 400/sqrt(16) = 100 vs 0
    out = oracle.block_attn(q, kc, vc, np.array([5], np.int32), oracle.MASK_AR)
    np.testing.assert_allclose(out[0, 0, 0], vc[0, 0, 2], rtol=0, atol=1e-30)
    # with score 1 * 4 / sqrt(16) = 1 against five zeros: weight e / (e + 5)
    kc[0, 0, 2, 3] = 4.0
    out, lse = oracle.block_attn(q, kc, vc, np.array([5], np.int32), oracle.MASK_AR,
                                 return_lse=True)
    w = math.e / (math.e + 5)
    expect = w * vc[0, 0, 2] + (1 - w) / 5 * (vc[0, 0].sum(0) - vc[0, 0, 2])
    np.testing.assert_allclose(out[0, 0, 0], expect, rtol=1e-13)
    assert lse[0, 0, 0] == pytest.approx(math.log(math.e + 5), rel=1e-14)


def test_outputs_inside_value_hull_and_lse_matches_logsumexp():
    case = synth.attn_case(2, 16, 8, 2, 64, [100, 3], seed=9)
    for mode in (oracle.MASK_DIFF, oracle.MASK_AR):
        out, lse = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode,
                                     return_lse=True)
        for b in range(2):
            L = int(case.ctx_lens[b])
            for i in range(16):
                e = L + 16 if mode == oracle.MASK_DIFF else L + i + 1
                for h in range(8):
                    g = h // 4
                    v = case.v_cache[b, g, :e].double().numpy()
                    o = out[b, i, h]
                    assert np.all(o <= v.max(0) + 1e-12) and np.all(o >= v.min(0) - 1e-12)
                    k = case.k_cache[b, g, :e].double()
                    s = (k @ case.q[b, i, h].double()) / math.sqrt(64)
                    assert lse[b, i, h] == pytest.approx(float(torch.logsumexp(s, 0)),
                                                         rel=1e-13)


def test_capacity_violation_is_an_error():
    case = synth.attn_case(1, 4, 2, 1, 8, [10], seed=1)
    with pytest.raises(ValueError):
        oracle.block_attn(case.q, case.k_cache, case.v_cache, np.array([11], np.int32),
                          oracle.MASK_AR)


def test_poisoned_tail_is_never_read():
    """Slots at or beyond L+K hold NaN; a finite result proves they were not read."""
    case = synth.attn_case(2, 8, 4, 2, 16, [30, 2], cap=64, seed=2)
    assert torch.isnan(case.k_cache[0, 0, 38]).all()
    for mode in (oracle.MASK_DIFF, oracle.MASK_AR):
        out = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode)
        assert np.isfinite(out).all()
