"""Pins of the oracle's block Q/K/V append (per-head RMS norm of q and k, rotary
embedding at positions L_b + i, K/V into cache slots [L_b, L_b + K)).

Each check is fixed by the mathematics, not by retyping the formula: hand-worked
d = 4 rotations, identity at position 0, norm preservation, relative-position
invariance of q.k, composition of rotations, the RMS-norm closed form, and the
slot bookkeeping.
"""
import math

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(17)


def one_head(x, pos, theta=10000.0, which="q", w=None, eps=1e-6):
    """Run a single head of a single token through the oracle."""
    d = x.shape[0]
    qkv = np.zeros((1, 3 * d))
    col = {"q": 0, "k": 1, "v": 2}[which]
    qkv[0, col * d:(col + 1) * d] = x
    kc = np.zeros((1, 1, pos + 1, d))
    vc = np.zeros((1, 1, pos + 1, d))
    ww = None if w is None else np.asarray(w, np.float64)
    q, kc, vc = oracle.qkv_append(qkv, [pos], 1, 1, 1, d, kc, vc, q_norm_w=ww, k_norm_w=ww,
                                  theta=theta, eps=eps)
    return {"q": q[0, 0, 0], "k": kc[0, 0, pos], "v": vc[0, 0, pos]}[which]


def test_hand_worked_d4_rotations():
    # theta = 1e4, d = 4: a_0 = p, a_1 = p * 1e4^(-1/2) = p / 100.  Pairs (0, 2), (1, 3).
    c1, s1 = math.cos(1.0), math.sin(1.0)
    c2, s2 = math.cos(0.01), math.sin(0.01)
    np.testing.assert_allclose(one_head(np.array([1.0, 0, 0, 0]), 1), [c1, 0, s1, 0], atol=1e-15)
    np.testing.assert_allclose(one_head(np.array([0, 1.0, 0, 0]), 1), [0, c2, 0, s2], atol=1e-15)
    np.testing.assert_allclose(one_head(np.array([0, 0, 1.0, 0]), 1), [-s1, 0, c1, 0], atol=1e-15)
    np.testing.assert_allclose(one_head(np.array([0, 0, 0, 1.0]), 1, which="k"),
                               [0, -s2, 0, c2], atol=1e-15)


def test_position_zero_is_the_identity_and_v_is_copied():
    x = RNG.normal(size=64)
    for which in ("q", "k", "v"):
        np.testing.assert_array_equal(one_head(x, 0, which=which), x)
    np.testing.assert_array_equal(one_head(x, 777, which="v"), x)


def test_rotation_preserves_norms_at_large_positions():
    for pos in (1, 4097, 131071):
        x = RNG.normal(size=128)
        y = one_head(x, pos, theta=1e6)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)
        # each rotated pair keeps its own norm too
        np.testing.assert_allclose(np.hypot(y[:64], y[64:]), np.hypot(x[:64], x[64:]),
                                   rtol=1e-12)


def test_q_dot_k_depends_only_on_the_position_difference():
    q, k = RNG.normal(size=128), RNG.normal(size=128)
    for m, n, s in ((5, 2, 1000), (40000, 39990, 17), (0, 3, 90000)):
        a = one_head(q, m, theta=1e6) @ one_head(k, n, theta=1e6, which="k")
        b = one_head(q, m + s, theta=1e6) @ one_head(k, n + s, theta=1e6, which="k")
        assert abs(a - b) < 1e-9 * max(1.0, abs(a))


def test_rotations_compose():
    x = RNG.normal(size=64)
    for m, n in ((3, 4), (1000, 24), (65536, 12345)):
        np.testing.assert_allclose(one_head(one_head(x, m), n), one_head(x, m + n), atol=1e-9)


def test_rms_norm_closed_form():
    x = 3.0 * RNG.normal(size=128)
    w = RNG.normal(size=128)
    y = one_head(x, 0, w=np.ones(128), eps=0.0)       # position 0: no rotation
    assert abs(np.mean(y * y) - 1.0) < 1e-12
    y = one_head(x, 0, w=w, eps=1e-3)
    np.testing.assert_allclose(y, x / math.sqrt(np.mean(x * x) + 1e-3) * w, rtol=1e-12)
    # scale invariance of the normalised head (eps = 0)
    np.testing.assert_allclose(one_head(5 * x, 9, w=w, eps=0.0), one_head(x, 9, w=w, eps=0.0),
                               rtol=1e-12)


def test_slots_heads_and_capacity():
    B, K, Hq, Hkv, d, cap = 2, 3, 4, 2, 8, 12
    L = np.array([2, 9], np.int32)
    qkv = RNG.normal(size=(B * K, (Hq + 2 * Hkv) * d))
    poison = np.full((B, Hkv, cap, d), 7.5)
    q, kc, vc = oracle.qkv_append(qkv, L, K, Hq, Hkv, d, poison, poison, theta=1e6)
    for b in range(B):
        written = np.zeros(cap, bool)
        written[L[b]:L[b] + K] = True
        assert np.all(kc[b][:, ~written] == 7.5) and np.all(vc[b][:, ~written] == 7.5)
        for i in range(K):
            row = qkv[b * K + i].reshape(Hq + 2 * Hkv, d)
            for g in range(Hkv):      # kv head g comes from packed head Hq + g / Hq + Hkv + g
                np.testing.assert_array_equal(vc[b, g, L[b] + i], row[Hq + Hkv + g])
                assert abs(np.linalg.norm(kc[b, g, L[b] + i]) -
                           np.linalg.norm(row[Hq + g])) < 1e-12
            for h in range(Hq):
                assert abs(np.linalg.norm(q[b, i, h]) - np.linalg.norm(row[h])) < 1e-12
    with pytest.raises(ValueError):
        oracle.qkv_append(qkv, np.array([2, 10], np.int32), K, Hq, Hkv, d, poison, poison)


def test_matches_rotate_half_restatement_in_torch_float64():
    """The same rotation written the way common model code states it:
    x * cos + rotate_half(x) * sin with cos/sin of [freqs, freqs]."""
    B, K, Hq, Hkv, d, cap, theta = 1, 5, 2, 1, 16, 64, 1e6
    L = np.array([40], np.int32)
    qkv = RNG.normal(size=(B * K, (Hq + 2 * Hkv) * d))
    q, kc, _ = oracle.qkv_append(qkv, L, K, Hq, Hkv, d, np.zeros((B, Hkv, cap, d)),
                                 np.zeros((B, Hkv, cap, d)), theta=theta)
    t = torch.tensor(qkv, dtype=torch.float64).view(K, Hq + 2 * Hkv, d)
    inv = 1.0 / theta ** (torch.arange(0, d, 2, dtype=torch.float64) / d)
    pos = torch.arange(40, 40 + K, dtype=torch.float64)
    emb = torch.cat([torch.outer(pos, inv)] * 2, dim=1)[:, None, :]

    def rot(x):
        return x * emb.cos() + torch.cat([-x[..., d // 2:], x[..., :d // 2]], dim=-1) * emb.sin()

    np.testing.assert_allclose(q[0], rot(t[:, :Hq]).numpy(), atol=1e-12)
    np.testing.assert_allclose(kc[0, 0, 40:45], rot(t[:, Hq:Hq + 1])[:, 0].numpy(), atol=1e-12)


def test_norm_comes_before_the_rotation():
    """Per-coordinate weights do not commute with the rotation: the output at
    position p equals the normalised head (position 0, no rotation) rotated to p."""
    x, w = RNG.normal(size=64), RNG.normal(size=64)
    normed = one_head(x, 0, w=w, which="k")
    for p in (1, 333, 70000):
        np.testing.assert_allclose(one_head(x, p, w=w, which="k"), one_head(normed, p, which="k"),
                                   atol=1e-12)
        assert np.abs(one_head(x, p, w=w) - w * one_head(x / np.sqrt(np.mean(x * x) + 1e-6),
                                                         p)).max() > 1e-3
