"""GPU parity of the block Q/K/V append against the fp64 oracle, and of the
append -> block attention pair against the oracle's pair."""
import numpy as np
import pytest
import torch

import oracle
from lossless_block_drafting_b200 import orthrus as ob

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2 = 2e-2, 5e-3


def bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def make_case(B, K, Hq, Hkv, d, ctx, cap, norm, seed):
    g = torch.Generator().manual_seed(seed)
    qkv = torch.randn(B * K, (Hq + 2 * Hkv) * d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, cap, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, cap, d, generator=g).to(torch.bfloat16)
    qw = kw = None
    if norm:
        qw = (1 + 0.2 * torch.randn(d, generator=g)).to(torch.bfloat16)
        kw = (1 + 0.2 * torch.randn(d, generator=g)).to(torch.bfloat16)
    return qkv, kc, vc, np.asarray(ctx, np.int32), qw, kw


def close(got, ref):
    got = got.double().cpu().numpy()
    err = got - ref
    assert np.isfinite(got).all()
    assert np.abs(err).max() <= ATOL and np.linalg.norm(err) <= RTOL_L2 * np.linalg.norm(ref), \
        (np.abs(err).max(), np.linalg.norm(err) / np.linalg.norm(ref))


CASES = [
    # B, K, Hq, Hkv, d, ctx_lens, cap, qk-norm
    (1, 32, 32, 8, 128, [40960], 40960 + 64, True),      # Qwen3-8B block at 40K
    (3, 8, 8, 2, 64, [0, 13, 500], 600, True),           # ragged, empty prefix, d 64
    (1, 1, 4, 2, 128, [131000], 131008, False),          # K = 1, no norm, large position
    (2, 32, 16, 4, 128, [7, 4090], 4200, True),
]


@pytest.mark.parametrize("B,K,Hq,Hkv,d,ctx,cap,norm", CASES)
def test_qkv_append_matches_oracle(B, K, Hq, Hkv, d, ctx, cap, norm):
    qkv, kc, vc, L, qw, kw = make_case(B, K, Hq, Hkv, d, ctx, cap, norm, seed=B + K + d)
    kc_d, vc_d = kc.cuda(), vc.cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = ob.block_qkv_append(qkv.cuda(), kc_d, vc_d, torch.from_numpy(L).cuda(), Hq, K,
                            q_norm_w=None if qw is None else qw.cuda(),
                            k_norm_w=None if kw is None else kw.cuda(), rope_theta=1e6,
                            rms_eps=1e-6, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rq, rk, rv = oracle.qkv_append(qkv, L, K, Hq, Hkv, d, kc.double().numpy(),
                                   vc.double().numpy(), q_norm_w=qw, k_norm_w=kw, theta=1e6,
                                   eps=1e-6)
    close(q, rq)
    kc_g, vc_g = kc_d.cpu(), vc_d.cpu()
    for b in range(B):
        sl = slice(int(L[b]), int(L[b]) + K)
        close(kc_g[b][:, sl], rk[b][:, sl])
        # values are copied bit for bit; every other slot is untouched
        assert torch.equal(vc_g[b][:, sl], bf16(rv[b][:, sl]))
        keep = torch.ones(cap, dtype=torch.bool)
        keep[sl] = False
        assert torch.equal(kc_g[b][:, keep], kc[b][:, keep])
        assert torch.equal(vc_g[b][:, keep], vc[b][:, keep])


def test_capacity_error_is_reported_and_clamped_like_attention():
    B, K, Hq, Hkv, d, cap = 1, 8, 4, 2, 64, 100
    qkv, kc, vc, _, qw, kw = make_case(B, K, Hq, Hkv, d, [0], cap, True, seed=3)
    kc_d, vc_d = kc.cuda(), vc.cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.block_qkv_append(qkv.cuda(), kc_d, vc_d, torch.tensor([97], dtype=torch.int32).cuda(),
                        Hq, K, q_norm_w=qw.cuda(), k_norm_w=kw.cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == ob.ECAPACITY
    _, rk, _ = oracle.qkv_append(qkv, np.array([cap - K], np.int32), K, Hq, Hkv, d,
                                 kc.double().numpy(), vc.double().numpy(), q_norm_w=qw,
                                 k_norm_w=kw)
    close(kc_d.cpu()[0][:, cap - K:], rk[0][:, cap - K:])


@pytest.mark.parametrize("mode", [ob.MASK_DIFF, ob.MASK_AR])
def test_append_then_block_attention_matches_the_oracle_pair(mode):
    """The append writes exactly what block attention then reads: the GPU pair
    against the oracle pair (append in fp64, attention over the rounded cache)."""
    B, K, Hq, Hkv, d, cap = 2, 32, 32, 8, 128, 3000
    L = np.array([1500, 2900], np.int32)
    qkv, kc, vc, _, qw, kw = make_case(B, K, Hq, Hkv, d, L, cap, True, seed=9)
    kc_d, vc_d, Ld = kc.cuda(), vc.cuda(), torch.from_numpy(L).cuda()
    q = ob.block_qkv_append(qkv.cuda(), kc_d, vc_d, Ld, Hq, K, q_norm_w=qw.cuda(),
                            k_norm_w=kw.cuda())
    out = ob.block_attn(q, kc_d, vc_d, Ld, mode).cpu()
    rq, rk, rv = oracle.qkv_append(qkv, L, K, Hq, Hkv, d, kc.double().numpy(),
                                   vc.double().numpy(), q_norm_w=qw, k_norm_w=kw)
    # the oracle's attention reads the bf16-rounded block (what the cache holds)
    ref = oracle.block_attn(bf16(rq), bf16(rk), bf16(rv), L, mode)
    close(out, ref)
