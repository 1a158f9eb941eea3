"""GPU parity of the prompt pre-filling attention against the fp64 oracle.

Pre-filling a chunk of P tokens at positions L_b + i is block attention in the
AR view's causal mask with the chunk in place of the K-token block (the AR head
pre-fills the shared cache: gist.science summary 2.1 item 1; the paper's
abstract), so the oracle is oracle.block_attn in AR mode with K = P.  Bars as
for block attention: max-abs <= 2e-2 and rel-L2 <= 5e-3 after conversion to
fp64.  Cases: ragged chunk lengths (not multiples of the 128-position tile),
chunks after a committed prefix, MHA and odd GQA groups (single-tile CTAs),
head_dim 64 and 128, NaN-poisoned slots past the chunk, Qwen3-8B shapes at
P = 512 and 4096 in full and P = 32768 on sampled rows, chunked pre-filling
against one pass, and the capacity clamp.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_block_drafting_b200 import orthrus as ob
from lossless_block_drafting_b200 import synth

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2 = 2e-2, 5e-3


def close(got_bf16, ref):
    got = got_bf16.double().cpu().numpy()
    assert np.isfinite(got).all()
    err = got - ref
    max_abs = np.abs(err).max()
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    assert max_abs <= ATOL and rel <= RTOL_L2, (max_abs, rel)


def run(case, dev_status=None):
    q = case.q.cuda()
    kc, vc = case.k_cache.cuda(), case.v_cache.cuda()
    cl = torch.from_numpy(case.ctx_lens).cuda()
    st = dev_status if dev_status is not None else torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ob.prefill_attn(q, kc, vc, cl, dev_status=st)
    torch.cuda.synchronize()
    if dev_status is None:
        assert int(st.item()) == 0, ob.status_str(int(st.item()))
    assert torch.equal(cl.cpu(), torch.from_numpy(case.ctx_lens))  # lengths untouched
    return out


PREFILL_CASES = [
    # B, P, Hq, Hkv, d, committed prefix per sequence
    (1, 1, 4, 2, 64, [0]),                 # one token
    (1, 37, 4, 2, 64, [0]),                # shorter than a tile
    (2, 300, 8, 2, 128, [0, 50]),          # ragged tail, chunk after a prefix
    (1, 256, 4, 4, 128, [0]),              # MHA: every CTA has one tile
    (1, 200, 6, 2, 64, [10]),              # G = 3: a pair and a single tile per group
    (3, 129, 32, 8, 128, [0, 1, 127]),     # Qwen3 heads, one position past a tile
    (1, 640, 16, 2, 128, [333]),           # several groups, prefix not group-aligned
]


@pytest.mark.parametrize("B,P,Hq,Hkv,d,prefix", PREFILL_CASES)
def test_prefill_matches_oracle(B, P, Hq, Hkv, d, prefix):
    case = synth.attn_case(B, P, Hq, Hkv, d, prefix, seed=B * 13 + P + d)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, oracle.MASK_AR)
    close(run(case), ref)


@pytest.mark.parametrize("P", [512, 4096])
def test_prefill_qwen3_8b_full(P):
    """Qwen3-8B attention shapes (32 query / 8 KV heads, head_dim 128), whole prompt."""
    case = synth.attn_case(1, P, 32, 8, 128, [0], seed=P)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, oracle.MASK_AR)
    close(run(case), ref)


def test_prefill_qwen3_8b_32768_sampled_rows():
    """P = 32768: every output, but the oracle computes sampled rows only -- row i
    of the chunk is the AR decode of one token at context i (keys [0, i + 1))."""
    P = 32768
    case = synth.attn_case(1, P, 32, 8, 128, [0], seed=7, poison=None)
    got = run(case).double().cpu().numpy()
    assert np.isfinite(got).all()
    rows = [0, 1, 127, 128, 4095, 16384, 20000, P - 129, P - 128, P - 1]
    rows += list(np.random.default_rng(0).choice(P, 6, replace=False))
    for i in rows:
        i = int(i)
        one = oracle.block_attn(case.q[:, i:i + 1], case.k_cache, case.v_cache,
                                np.array([i], np.int32), oracle.MASK_AR)
        close(torch.from_numpy(got[:, i:i + 1]).to(torch.bfloat16), one)


def test_prefill_in_chunks_equals_one_pass():
    """Pre-filling 300 tokens and then 212 more (the second chunk at L = 300)
    gives what one 512-token pass gives, and both match the oracle."""
    case = synth.attn_case(1, 512, 32, 8, 128, [0], seed=3)
    whole = run(case)
    q = case.q.cuda()
    kc, vc = case.k_cache.cuda(), case.v_cache.cuda()
    out1 = ob.prefill_attn(q[:, :300].contiguous(), kc, vc, torch.tensor([0], dtype=torch.int32,
                                                                          device="cuda"))
    out2 = ob.prefill_attn(q[:, 300:].contiguous(), kc, vc, torch.tensor([300], dtype=torch.int32,
                                                                           device="cuda"))
    torch.cuda.synchronize()
    parts = torch.cat([out1, out2], dim=1)
    assert (parts.double() - whole.double()).abs().max().item() <= ATOL
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, oracle.MASK_AR)
    close(parts, ref)


def test_prefill_capacity_error_is_reported_and_clamped():
    case = synth.attn_case(1, 100, 8, 2, 64, [0], cap=150, seed=5, poison=None)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = synth.AttnCase(case.q, case.k_cache, case.v_cache, np.array([80], np.int32), 100)
    out = run(bad, dev_status=st)
    assert int(st.item()) == ob.ECAPACITY
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, np.array([50], np.int32),
                            oracle.MASK_AR)
    close(out, ref)  # clamped to L = cap - P = 50
