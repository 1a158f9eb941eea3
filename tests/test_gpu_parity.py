"""GPU parity: every CUDA kernel against the fp64 CPU oracle on the same seeded inputs.

Bars (fixed by the benchmark spec, applied in fp64 after conversion):
  consensus / commit      bit-exact
  attention               max-abs <= 2e-2 and rel-L2 <= 5e-3 over the tensor
  LM-head argmax          exact on every row whose oracle top-2 gap >= 1e-3
Cases span several 64-key tiles with ragged tails, empty prefixes, K = 1 and
32, both head dims, GQA packing, NaN-poisoned unused cache slots, and the
tiny / Qwen3-8B single-layer / 40K-context / ragged-batch workloads.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_block_drafting_b200 import orthrus as ob
from lossless_block_drafting_b200 import synth

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2, GAP = 2e-2, 5e-3, 1e-3


def attn_gpu(case: synth.AttnCase, mode, dev_status=None, workspace=None):
    """Run the CUDA path; unless the caller inspects the status itself, assert the
    kernels reported no device-side error (including a bounded wait giving up)."""
    q = case.q.cuda()
    kc = case.k_cache.cuda()
    vc = case.v_cache.cuda()
    cl = torch.from_numpy(case.ctx_lens).cuda()
    st = dev_status if dev_status is not None else torch.zeros(1, dtype=torch.int32,
                                                               device="cuda")
    out = ob.block_attn(q, kc, vc, cl, mode, dev_status=st, workspace=workspace)
    torch.cuda.synchronize()
    if dev_status is None:
        assert int(st.item()) == 0, ob.status_str(int(st.item()))
    return out.cpu()


def lmhead_gpu(h, W, want_max=False):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = ob.lmhead_argmax(h.cuda(), W.cuda(), want_max=want_max, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, ob.status_str(int(st.item()))
    return res


def assert_attn_close(got_bf16, ref):
    got = got_bf16.double().numpy()
    assert np.isfinite(got).all()
    err = got - ref
    max_abs = np.abs(err).max()
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    assert max_abs <= ATOL and rel <= RTOL_L2, (max_abs, rel)


ATTN_CASES = [
    # B, K, Hq, Hkv, d, ctx_lens, cap
    (1, 8, 4, 2, 64, [512], None),                 # tiny oracle-check step
    (1, 1, 4, 2, 64, [77], None),                  # K = 1 (plain decode)
    (2, 5, 6, 3, 64, [0, 13], 40),                 # empty prefix, ragged, slack slots
    (3, 32, 8, 2, 128, [40, 1, 130], 200),          # K = 32, GQA 4, d 128
    (1, 4, 2, 2, 128, [3], None),                  # MHA
    (2, 32, 32, 8, 128, [1000, 257], 1400),         # Qwen3-8B heads, ragged
    (1, 16, 16, 2, 64, [300], None),               # G*K = 128 exactly
    (2, 32, 16, 2, 128, [100, 70], None),          # G*K = 256 -> two head chunks
    (1, 8, 4, 1, 64, [50], None),                  # one short segment: most CTAs idle
    (1, 32, 8, 2, 128, [6000], None),              # 2 segments x 74 CTAs: merge in 2 batches
    (1, 32, 12, 2, 64, [500], None),               # G = 6 over 4-head chunks: padding heads
    (20, 4, 16, 8, 64, list(range(60, 1260, 60)), None),  # 160 segments > 148 CTAs
    (36, 4, 2, 1, 64, [17 * i % 300 for i in range(36)], None),  # B > 32, 36 segments
    (40, 2, 8, 4, 64, [5 + 29 * i % 700 for i in range(40)], None),  # B > 32, stream-K
]


@pytest.mark.parametrize("det", [False, True], ids=["balanced", "deterministic"])
@pytest.mark.parametrize("mode", [ob.MASK_DIFF, ob.MASK_AR])
@pytest.mark.parametrize("B,K,Hq,Hkv,d,ctx,cap", ATTN_CASES)
def test_block_attn_matches_oracle(B, K, Hq, Hkv, d, ctx, cap, mode, det):
    case = synth.attn_case(B, K, Hq, Hkv, d, ctx, cap=cap, seed=B * 7 + K + d)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode)
    flag = ob.ATTN_DETERMINISTIC if det else 0
    assert_attn_close(attn_gpu(case, mode | flag), ref)


@pytest.mark.parametrize("mode", [ob.MASK_DIFF, ob.MASK_AR])
def test_block_attn_qwen3_8b_layer_ctx4096(mode):
    """Qwen3-8B-shaped single layer: 32q/8kv, d 128, context 4096, K 32."""
    case = synth.attn_case(1, 32, 32, 8, 128, [4096], seed=21)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode)
    assert_attn_close(attn_gpu(case, mode), ref)


@pytest.mark.parametrize("K,mode", [(32, ob.MASK_DIFF), (32, ob.MASK_AR), (1, ob.MASK_AR)])
def test_block_attn_40k_context(K, mode):
    """The 40K comparison point: context 40960, both modes and K = 1 plain decode."""
    case = synth.attn_case(1, K, 32, 8, 128, [40960], seed=33)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode)
    assert_attn_close(attn_gpu(case, mode), ref)


def test_block_attn_ragged_batch_8():
    """Config 4: 8 sequences, lengths U[1024, 32768], every sequence against the oracle."""
    lens = synth.ctx_lens_uniform(8, 1024, 32768, seed=4)
    case = synth.attn_case(8, 32, 32, 8, 128, lens, cap=32768 + 32, seed=44, poison=None)
    for mode in (ob.MASK_DIFF, ob.MASK_AR):
        got = attn_gpu(case, mode)
        ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode)
        assert_attn_close(got, ref)
        for b in range(8):   # and sequence by sequence (the bar holds per sequence too)
            assert_attn_close(got[b:b + 1], ref[b:b + 1])


@pytest.mark.parametrize("mode", [ob.MASK_DIFF, ob.MASK_AR])
def test_block_attn_131072_context(mode):
    """The longest context of the sweep: 131072 keys, Qwen3-8B heads, K = 32."""
    case = synth.attn_case(1, 32, 32, 8, 128, [131072], seed=131, poison=None)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, mode)
    assert_attn_close(attn_gpu(case, mode), ref)


def test_block_attn_ar_row_equals_single_token_decode_on_gpu():
    """Batch-vs-sequential on the device: AR row i ~= K=1 decode at context L+i."""
    L, K = 700, 8
    case = synth.attn_case(1, K, 32, 8, 128, [L], seed=5)
    block = attn_gpu(case, ob.MASK_AR).double()
    for i in range(K):
        one = synth.AttnCase(case.q[:, i:i + 1].contiguous(), case.k_cache, case.v_cache,
                             np.array([L + i], np.int32), 1)
        single = attn_gpu(one, ob.MASK_AR).double()
        assert (single[:, 0] - block[:, i]).abs().max() <= ATOL


def test_block_attn_capacity_error_is_reported_and_clamped():
    case = synth.attn_case(1, 8, 4, 2, 64, [100], cap=108, seed=6)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = synth.AttnCase(case.q, case.k_cache, case.v_cache, np.array([105], np.int32), 8)
    out = attn_gpu(bad, ob.MASK_AR, dev_status=st)
    assert int(st.item()) == ob.ECAPACITY
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, np.array([100], np.int32),
                            ob.MASK_AR)
    assert_attn_close(out, ref)   # clamped to L = cap - K = 100


def test_block_attn_repeat_calls_same_workspace_are_deterministic():
    case = synth.attn_case(2, 32, 32, 8, 128, [3000, 5000], seed=8)
    q, kc, vc = case.q.cuda(), case.k_cache.cuda(), case.v_cache.cuda()
    cl = torch.from_numpy(case.ctx_lens).cuda()
    ws = torch.zeros(ob.block_attn_workspace_size(2, 32, 8, 128, 32), dtype=torch.uint8, device="cuda")
    mode = ob.MASK_AR | ob.ATTN_DETERMINISTIC
    a = ob.block_attn(q, kc, vc, cl, mode, workspace=ws).clone()
    b = ob.block_attn(q, kc, vc, cl, mode, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # 16 segments (2 sequences x 8 KV heads) <= SMs: each CTA works inside one
    # segment, so the grid-barrier ticket is unused and each segment's
    # completion counter (after the 256-byte ticket block) grew by 2^20 per call
    head = ws[:256 + 16 * 8].view(torch.int64).cpu()
    assert int(head[0]) == 0
    assert head[32:48].tolist() == [2 << 20] * 16


def _counters(ws, S):
    """(completion counters, claim counters) of the first S segments: the
    workspace head is a 256-byte grid ticket, then SMs completion counters,
    then SMs claim counters (u64)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    head = ws[:256 + 2 * sms * 8].view(torch.int64).cpu()
    u = [int(x) & ((1 << 64) - 1) for x in head.tolist()]
    return u[32:32 + S], u[32 + sms:32 + sms + S]


def test_block_attn_balanced_calls_reuse_the_workspace():
    """Balanced mode claims key groups from per-segment counters that the
    segment's last CTA puts back to 0 after every call: many calls on one
    workspace, alternating with deterministic calls, all stay within tolerance
    of the oracle."""
    case = synth.attn_case(1, 32, 32, 8, 128, [9000], seed=12)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, ob.MASK_AR)
    ws = torch.zeros(ob.block_attn_workspace_size(1, 32, 8, 128, 32), dtype=torch.uint8,
                     device="cuda")
    for i in range(6):
        flag = ob.ATTN_DETERMINISTIC if i % 3 == 2 else 0
        assert_attn_close(attn_gpu(case, ob.MASK_AR | flag, workspace=ws), ref)
    done, claims = _counters(ws, 8)
    assert done == [6 << 20] * 8      # completion counters: 2^20 per call
    assert claims == [0] * 8          # claim counters: reset after every call


@pytest.mark.parametrize("start_calls", [(1 << 32) - 2, (1 << 44) - 2],
                         ids=["2^32_calls", "u64_wrap"])
def test_block_attn_counters_near_wrap(start_calls):
    """A long-lived workspace: the completion counters are seeded as if
    start_calls calls had already run (2^32 - 2 calls, the point where a 32-bit
    call count would wrap; 2^44 - 2 calls, where the 64-bit counter itself wraps
    past 2^64).  Four balanced calls across that boundary each match the oracle,
    report no device error, and leave the counters where they must be."""
    case = synth.attn_case(1, 32, 32, 8, 128, [9000], seed=13)
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, ob.MASK_AR)
    ws = torch.zeros(ob.block_attn_workspace_size(1, 32, 8, 128, 32), dtype=torch.uint8,
                     device="cuda")
    seed = (start_calls << 20) & ((1 << 64) - 1)
    signed = seed - (1 << 64) if seed >= (1 << 63) else seed
    ws[256:256 + 8 * 8].view(torch.int64).fill_(signed)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(4):
        assert_attn_close(attn_gpu(case, ob.MASK_AR, dev_status=st, workspace=ws), ref)
        assert int(st.item()) == 0, ob.status_str(int(st.item()))
    done, claims = _counters(ws, 8)
    assert done == [((start_calls + 4) << 20) & ((1 << 64) - 1)] * 8
    assert claims == [0] * 8


def test_block_attn_one_workspace_alternating_shapes():
    """One zeroed workspace, sized for the largest of three shapes, serves calls
    that alternate between them (per-segment partition with balanced claims,
    a short single segment, and a stream-K batch with more segments than SMs):
    the counters sit at the same place for every shape and every call leaves
    them in the state the next one starts from."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    Bs = sms // 8 + 2
    shapes = [
        (1, 32, 32, 8, 128, [7000], 21),
        (1, 8, 4, 1, 64, [300], 22),
        (Bs, 4, 16, 8, 64, [60 + 7 * i for i in range(Bs)], 23),
    ]
    cases = []
    for B, K, Hq, Hkv, d, ctx, seed in shapes:
        c = synth.attn_case(B, K, Hq, Hkv, d, ctx, seed=seed)
        cases.append((c, (B, Hq, Hkv, d, K)))
    size = max(ob.block_attn_workspace_size(*dims) for _, dims in cases)
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    refs = {}
    for i in (0, 1, 2, 0, 2, 1, 0, 0, 1):
        c, _ = cases[i]
        for mode in (ob.MASK_AR, ob.MASK_DIFF):
            if (i, mode) not in refs:
                refs[(i, mode)] = oracle.block_attn(c.q, c.k_cache, c.v_cache, c.ctx_lens, mode)
            assert_attn_close(attn_gpu(c, mode, workspace=ws), refs[(i, mode)])


def test_block_attn_stream_k_mode_advances_the_grid_ticket():
    # 20 sequences x 8 KV heads = 160 segments > 148 SMs: the flat tile range is
    # split evenly and all CTAs meet at the grid barrier before the merge
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B = sms // 8 + 2
    case = synth.attn_case(B, 4, 16, 8, 64, [60 + 7 * i for i in range(B)], seed=9)
    q, kc, vc = case.q.cuda(), case.k_cache.cuda(), case.v_cache.cuda()
    cl = torch.from_numpy(case.ctx_lens).cuda()
    ws = torch.zeros(ob.block_attn_workspace_size(B, 16, 8, 64, 4), dtype=torch.uint8,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(3):
        out = ob.block_attn(q, kc, vc, cl, ob.MASK_DIFF, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert int(ws[:8].view(torch.int64).item()) == 3 * sms
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, ob.MASK_DIFF)
    assert_attn_close(out.cpu(), ref)


def _check_argmax(got, ref_am, gap):
    got = got.cpu().numpy()
    firm = gap >= GAP
    assert np.array_equal(got[firm], ref_am[firm]), np.nonzero(got[firm] != ref_am[firm])


@pytest.mark.parametrize("R,H,V", [(5, 256, 3000), (32, 512, 20000), (33, 128, 4099),
                                   (7, 64, 1)])
def test_lmhead_argmax_small(R, H, V):
    h, W = synth.lmhead_case(R, H, V, seed=R + V)
    am, top1, gap = oracle.lmhead_argmax(h, W)
    got, mx = lmhead_gpu(h, W, want_max=True)
    _check_argmax(got, am, gap)
    np.testing.assert_allclose(mx.cpu().numpy(), top1, rtol=1e-3, atol=1e-3)


def test_lmhead_argmax_two_passes():
    """R > 256 runs in two passes of the kernel."""
    h, W = synth.lmhead_case(300, 128, 5000, seed=3)
    am, _, gap = oracle.lmhead_argmax(h, W)
    got = lmhead_gpu(h, W)
    _check_argmax(got, am, gap)


def test_lmhead_argmax_ties_pick_lowest_index():
    H, V = 128, 2048
    h = torch.zeros(4, H, dtype=torch.bfloat16)
    h[:, 0] = 1.0
    W = torch.zeros(V, H, dtype=torch.bfloat16)
    W[[5, 900, 2047], 0] = 3.0          # three-way exact tie for every row
    got = lmhead_gpu(h, W)
    assert got.cpu().tolist() == [5, 5, 5, 5]


def test_lmhead_qwen3_8b_full_vocab():
    """Config-2 LM head: hidden 4096 x vocab 151936, W ~ N(0, 0.02), h ~ N(0, 1)."""
    h, W = synth.lmhead_case(32, 4096, 151936, seed=2)
    am, top1, gap = oracle.lmhead_argmax(h, W)
    got, mx = lmhead_gpu(h, W, want_max=True)
    _check_argmax(got, am, gap)
    np.testing.assert_allclose(mx.cpu().numpy(), top1, rtol=1e-3, atol=2e-3)


def test_lmhead_ragged_batch_rows_256():
    """Config-4 LM head (R = 8 x 32 = 256 rows, full vocabulary), every row against
    the oracle."""
    h, W = synth.lmhead_case(256, 4096, 151936, seed=9)
    am, top1, gap = oracle.lmhead_argmax(h, W)
    got, mx = lmhead_gpu(h, W, want_max=True)
    _check_argmax(got, am, gap)
    np.testing.assert_allclose(mx.cpu().numpy(), top1, rtol=1e-3, atol=2e-3)


def test_row_argmax_f32_config1_and_verify():
    """Tiny config: fp32 logits [8 x 4096], drafts planted for a prefix U{0..8}."""
    logits = synth.normal_f32((8, 4096), seed=1)
    am_ref, _, _ = oracle.row_argmax(logits)
    got = ob.row_argmax_f32(logits.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), am_ref)
    for seed in range(6):
        a = synth.accept_uniform(1, 8, seed=seed)
        draft = synth.plant_draft(am_ref[None, :], a, 4096, seed=seed + 100)
        acc_ref, nxt_ref = oracle.verify(am_ref[None, :], draft)
        acc, nxt = ob.verify(got[None, :].contiguous(), torch.from_numpy(draft).cuda())
        torch.cuda.synchronize()
        assert acc.item() == acc_ref[0] == a[0] and nxt.item() == nxt_ref[0]


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_verify_commit_exhaustive_tiny(K):
    import itertools
    seqs = np.array(list(itertools.product(range(3), repeat=K)), np.int32)
    am = np.repeat(seqs, len(seqs), axis=0)
    dr = np.tile(seqs, (len(seqs), 1))
    B = am.shape[0]
    lens = np.random.default_rng(K).integers(0, 50, size=B).astype(np.int32)
    cap = 52
    acc_ref, nxt_ref = oracle.verify(am, dr)
    lens_ref, st_ref = oracle.kv_commit(lens, acc_ref, K, cap)
    cl = torch.from_numpy(lens).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    acc, nxt = ob.verify_commit(torch.from_numpy(am).cuda(), torch.from_numpy(dr).cuda(), cl,
                                cap, dev_status=st)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert np.array_equal(nxt.cpu().numpy(), nxt_ref)
    assert np.array_equal(cl.cpu().numpy(), lens_ref)
    assert int(st.item()) == st_ref
    # separate verify, then commit
    cl2 = torch.from_numpy(lens).cuda()
    acc2, nxt2 = ob.verify(torch.from_numpy(am).cuda(), torch.from_numpy(dr).cuda())
    ob.kv_commit(cl2, acc2, K, cap)
    torch.cuda.synchronize()
    assert np.array_equal(acc2.cpu().numpy(), acc_ref)
    assert np.array_equal(nxt2.cpu().numpy(), nxt_ref)
    assert np.array_equal(cl2.cpu().numpy(), lens_ref)


def test_verify_commit_planted_ragged_batch():
    """Config 4: 8 sequences, accept lengths U{0..32}, commit adds min(a+1, 32)."""
    B, K, V = 8, 32, 151936
    target = np.random.default_rng(3).integers(0, V, size=(B, K)).astype(np.int32)
    a = synth.accept_uniform(B, K, seed=4)
    draft = synth.plant_draft(target, a, V, seed=5)
    lens = synth.ctx_lens_uniform(B, 1024, 32768, seed=4)
    cap = 32768 + 32
    lens_ref, st_ref = oracle.kv_commit(lens, a, K, cap)
    cl = torch.from_numpy(lens).cuda()
    acc, nxt = ob.verify_commit(torch.from_numpy(target).cuda(), torch.from_numpy(draft).cuda(),
                                cl, cap)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), a)
    assert np.array_equal(cl.cpu().numpy(), lens_ref)


def test_commit_errors_on_device():
    cl = torch.tensor([10, 10, 10], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.kv_commit(cl, torch.tensor([3, 40, 0], dtype=torch.int32, device="cuda"), 32, 12,
                 dev_status=st)
    torch.cuda.synchronize()
    # a=3 -> 14 > cap 12 clamps (ECAPACITY); a=40 > K is rejected (EINVAL); a=0 -> 11
    assert cl.cpu().tolist() == [12, 10, 11]
    assert int(st.item()) in (ob.ECAPACITY, ob.EINVAL)


def test_end_to_end_step_qwen3_8b_layer():
    """Attention (both views) + LM head + verify/commit on config-2 shapes; drafts are
    planted from the ORACLE argmax with accept length ~ Geometric(0.2) capped at 32."""
    K, V = 32, 151936
    h, W = synth.lmhead_case(K, 4096, V, seed=12)
    am_ref, _, gap = oracle.lmhead_argmax(h, W)
    a = synth.accept_geometric(1, 0.2, 32, seed=13)
    draft = synth.plant_draft(am_ref[None, :], a, V, seed=14)
    acc_ref, nxt_ref = oracle.verify(am_ref[None, :], draft)
    case = synth.attn_case(1, K, 32, 8, 128, [4096], seed=15)
    cl = torch.from_numpy(case.ctx_lens).cuda()
    kc, vc = case.k_cache.cuda(), case.v_cache.cuda()
    ob.block_attn(case.q.cuda(), kc, vc, cl, ob.MASK_DIFF)
    ob.block_attn(case.q.cuda(), kc, vc, cl, ob.MASK_AR)
    am = ob.lmhead_argmax(h.cuda(), W.cuda())
    acc, nxt = ob.verify_commit(am[None, :].contiguous(), torch.from_numpy(draft).cuda(), cl,
                                case.k_cache.shape[2])
    torch.cuda.synchronize()
    first = int(acc_ref[0])
    if (gap[:min(first + 1, K)] >= GAP).all():   # no near-tie at or before the mismatch
        assert int(acc.item()) == first and int(nxt.item()) == int(nxt_ref[0])
    assert int(cl.item()) == 4096 + min(int(acc.item()) + 1, K)
