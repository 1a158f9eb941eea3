"""The bounded-wait timeout path, exercised on the GPU without any fault.

Every wait inside the kernels (on an mbarrier, on a segment's completion
counter, at the grid barrier) gives up after the library's wait limit, raises
the CTA's abort flag, stores ORTHRUS_ETIMEOUT in dev_status, lets its in-flight
copies and MMAs land, frees its tensor memory and returns.  Here the limit is
set to 100 ns, far below the microseconds that a TMA load or an MMA takes, so
real waits run out; the test then checks that the kernel returned (the stream
synchronises), that the status says ETIMEOUT, and that after restoring the
default limit a call on a re-zeroed workspace matches the oracle again.
Nothing waits on a flag that is never set: every wait here would complete on
its own, only later than the limit allows.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_block_drafting_b200 import orthrus as ob
from lossless_block_drafting_b200 import synth

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2, GAP = 2e-2, 5e-3, 1e-3


def _close(got_bf16, ref):
    got = got_bf16.double().numpy()
    err = got - ref
    assert np.abs(err).max() <= ATOL
    assert np.linalg.norm(err) <= RTOL_L2 * np.linalg.norm(ref)


@pytest.fixture
def short_waits():
    ob.set_wait_limit_ns(100)
    try:
        yield
    finally:
        ob.set_wait_limit_ns(0)


def test_block_attn_wait_runs_out_then_recovers(short_waits):
    case = synth.attn_case(1, 32, 32, 8, 128, [9000], seed=61)
    q, kc, vc = case.q.cuda(), case.k_cache.cuda(), case.v_cache.cuda()
    cl = torch.from_numpy(case.ctx_lens).cuda()
    ws = ob.new_block_attn_workspace(1, 32, 8, 128, 32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.block_attn(q, kc, vc, cl, ob.MASK_AR, workspace=ws, dev_status=st)
    torch.cuda.synchronize()          # the kernel returned
    assert int(st.item()) == ob.ETIMEOUT, ob.status_str(int(st.item()))

    ob.set_wait_limit_ns(0)           # default limit, fresh workspace and status
    ws.zero_()
    st.zero_()
    out = ob.block_attn(q, kc, vc, cl, ob.MASK_AR, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, ob.status_str(int(st.item()))
    ref = oracle.block_attn(case.q, case.k_cache, case.v_cache, case.ctx_lens, ob.MASK_AR)
    _close(out.cpu(), ref)


def test_lmhead_wait_runs_out_then_recovers(short_waits):
    h, W = synth.lmhead_case(32, 1024, 40000, seed=62)
    hd, Wd = h.cuda(), W.cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.lmhead_argmax(hd, Wd, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == ob.ETIMEOUT, ob.status_str(int(st.item()))

    ob.set_wait_limit_ns(0)
    st.zero_()
    got = ob.lmhead_argmax(hd, Wd, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, ob.status_str(int(st.item()))
    am, _, gap = oracle.lmhead_argmax(h, W)
    firm = gap >= GAP
    assert np.array_equal(got.cpu().numpy()[firm], am[firm])
