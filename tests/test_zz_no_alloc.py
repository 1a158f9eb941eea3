"""The allocation-free LM-head entry point agrees with the workspace one.

orthrus_lmhead_argmax_noalloc exists for callers that cannot allocate device
memory (no allocator of their own, or a memory plan frozen after start-up); it
keeps its scratch in the library's own fixed device array.  This file is named
to be collected last, so a failure here never hides another test's result.  It
calls both entry points through the C ABI twice in a row (the scratch keeps
the previous call's contents, which must not leak into the next result) and
requires identical argmax and max-logit outputs.  R = 300 runs two passes of
the kernel over the same scratch (rows 0..255, then 256..299).
"""
import ctypes

import pytest
import torch

from lossless_block_drafting_b200 import build as libbuild
from lossless_block_drafting_b200 import orthrus as ob
from lossless_block_drafting_b200 import synth

pytestmark = pytest.mark.gpu


def _c(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("R,H,V", [(32, 4096, 151936), (5, 256, 3000), (300, 256, 5000)])
def test_noalloc_matches_workspace_entry_point_twice(R, H, V):
    libbuild.build()
    lib = ob.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ws = torch.empty(ob.lmhead_workspace_size(R, V), dtype=torch.uint8, device="cuda")
    for call in range(2):
        h, W = synth.lmhead_case(R, H, V, seed=100 + call)
        h, W = h.cuda(), W.cuda()
        ref_am = torch.empty(R, dtype=torch.int32, device="cuda")
        ref_mx = torch.empty(R, dtype=torch.float32, device="cuda")
        got_am = torch.full((R,), -7, dtype=torch.int32, device="cuda")
        got_mx = torch.full((R,), float("nan"), dtype=torch.float32, device="cuda")
        st = torch.zeros(2, dtype=torch.int32, device="cuda")
        rc = lib.orthrus_lmhead_argmax(_c(h), _c(W), R, H, V, _c(ref_am), _c(ref_mx), _c(ws),
                                       ws.numel(), _c(st[0:1]), stream)
        assert rc == ob.OK, ob.status_str(rc)
        rc = lib.orthrus_lmhead_argmax_noalloc(_c(h), _c(W), R, H, V, _c(got_am), _c(got_mx),
                                               _c(st[1:2]), stream)
        assert rc == ob.OK, ob.status_str(rc)
        torch.cuda.synchronize()
        assert st.tolist() == [0, 0]
        assert torch.equal(got_am, ref_am), call
        assert torch.equal(got_mx, ref_mx), call
        assert int(got_am.min()) >= 0 and int(got_am.max()) < V
