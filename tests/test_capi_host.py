"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before any launch (CPU only: no CUDA call is reached)."""
import ctypes
import os
import re

import pytest

from lossless_block_drafting_b200 import build as libbuild
from lossless_block_drafting_b200 import orthrus as ob

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "orthrus.h")


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return ob.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(orthrus_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("orthrus_block_attn", "orthrus_lmhead_argmax", "orthrus_verify",
                 "orthrus_kv_commit", "orthrus_verify_commit", "orthrus_row_argmax_f32",
                 "orthrus_block_attn_workspace_size", "orthrus_lmhead_workspace_size",
                 "orthrus_status_str", "orthrus_abi_version", "orthrus_block_qkv_append",
                 "orthrus_set_wait_limit_ns", "orthrus_prefill_attn"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(0, -9, -1):
        s = ob.status_str(code)
        assert s.startswith("ORTHRUS")
    assert "unknown" in ob.status_str(-99)
    assert lib.orthrus_abi_version() == 3


def test_wait_limit_setter_accepts_any_value(lib):
    # host-only: the limit is read at each launch; 0 restores the default
    for ns in (1, 100, 2_000_000_000, 0):
        assert lib.orthrus_set_wait_limit_ns(ns) == ob.OK


def _view(B=1, Hkv=2, cap=64, d=64, k=0x1000, v=0x2000, lens=0x3000):
    return ob.KVCacheView(k, v, lens, B, Hkv, cap, d)


A = 0x10000  # a 16-byte aligned fake device address; never dereferenced on error paths


@pytest.mark.parametrize("kwargs,status", [
    (dict(K=0), ob.EINVAL),
    (dict(K=33), ob.EINVAL),
    (dict(mode=2), ob.EINVAL),
    (dict(Hq=3), ob.ESHAPE),            # Hq % Hkv != 0
    (dict(d=96), ob.EUNSUPPORTED),
    (dict(cap=4, K=8), ob.ESHAPE),      # cap < K
    (dict(q=A + 8), ob.EALIGN),
    (dict(q=None), ob.EINVAL),
])
def test_block_attn_host_validation(lib, kwargs, status):
    K = kwargs.get("K", 8)
    view = _view(cap=kwargs.get("cap", 64), d=kwargs.get("d", 64))
    q = kwargs.get("q", A)
    rc = lib.orthrus_block_attn(q, ctypes.byref(view), kwargs.get("Hq", 4), K,
                                kwargs.get("mode", 0), A, A, 1 << 20, None, None)
    assert rc == status


def test_block_attn_empty_batch_is_a_noop(lib):
    view = _view(B=0)
    assert lib.orthrus_block_attn(A, ctypes.byref(view), 4, 8, 1, A, A, 0, None, None) == ob.OK


def test_lmhead_host_validation(lib):
    f = lib.orthrus_lmhead_argmax
    assert f(None, A, 4, 128, 10, A, None, A, 1 << 20, None, None) == ob.EINVAL
    assert f(A, A, 4, 100, 10, A, None, A, 1 << 20, None, None) == ob.EUNSUPPORTED  # H % 64
    assert f(A, A, 4, 32, 10, A, None, A, 1 << 20, None, None) == ob.EINVAL         # H < 64
    assert f(A, A, 4, 128, 0, A, None, A, 1 << 20, None, None) == ob.EINVAL         # V < 1
    assert f(A + 4, A, 4, 128, 10, A, None, A, 1 << 20, None, None) == ob.EALIGN
    assert f(A, A, 0, 128, 10, A, None, A, 1 << 20, None, None) == ob.OK           # R = 0


def test_consensus_host_validation(lib):
    assert lib.orthrus_verify(A, A, 1, 0, A, A, None) == ob.EINVAL
    assert lib.orthrus_verify(A, A, 1, 33, A, A, None) == ob.EINVAL
    assert lib.orthrus_verify(None, A, 1, 4, A, A, None) == ob.EINVAL
    assert lib.orthrus_verify(A, A, 0, 4, A, A, None) == ob.OK  # empty batch
    view = _view(B=3)
    assert lib.orthrus_verify_commit(A, A, 2, 4, A, A, ctypes.byref(view), None, None) == \
        ob.ESHAPE
    assert lib.orthrus_kv_commit(None, A, 4, None, None) == ob.EINVAL
    assert lib.orthrus_kv_commit(ctypes.byref(_view(B=0)), A, 4, None, None) == ob.OK
    assert lib.orthrus_row_argmax_f32(A, 2, 0, A, None) == ob.EINVAL


def test_workspace_query_reports_cuda_failure_without_a_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    n = ctypes.c_size_t(0)
    assert lib.orthrus_block_attn_workspace_size(1, 32, 8, 128, 32, ctypes.byref(n)) == ob.ECUDA
    assert lib.orthrus_block_attn_workspace_size(1, 32, 8, 96, 32, ctypes.byref(n)) == \
        ob.EUNSUPPORTED


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 8, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ob.block_attn(q, q, q, torch.zeros(1, dtype=torch.int32), ob.MASK_AR)


def test_qkv_append_host_validation(lib):
    f = lib.orthrus_block_qkv_append
    view = _view(B=2, Hkv=2, cap=64, d=128)
    args = lambda **kw: (kw.get("qkv", A), kw.get("qw", None), kw.get("kw", None),
                         kw.get("theta", 1e6), kw.get("eps", 1e-6), kw.get("Hq", 4),
                         kw.get("K", 8), ctypes.byref(kw.get("view", view)), kw.get("out", A),
                         None, None)
    assert f(*args(qkv=None)) == ob.EINVAL
    assert f(*args(K=0)) == ob.EINVAL
    assert f(*args(theta=0.0)) == ob.EINVAL
    assert f(*args(eps=-1.0)) == ob.EINVAL
    assert f(*args(qw=A)) == ob.EINVAL                     # one weight without the other
    assert f(*args(Hq=3)) == ob.ESHAPE
    assert f(*args(view=_view(B=2, Hkv=2, cap=64, d=96))) == ob.EUNSUPPORTED
    assert f(*args(K=65)) == ob.ESHAPE                     # cap < K
    assert f(*args(out=A + 2)) == ob.EALIGN
    assert f(*args(view=_view(B=0, Hkv=2, cap=64, d=128))) == ob.OK


@pytest.mark.parametrize("kwargs,status", [
    (dict(P=0), ob.EINVAL),
    (dict(Hq=3), ob.ESHAPE),            # Hq % Hkv != 0
    (dict(d=96), ob.EUNSUPPORTED),
    (dict(cap=16, P=32), ob.ESHAPE),    # cap < P
    (dict(q=A + 8), ob.EALIGN),
    (dict(q=None), ob.EINVAL),
])
def test_prefill_attn_host_validation(lib, kwargs, status):
    view = _view(cap=kwargs.get("cap", 64), d=kwargs.get("d", 64))
    rc = lib.orthrus_prefill_attn(kwargs.get("q", A), ctypes.byref(view), kwargs.get("Hq", 4),
                                  kwargs.get("P", 8), A, None, None)
    assert rc == status


def test_prefill_attn_empty_batch_is_a_noop(lib):
    view = _view(B=0)
    assert lib.orthrus_prefill_attn(A, ctypes.byref(view), 4, 8, A, None, None) == ob.OK
