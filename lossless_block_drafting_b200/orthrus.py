"""Python binding of ``liborthrus.so`` (C ABI in ``include/orthrus.h``).

Argument marshalling only: every function checks torch tensors (device, dtype,
contiguity), passes their device pointers and the current CUDA stream to the C
entry point of the same name, and raises :class:`OrthrusError` on a non-zero
status.  All arithmetic runs in the library's CUDA kernels; there is no CPU
path, and a missing library raises instead of falling back.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

MASK_DIFF = 0
MASK_AR = 1
ATTN_DETERMINISTIC = 0x100  # OR into mask_mode: fixed key ranges, bitwise-repeatable output

OK, EINVAL, ESHAPE, EUNSUPPORTED, ECUDA, ECAPACITY, EWORKSPACE, EALIGN, ETIMEOUT = \
    0, -1, -2, -3, -4, -5, -6, -7, -8

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liborthrus.so")

_lock = threading.Lock()
_lib = None


class OrthrusError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status) if _lib else status}")


class KVCacheView(ctypes.Structure):
    """Mirror of ``orthrus_kv_cache`` (one layer of the shared KV cache)."""
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("ctx_lens", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("cap", ctypes.c_int),
                ("d", ctypes.c_int)]


def load(path: str | None = None):
    """Load the library once (raises if it is missing: build it first)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise OrthrusError(ECUDA, f"{p} not found; build it with "
                                      "`python -m lossless_block_drafting_b200.build`")
        lib = ctypes.CDLL(p)
        V, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        PSZ = ctypes.POINTER(ctypes.c_size_t)
        PC = ctypes.POINTER(KVCacheView)
        sig = {
            "orthrus_status_str": ([I], ctypes.c_char_p),
            "orthrus_abi_version": ([], I),
            "orthrus_set_wait_limit_ns": ([ctypes.c_uint64], I),
            "orthrus_block_attn_workspace_size": ([I, I, I, I, I, PSZ], I),
            "orthrus_block_attn": ([V, PC, I, I, I, V, V, SZ, V, V], I),
            "orthrus_prefill_attn": ([V, PC, I, I, V, V, V], I),
            "orthrus_lmhead_workspace_size": ([I, I, PSZ], I),
            "orthrus_lmhead_argmax": ([V, V, I, I, I, V, V, V, SZ, V, V], I),
            "orthrus_lmhead_argmax_noalloc": ([V, V, I, I, I, V, V, V, V], I),
            "orthrus_row_argmax_f32": ([V, I, I, V, V], I),
            "orthrus_verify": ([V, V, I, I, V, V, V], I),
            "orthrus_kv_commit": ([PC, V, I, V, V], I),
            "orthrus_verify_commit": ([V, V, I, I, V, V, PC, V, V], I),
            "orthrus_block_qkv_append": ([V, V, V, ctypes.c_float, ctypes.c_float, I, I, PC,
                                          V, V, V], I),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
        return lib


def set_wait_limit_ns(ns: int) -> None:
    """Limit after which a kernel's bounded waits give up (0 restores 2 s)."""
    _check(load().orthrus_set_wait_limit_ns(int(ns)), "orthrus_set_wait_limit_ns")


def status_str(status: int) -> str:
    return load().orthrus_status_str(int(status)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise OrthrusError(rc, what)


def _stream(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _on(stream):
    """Context for buffers a call allocates itself: on the launch stream, so a
    zero fill is ordered before the kernel and the caching allocator reuses a
    temporary only after that stream is done with it."""
    return contextlib.nullcontext() if stream is None else torch.cuda.stream(stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def kv_cache_view(k_cache, v_cache, ctx_lens) -> KVCacheView:
    """Describe one layer's cache: k/v bf16 [B, Hkv, cap, d], ctx_lens int32 [B]."""
    _need(k_cache, torch.bfloat16, "k_cache", 4)
    _need(v_cache, torch.bfloat16, "v_cache", 4)
    _need(ctx_lens, torch.int32, "ctx_lens", 1)
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    B, Hkv, cap, d = k_cache.shape
    if ctx_lens.shape[0] != B:
        raise ValueError("ctx_lens must be [B]")
    return KVCacheView(k_cache.data_ptr(), v_cache.data_ptr(), ctx_lens.data_ptr(), B, Hkv, cap, d)


def block_attn_workspace_size(B: int, Hq: int, Hkv: int, d: int, K: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().orthrus_block_attn_workspace_size(B, Hq, Hkv, d, K, ctypes.byref(n)),
           "orthrus_block_attn_workspace_size")
    return int(n.value)


def new_block_attn_workspace(B: int, Hq: int, Hkv: int, d: int, K: int, device=None):
    """A zero-filled workspace for block_attn (its barrier words must start at 0)."""
    return torch.zeros(block_attn_workspace_size(B, Hq, Hkv, d, K), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def block_attn(q, k_cache, v_cache, ctx_lens, mask_mode: int, out=None, workspace=None,
               dev_status=None, stream=None, cache_view: KVCacheView | None = None):
    """Block-query attention: q bf16 [B,K,Hq,d] over the cache -> bf16 [B,K,Hq,d]."""
    _need(q, torch.bfloat16, "q", 4)
    view = cache_view if cache_view is not None else kv_cache_view(k_cache, v_cache, ctx_lens)
    B, K, Hq, d = q.shape
    with _on(stream):
        if out is None:
            out = torch.empty_like(q)
        if workspace is None:
            workspace = new_block_attn_workspace(B, Hq, view.Hkv, d, K, q.device)
    _need(out, torch.bfloat16, "out", 4)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status")
    rc = load().orthrus_block_attn(_ptr(q), ctypes.byref(view), Hq, K, int(mask_mode), _ptr(out),
                                   _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                   _stream(stream))
    _check(rc, "orthrus_block_attn")
    return out


def prefill_attn(q, k_cache, v_cache, ctx_lens, out=None, dev_status=None, stream=None,
                 cache_view: KVCacheView | None = None):
    """Causal attention of a prompt chunk q bf16 [B, P, Hq, d] at positions
    ctx_lens[b] + i over the cache -> bf16 [B, P, Hq, d] (ctx_lens unchanged)."""
    _need(q, torch.bfloat16, "q", 4)
    view = cache_view if cache_view is not None else kv_cache_view(k_cache, v_cache, ctx_lens)
    B, P, Hq, d = q.shape
    if B != view.B or d != view.d:
        raise ValueError("q must be [B, P, Hq, d] of the cache's B and d")
    if out is None:
        with _on(stream):
            out = torch.empty_like(q)
    _need(out, torch.bfloat16, "out", 4)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status")
    rc = load().orthrus_prefill_attn(_ptr(q), ctypes.byref(view), Hq, P, _ptr(out),
                                     _ptr(dev_status), _stream(stream))
    _check(rc, "orthrus_prefill_attn")
    return out


def lmhead_workspace_size(R: int, V: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().orthrus_lmhead_workspace_size(R, V, ctypes.byref(n)),
           "orthrus_lmhead_workspace_size")
    return int(n.value)


def lmhead_argmax(h, W, argmax=None, max_logit=None, workspace=None, stream=None,
                  want_max: bool = False, dev_status=None):
    """Greedy token per row of h [R,H] under LM head W [V,H] (bf16) -> int32 [R]."""
    _need(h, torch.bfloat16, "h", 2)
    _need(W, torch.bfloat16, "W", 2)
    R, H = h.shape
    V, H2 = W.shape
    if H2 != H:
        raise ValueError("h and W hidden sizes differ")
    with _on(stream):
        if argmax is None:
            argmax = torch.empty(R, dtype=torch.int32, device=h.device)
        if want_max and max_logit is None:
            max_logit = torch.empty(R, dtype=torch.float32, device=h.device)
        if workspace is None:
            workspace = torch.empty(lmhead_workspace_size(R, V), dtype=torch.uint8,
                                    device=h.device)
    _need(argmax, torch.int32, "argmax", 1)
    if max_logit is not None:
        _need(max_logit, torch.float32, "max_logit", 1)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status")
    rc = load().orthrus_lmhead_argmax(_ptr(h), _ptr(W), R, H, V, _ptr(argmax), _ptr(max_logit),
                                      _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                      _stream(stream))
    _check(rc, "orthrus_lmhead_argmax")
    return (argmax, max_logit) if max_logit is not None else argmax


def lmhead_argmax_noalloc(h, W, argmax=None, max_logit=None, stream=None,
                          want_max: bool = False, dev_status=None):
    """lmhead_argmax without a caller workspace: the library's own fixed device
    scratch is used instead (shared by all calls; order overlapping calls on one
    stream, and make the first call on a device before any graph capture)."""
    _need(h, torch.bfloat16, "h", 2)
    _need(W, torch.bfloat16, "W", 2)
    R, H = h.shape
    V, H2 = W.shape
    if H2 != H:
        raise ValueError("h and W hidden sizes differ")
    with _on(stream):
        if argmax is None:
            argmax = torch.empty(R, dtype=torch.int32, device=h.device)
        if want_max and max_logit is None:
            max_logit = torch.empty(R, dtype=torch.float32, device=h.device)
    _need(argmax, torch.int32, "argmax", 1)
    if max_logit is not None:
        _need(max_logit, torch.float32, "max_logit", 1)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status")
    rc = load().orthrus_lmhead_argmax_noalloc(_ptr(h), _ptr(W), R, H, V, _ptr(argmax),
                                              _ptr(max_logit), _ptr(dev_status),
                                              _stream(stream))
    _check(rc, "orthrus_lmhead_argmax_noalloc")
    return (argmax, max_logit) if max_logit is not None else argmax


def row_argmax_f32(logits, argmax=None, stream=None):
    """Greedy index per row of fp32 logits [R, V] -> int32 [R]."""
    _need(logits, torch.float32, "logits", 2)
    R, V = logits.shape
    if argmax is None:
        with _on(stream):
            argmax = torch.empty(R, dtype=torch.int32, device=logits.device)
    _need(argmax, torch.int32, "argmax", 1)
    _check(load().orthrus_row_argmax_f32(_ptr(logits), R, V, _ptr(argmax), _stream(stream)),
           "orthrus_row_argmax_f32")
    return argmax


def verify(argmax, draft, accept_len=None, next_tok=None, stream=None):
    """Exact consensus: argmax, draft int32 [B,K] -> (accept_len, next_tok) int32 [B]."""
    _need(argmax, torch.int32, "argmax", 2)
    _need(draft, torch.int32, "draft", 2)
    if argmax.shape != draft.shape:
        raise ValueError("argmax and draft shapes differ")
    B, K = argmax.shape
    with _on(stream):
        if accept_len is None:
            accept_len = torch.empty(B, dtype=torch.int32, device=argmax.device)
        if next_tok is None:
            next_tok = torch.empty(B, dtype=torch.int32, device=argmax.device)
    _check(load().orthrus_verify(_ptr(argmax), _ptr(draft), B, K, _ptr(accept_len),
                                 _ptr(next_tok), _stream(stream)), "orthrus_verify")
    return accept_len, next_tok


def _lens_view(ctx_lens, cap: int) -> KVCacheView:
    _need(ctx_lens, torch.int32, "ctx_lens", 1)
    return KVCacheView(None, None, ctx_lens.data_ptr(), ctx_lens.shape[0], 0, int(cap), 0)


def kv_commit(ctx_lens, accept_len, K: int, cap: int, dev_status=None, stream=None):
    """ctx_lens[b] += min(accept_len[b] + 1, K) in place (clamped to cap)."""
    _need(accept_len, torch.int32, "accept_len", 1)
    view = _lens_view(ctx_lens, cap)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status")
    _check(load().orthrus_kv_commit(ctypes.byref(view), _ptr(accept_len), int(K),
                                    _ptr(dev_status), _stream(stream)), "orthrus_kv_commit")
    return ctx_lens


def verify_commit(argmax, draft, ctx_lens, cap: int, accept_len=None, next_tok=None,
                  dev_status=None, stream=None):
    """verify + kv_commit in one launch -> (accept_len, next_tok); ctx_lens updated."""
    _need(argmax, torch.int32, "argmax", 2)
    _need(draft, torch.int32, "draft", 2)
    B, K = argmax.shape
    with _on(stream):
        if accept_len is None:
            accept_len = torch.empty(B, dtype=torch.int32, device=argmax.device)
        if next_tok is None:
            next_tok = torch.empty(B, dtype=torch.int32, device=argmax.device)
    view = _lens_view(ctx_lens, cap)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status")
    _check(load().orthrus_verify_commit(_ptr(argmax), _ptr(draft), B, K, _ptr(accept_len),
                                        _ptr(next_tok), ctypes.byref(view), _ptr(dev_status),
                                        _stream(stream)), "orthrus_verify_commit")
    return accept_len, next_tok


def block_qkv_append(qkv, k_cache, v_cache, ctx_lens, Hq: int, K: int, q_norm_w=None,
                     k_norm_w=None, rope_theta: float = 1e6, rms_eps: float = 1e-6,
                     q_out=None, dev_status=None, stream=None,
                     cache_view: KVCacheView | None = None):
    """Per-head RMS norm of q/k, rotary embedding at L_b + i, block K/V into cache
    slots [L_b, L_b + K): qkv bf16 [B*K, (Hq + 2 Hkv) d] -> q_out bf16 [B, K, Hq, d]."""
    _need(qkv, torch.bfloat16, "qkv", 2)
    view = cache_view if cache_view is not None else kv_cache_view(k_cache, v_cache, ctx_lens)
    B, d = view.B, view.d
    if qkv.shape != (B * K, (Hq + 2 * view.Hkv) * d):
        raise ValueError("qkv must be [B*K, (Hq + 2 Hkv) d]")
    for w, name in ((q_norm_w, "q_norm_w"), (k_norm_w, "k_norm_w")):
        if w is not None:
            _need(w, torch.bfloat16, name, 1)
    if q_out is None:
        with _on(stream):
            q_out = torch.empty(B, K, Hq, d, dtype=torch.bfloat16, device=qkv.device)
    _need(q_out, torch.bfloat16, "q_out", 4)
    if dev_status is not None:
        _need(dev_status, torch.int32, "dev_status")
    rc = load().orthrus_block_qkv_append(_ptr(qkv), _ptr(q_norm_w), _ptr(k_norm_w),
                                         float(rope_theta), float(rms_eps), int(Hq), int(K),
                                         ctypes.byref(view), _ptr(q_out), _ptr(dev_status),
                                         _stream(stream))
    _check(rc, "orthrus_block_qkv_append")
    return q_out
