"""Plain fp64 CPU oracle for the Orthrus dual-view decode step.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The CUDA
library never imports, links or executes anything here, and this package never
imports the CUDA library: the two share only the seeded input generators.

The arithmetic lives in ``orthrus_oracle.c`` (plain loops, fp64, OpenMP over
independent output rows).  This module only marshals arrays into it and builds
it with gcc on first use.  Functions accept numpy arrays (float64 / float32 /
int32) or CPU torch tensors; bf16 tensors are passed as their raw bits, which
the C code widens to fp64 exactly, so the oracle reads the same bits as the GPU.

Sources: the gist.science summary of "Orthrus: Memory-Efficient Parallel Token
Generation via Dual-View Diffusion" (technical summary sections 2.1-2.3), the
Hacker News thread "Orthrus-Qwen3: up to 7.8x tokens/forward on Qwen3, identical
output distribution" (post #21), and the paper's abstract.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "orthrus_oracle.c")
_SO = os.path.join(_HERE, "_build", "liborthrus_oracle.so")

F64, BF16, F32 = 0, 1, 2
MASK_DIFF, MASK_AR = 0, 1
OK, EINVAL, ENOMEM, ECAPACITY = 0, -1, -2, -5

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math) into oracle/_build."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_block_attn.argtypes = [P, I, P, P, I, P, I, I, I, I, I, I, I,
                                              ctypes.c_double, P, P]
            lib.oracle_lmhead_argmax.argtypes = [P, I, P, I, I, I, I, P, P, P]
            lib.oracle_row_argmax.argtypes = [P, I, I, I, P, P, P]
            lib.oracle_verify.argtypes = [P, P, I, I, P, P]
            lib.oracle_kv_commit.argtypes = [P, P, I, I, I, P]
            D = ctypes.c_double
            lib.oracle_qkv_append.argtypes = [P, I, P, P, I, D, D, P, I, I, I, I, I, I,
                                              P, P, P]
            for f in ("oracle_block_attn", "oracle_lmhead_argmax", "oracle_row_argmax",
                      "oracle_verify", "oracle_kv_commit", "oracle_version",
                      "oracle_num_threads", "oracle_qkv_append"):
                getattr(lib, f).restype = I
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_load().oracle_num_threads())


def _as_float_input(x):
    """Return (contiguous numpy array, dtype code) without changing any value."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:  # raw bf16 bits
        return x, BF16
    raise TypeError(f"unsupported oracle input dtype {x.dtype}")


def _as_i32(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x), dtype=np.int32)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def block_attn(q, k_cache, v_cache, ctx_lens, mask_mode: int, scale: float = 0.0,
               return_lse: bool = False):
    """Block-query attention (gist.science summary §2.1-2.3, items 1-2).

    q [B, K, Hq, d]; k_cache, v_cache [B, Hkv, cap, d]; ctx_lens [B].
    mask_mode MASK_DIFF: keys [0, L_b + K) (prefix + bidirectional block).
    mask_mode MASK_AR:   keys [0, L_b + i + 1) for block row i (causal).
    Returns fp64 [B, K, Hq, d] (and the natural-log LSE [B, K, Hq] if asked).
    """
    lib = _load()
    qa, qdt = _as_float_input(q)
    ka, kdt = _as_float_input(k_cache)
    va, vdt = _as_float_input(v_cache)
    if kdt != vdt:
        raise TypeError("k_cache and v_cache must share a dtype")
    cl = _as_i32(ctx_lens)
    B, K, Hq, d = qa.shape
    B2, Hkv, cap, d2 = ka.shape
    if (B2, d2) != (B, d) or va.shape != ka.shape or cl.shape != (B,):
        raise ValueError("shape mismatch")
    out = np.empty((B, K, Hq, d), np.float64)
    lse = np.empty((B, K, Hq), np.float64) if return_lse else None
    rc = lib.oracle_block_attn(_ptr(qa), qdt, _ptr(ka), _ptr(va), kdt, _ptr(cl), B, K, Hq,
                               Hkv, cap, d, int(mask_mode), float(scale), _ptr(out), _ptr(lse))
    if rc != OK:
        raise ValueError(f"oracle_block_attn failed with status {rc}")
    return (out, lse) if return_lse else out


def lmhead_argmax(h, W):
    """LM head + greedy choice (gist.science summary §2.3 items 2-3).

    h [R, H], W [V, H] -> (argmax int32 [R], top1 fp64 [R], gap fp64 [R]) where
    gap is the top-1 minus top-2 logit (0 on an exact tie, lowest index wins).
    """
    lib = _load()
    ha, hdt = _as_float_input(h)
    wa, wdt = _as_float_input(W)
    R, H = ha.shape
    V, H2 = wa.shape
    if H2 != H:
        raise ValueError("hidden size mismatch")
    am = np.empty(R, np.int32)
    top1 = np.empty(R, np.float64)
    gap = np.empty(R, np.float64)
    rc = lib.oracle_lmhead_argmax(_ptr(ha), hdt, _ptr(wa), wdt, R, H, V, _ptr(am),
                                  _ptr(top1), _ptr(gap))
    if rc != OK:
        raise ValueError(f"oracle_lmhead_argmax failed with status {rc}")
    return am, top1, gap


def row_argmax(logits):
    """Greedy choice over given logits [R, V] -> (argmax, top1, gap)."""
    lib = _load()
    la, dt = _as_float_input(logits)
    R, V = la.shape
    am = np.empty(R, np.int32)
    top1 = np.empty(R, np.float64)
    gap = np.empty(R, np.float64)
    rc = lib.oracle_row_argmax(_ptr(la), dt, R, V, _ptr(am), _ptr(top1), _ptr(gap))
    if rc != OK:
        raise ValueError(f"oracle_row_argmax failed with status {rc}")
    return am, top1, gap


def verify(argmax, draft):
    """Exact consensus (gist.science summary §2.3 item 3; HN thread post #21).

    argmax, draft [B, K] -> (accept_len int32 [B], next_tok int32 [B]).
    """
    lib = _load()
    am = _as_i32(argmax)
    dr = _as_i32(draft)
    if am.shape != dr.shape or am.ndim != 2:
        raise ValueError("argmax and draft must both be [B, K]")
    B, K = am.shape
    acc = np.empty(B, np.int32)
    nxt = np.empty(B, np.int32)
    rc = lib.oracle_verify(_ptr(am), _ptr(dr), B, K, _ptr(acc), _ptr(nxt))
    if rc != OK:
        raise ValueError(f"oracle_verify failed with status {rc}")
    return acc, nxt


def kv_commit(ctx_lens, accept_len, K: int, cap: int):
    """Length-pointer commit (gist.science summary §2.3 item 3; abstract: O(1)).

    Returns (new ctx_lens int32 [B], status) with L_b += min(a_b + 1, K),
    clamped to cap (status ECAPACITY) and a_b outside [0, K] rejected (EINVAL).
    """
    lib = _load()
    cl = _as_i32(ctx_lens).copy()
    acc = _as_i32(accept_len)
    B = cl.shape[0]
    st = np.zeros(1, np.int32)
    rc = lib.oracle_kv_commit(_ptr(cl), _ptr(acc), B, int(K), int(cap), _ptr(st))
    if rc != OK:
        raise ValueError(f"oracle_kv_commit failed with status {rc}")
    return cl, int(st[0])


def qkv_append(qkv, ctx_lens, K: int, Hq: int, Hkv: int, d: int, k_cache, v_cache,
               q_norm_w=None, k_norm_w=None, theta: float = 1e6, eps: float = 1e-6):
    """Block Q/K/V append: per-head RMS norm of q and k (if weights are given),
    rotary embedding at positions L_b + i, K/V written into slots [L_b, L_b + K).

    qkv [B*K, (Hq + 2 Hkv) d] (token-major, heads packed q | k | v); ctx_lens [B];
    k_cache, v_cache fp64 [B, Hkv, cap, d], updated in place (a copy is made if
    they are not writable fp64 arrays, and the updated arrays are returned).
    Returns (q_out fp64 [B, K, Hq, d], k_cache, v_cache).
    """
    lib = _load()
    xa, xdt = _as_float_input(qkv)
    cl = _as_i32(ctx_lens)
    B = cl.shape[0]
    if xa.shape != (B * K, (Hq + 2 * Hkv) * d):
        raise ValueError("qkv shape mismatch")
    kc = np.ascontiguousarray(np.asarray(k_cache, dtype=np.float64)).copy()
    vc = np.ascontiguousarray(np.asarray(v_cache, dtype=np.float64)).copy()
    if kc.shape != vc.shape or kc.shape[:2] != (B, Hkv) or kc.shape[3] != d:
        raise ValueError("cache shape mismatch")
    cap = kc.shape[2]
    qw = kw = None
    wdt = F64
    if q_norm_w is not None or k_norm_w is not None:
        if q_norm_w is None or k_norm_w is None:
            raise ValueError("give both norm weights or neither")
        qw, wdt = _as_float_input(q_norm_w)
        kw, wdt2 = _as_float_input(k_norm_w)
        if wdt2 != wdt:
            raise TypeError("norm weights must share a dtype")
    q_out = np.empty((B, K, Hq, d), np.float64)
    rc = lib.oracle_qkv_append(_ptr(xa), xdt, _ptr(qw), _ptr(kw), wdt, float(theta),
                               float(eps), _ptr(cl), B, K, Hq, Hkv, d, cap, _ptr(q_out),
                               _ptr(kc), _ptr(vc))
    if rc != OK:
        raise ValueError(f"oracle_qkv_append failed with status {rc}")
    return q_out, kc, vc
