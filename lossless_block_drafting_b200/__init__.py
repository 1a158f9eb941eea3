"""Orthrus dual-view decode-step hot path for NVIDIA B200 (sm_100a).

The compute lives in ``liborthrus.so`` (hand-written CUDA, C ABI declared in
``include/orthrus.h``); the Python functions in :mod:`.orthrus` only marshal
torch tensors into that ABI.  The library is loaded on first use and a missing
or unloadable library raises: there is no CPU fallback.
"""
