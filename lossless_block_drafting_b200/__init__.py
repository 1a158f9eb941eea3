"""Orthrus dual-view decode-step hot path for NVIDIA B200 (sm_100a).

The compute lives in ``liborthrus.so`` (hand-written CUDA, C ABI declared in
``include/orthrus.h``); the Python functions in :mod:`.orthrus` only marshal
torch tensors into that ABI.  The library is loaded on first use and a missing
or unloadable library raises: there is no CPU fallback.

Modules: :mod:`.orthrus` (the binding), :mod:`.build` (compiles the library
in-tree), :mod:`.synth` (seeded synthetic inputs shared with the tests) and
:mod:`.toy_decode` (block decoding end to end on a random-weight toy model,
driving the library's kernels).
"""
