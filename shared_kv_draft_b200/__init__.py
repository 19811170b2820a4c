"""Orthrus dual-view decode step on B200 (sm_100a).

The compute path is the C-ABI library ``liborthrus.so`` (hand-written CUDA for
sm_100a, declared in ``include/orthrus.h``); ``shared_kv_draft_b200.orthrus``
is its ctypes binding. Build the library with ``python -m shared_kv_draft_b200.build``.
"""
__all__ = ["orthrus", "build"]
