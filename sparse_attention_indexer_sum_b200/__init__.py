"""B200-native (sm_100a) hot path of DeepSeek Sparse Attention with IndexCache.

The compute lives in the C-ABI library ``libic_b200.so`` (hand-written CUDA for
sm_100a, declared in ``include/ic.h``); ``binding`` marshals torch tensors into
it.  Importing this package loads nothing: the library is opened on first use
and the call fails loudly if it is missing.
"""
__all__ = ["binding", "synth"]
