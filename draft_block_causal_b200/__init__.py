"""B200-native Domino head: greedy drafting, teacher-forced logits and greedy accept length.

The compute path is the C-ABI library ``libdomino.so`` (hand-written sm_100a CUDA kernels,
declared in ``include/domino.h``); :mod:`draft_block_causal_b200.domino` is a thin ctypes
binding over it.  :mod:`draft_block_causal_b200.synth` generates seeded synthetic inputs.

Importing the package loads nothing: the library is opened on first use, and every entry
point raises if it is missing -- there is no CPU fallback.
"""

__all__ = ["domino", "synth"]
