"""B200-native attention core of a hybrid sliding-window / full-attention GQA
decoder layer: RoPE on Q and K, a banded causal mask (query i sees key j iff
i-W < j <= i; W infinite on full layers), GQA head sharing, online softmax,
P.V and a per-head sigmoid output gate.

The compute lives in ``libswa.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/swa.h``); ``full_gqa_attention_swa_b200.api`` is a thin
ctypes binding over it.  Importing the package loads nothing; the first call
into ``api`` loads the library and raises if it is missing.
"""
