"""The workloads, as the pages' models shape them.

Numbers only (no arithmetic of the method).  Sources (page title, section):

* "Step-3.7-Flash-oQ3e" explainer, sections 1, 2.2, 2.3: 64 q-heads / 8 KV
  groups, head_dim 128, sliding window 512 with 96 q-heads on sliding layers,
  rope_theta 5e6 on full layers and 1e4 on sliding ones, partial rotary 0.5
  on full layers.
* "Muse-Glimmer-30B-6bit" explainer, GQA / sliding-window / RoPE sections:
  32 q-heads / 2 KV heads, window 2048, rope theta 5e5 on sliding layers and
  0 (no rotation) on full layers, 128K context.
"""
from __future__ import annotations

from dataclasses import dataclass, field

WINDOW_FULL = -1


@dataclass(frozen=True)
class PrefillLayer:
    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    window: int
    theta: float
    rotary_dim: int
    seed: int


@dataclass(frozen=True)
class DecodeLayer:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    window: int
    theta: float
    rotary_dim: int
    len_lo: int
    len_hi: int
    capacity: int
    seed: int


@dataclass(frozen=True)
class ChunkLayer:
    """A continued prefill: S new tokens at positions pos0 .. pos0 + S - 1
    against a KV cache holding positions < pos0."""
    name: str
    B: int
    pos0: int
    S: int
    Hq: int
    Hkv: int
    D: int
    window: int
    theta: float
    rotary_dim: int
    seed: int


@dataclass(frozen=True)
class MultiQueryLayer:
    """Multi-query decode: T new tokens per sequence (lengths counting them
    uniform in [len_lo, len_hi]); the cache holds the earlier tokens."""
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int
    window: int
    theta: float
    rotary_dim: int
    len_lo: int
    len_hi: int
    capacity: int
    seed: int


# tiny oracle case: B1 S256 Hq8 Hkv1 W64, theta 1e4 on all 128 dims
TINY = PrefillLayer("tiny_B1_S256_Hq8_Hkv1_W64", 1, 256, 8, 1, 128, 64, 1e4, 128, 1000)

# Step-3.7-Flash sliding layer prefill
STEP_SLIDING = PrefillLayer("step37_sliding_B1_S8192_Hq96_Hkv8_W512", 1, 8192, 96, 8, 128, 512,
                            1e4, 128, 1001)

# Step-3.7-Flash full-attention layer prefill (partial rotary 0.5 -> 64 dims)
STEP_FULL = PrefillLayer("step37_full_B1_S32768_Hq64_Hkv8_causal", 1, 32768, 64, 8, 128,
                         WINDOW_FULL, 5e6, 64, 1002)

# Muse-Glimmer layers prefill: a sliding layer, then a full layer with no RoPE
MUSE_SLIDING = PrefillLayer("muse_sliding_B4_S16384_Hq32_Hkv2_W2048", 4, 16384, 32, 2, 128, 2048,
                            5e5, 128, 1003)
MUSE_FULL = PrefillLayer("muse_full_B4_S16384_Hq32_Hkv2_causal_norope", 4, 16384, 32, 2, 128,
                         WINDOW_FULL, 0.0, 128, 1003)

# batched decode, one query per sequence, context lengths U[4096, 131072]
DECODE_SLIDING = DecodeLayer("decode_sliding_B64_Hq96_Hkv8_W512", 64, 96, 8, 128, 512, 1e4, 128,
                             4096, 131072, 512, 1004)
DECODE_FULL = DecodeLayer("decode_full_B64_Hq64_Hkv8", 64, 64, 8, 128, WINDOW_FULL, 5e6, 64,
                          4096, 131072, 131072, 1004)

# multi-query decode of the Step layers: the token being decoded plus the
# three tokens that the spec card's three MTP layers (architecture notes)
# propose, T = 4
MQ_SLIDING = MultiQueryLayer("decode_mq_sliding_B64_T4_Hq96_Hkv8_W512", 64, 4, 96, 8, 128, 512, 1e4, 128,
                             4096, 131072, 512, 1007)
MQ_FULL = MultiQueryLayer("decode_mq_full_B64_T4_Hq64_Hkv8", 64, 4, 64, 8, 128, WINDOW_FULL, 5e6, 64,
                          4096, 131072, 131072, 1008)

# continued prefill: the second half of the Step sliding and full prefills,
# chunked against the cache the first half left
CHUNK_SLIDING = ChunkLayer("step37_sliding_chunk_B1_pos4096_S4096_Hq96_Hkv8_W512", 1, 4096, 4096, 96, 8, 128,
                           512, 1e4, 128, 1005)
CHUNK_FULL = ChunkLayer("step37_full_chunk_B1_pos16384_S16384_Hq64_Hkv8", 1, 16384, 16384, 64, 8, 128,
                        WINDOW_FULL, 5e6, 64, 1006)

PREFILL = {c.name: c for c in (TINY, STEP_SLIDING, STEP_FULL, MUSE_SLIDING, MUSE_FULL)}
CHUNK = {c.name: c for c in (CHUNK_SLIDING, CHUNK_FULL)}
DECODE = {c.name: c for c in (DECODE_SLIDING, DECODE_FULL)}
MULTI_QUERY = {c.name: c for c in (MQ_SLIDING, MQ_FULL)}
