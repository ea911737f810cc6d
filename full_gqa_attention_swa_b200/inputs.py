"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module draws numbers and nothing else: it holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it without sharing any method code.

Distribution (the pages give no data; the workloads only fix shapes): Q, K,
V and cache entries are N(0, 1) rounded to bf16; gate logits are N(0, 1) in
fp32; decode context lengths are uniform integers in [lo, hi].  Every tensor
has its own seed derived from the workload seed and a tensor tag, so a
tensor's values do not depend on which other tensors were drawn.

Tensors are drawn on the CPU (torch's CPU generator) unless ``device`` is a
CUDA device, in which case torch's CUDA generator draws them in place; the
big decode caches are drawn that way, and the oracle then reads a copy of
exactly those values.
"""
from __future__ import annotations

import torch

_TAGS = {"q": 1, "k": 2, "v": 3, "gate": 4, "k_cache": 5, "v_cache": 6, "seq_lens": 7,
         "k_new": 8, "v_new": 9, "perm": 10}


def sub_seed(seed: int, tag: str) -> int:
    return (int(seed) * 1_000_003 + _TAGS[tag] * 7919) & 0x7FFF_FFFF_FFFF


def _gen(seed: int, tag: str, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(sub_seed(seed, tag))
    return g


def normal_bf16(shape, seed: int, tag: str, device="cpu") -> torch.Tensor:
    """N(0,1) drawn in fp32, rounded to bf16 (round-to-nearest-even)."""
    dev = torch.device(device)
    x = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    if x.numel() == 0:
        return x
    # draw in slabs so huge caches never need a full fp32 copy
    flat = x.view(-1)
    g = _gen(seed, tag, dev)
    slab = 1 << 26
    for s in range(0, flat.numel(), slab):
        n = min(slab, flat.numel() - s)
        flat[s:s + n] = torch.randn(n, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    return x


def normal_f32(shape, seed: int, tag: str, device="cpu") -> torch.Tensor:
    dev = torch.device(device)
    return torch.randn(shape, generator=_gen(seed, tag, dev), device=dev, dtype=torch.float32)


def uniform_int(n: int, lo: int, hi: int, seed: int, tag: str = "seq_lens") -> torch.Tensor:
    """n integers uniform in [lo, hi] (inclusive), int32, on the CPU."""
    g = _gen(seed, tag, "cpu")
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64).to(torch.int32)


def permutation(n: int, seed: int) -> torch.Tensor:
    g = _gen(seed, "perm", "cpu")
    return torch.randperm(n, generator=g)


def prefill_inputs(B: int, S: int, Hq: int, Hkv: int, D: int, seed: int, device="cpu",
                   with_gate: bool = True) -> dict:
    """q [B,S,Hq,D], k/v [B,S,Hkv,D] bf16; gate [B,S,Hq] fp32 (or None)."""
    return {
        "q": normal_bf16((B, S, Hq, D), seed, "q", device),
        "k": normal_bf16((B, S, Hkv, D), seed, "k", device),
        "v": normal_bf16((B, S, Hkv, D), seed, "v", device),
        "gate": normal_f32((B, S, Hq), seed, "gate", device) if with_gate else None,
    }


def decode_inputs(B: int, Hq: int, Hkv: int, D: int, capacity: int, seed: int, device="cpu",
                  fill_len=None) -> dict:
    """q [B,Hq,D] bf16 (taken as already rotated), gate [B,Hq] fp32, and a
    cache pair [B,Hkv,capacity,D] bf16 of N(0,1) entries.

    fill_len (optional [B] ints): slots at or beyond fill_len[b] are zeroed
    instead of drawn, so a full-capacity cache need not be drawn entirely.
    """
    dev = torch.device(device)
    kc = normal_bf16((B, Hkv, capacity, D), seed, "k_cache", dev)
    vc = normal_bf16((B, Hkv, capacity, D), seed, "v_cache", dev)
    if fill_len is not None:
        for b, n in enumerate(list(fill_len)):
            n = int(n)
            if n < capacity:
                kc[b, :, n:].zero_()
                vc[b, :, n:].zero_()
    return {
        "q": normal_bf16((B, Hq, D), seed, "q", dev),
        "gate": normal_f32((B, Hq), seed, "gate", dev),
        "k_cache": kc,
        "v_cache": vc,
    }


def as_bits(t: torch.Tensor):
    """A bf16 tensor's bit patterns as a numpy uint16 array (CPU copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
