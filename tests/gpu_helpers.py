"""Shared helpers for the GPU parity tests (not a test module)."""
import numpy as np
import torch

import oracle
from full_gqa_attention_swa_b200 import api, inputs

# |gpu - oracle| <= ATOL + RTOL * |oracle|, elementwise (bf16 I/O, fp32 accumulate)
ATOL = 1e-2
RTOL = 1e-2


def oracle_layer(p: api.LayerParams) -> oracle.Layer:
    return oracle.Layer(p.num_q_heads, p.num_kv_heads, p.head_dim, p.window, p.rope_theta, p.rotary_dim,
                        p.softmax_scale, p.inv_freq)


def scaled_inv_freq(theta, r, factor=2.0, low=1.0, high=4.0, context=8192):
    """A long-context frequency table a caller would pass as inv_freq: the
    llama3-style rule (wavelengths shorter than context/high kept, longer
    than context/low divided by factor, a linear blend between).  The pages
    name this scaling for the full layers without its parameters, so the
    values here are test inputs, not a reading of them."""
    w = float(theta) ** (-2.0 * np.arange(r // 2) / r)
    wavelen = 2 * np.pi / w
    blend = np.clip((context / wavelen - low) / (high - low), 0.0, 1.0)
    return tuple(float(x) for x in (1.0 - blend) * w / factor + blend * w)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_close(gpu, ref: np.ndarray, what: str = ""):
    g = to_f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; max err "
                             f"{err.max():.3e}; first bad {idx.tolist()} gpu {g[tuple(idx[0])]} ref "
                             f"{ref[tuple(idx[0])]}")
    return {"max_abs": float(err.max()), "rms": float(np.sqrt((err ** 2).mean()))}


def bits(t):
    return inputs.as_bits(t)


def check_no_device_error():
    assert api.device_error(reset=True) == 0


def prefill_rows_sample(B, S, Hq, window, seed, n_random=64):
    """Seeded stratified sample of (b, i, h) rows: the first rows, rows at
    every band edge and tile edge near the window, the last rows, and random
    rows; every head appears."""
    rng = np.random.default_rng(seed)
    W = window if window > 0 else S
    pos = {0, 1, 2, 127, 128, 129, S - 1, S - 2, S - 128, S - 129}
    for base in (W - 2, W - 1, W, W + 1, W + 127, W + 128, W + 129, 2 * W - 1, 2 * W):
        pos.add(base)
    pos = sorted(p for p in pos if 0 <= p < S)
    rows = []
    for i, p in enumerate(pos):
        rows.append((i % B, p, (7 * i) % Hq))
    for _ in range(n_random):
        rows.append((int(rng.integers(B)), int(rng.integers(S)), int(rng.integers(Hq))))
    for h in range(Hq):
        rows.append((h % B, int(rng.integers(S)), h))
    return np.array(rows, np.int64)
