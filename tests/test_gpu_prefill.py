"""swa_attn_prefill on the GPU against the oracle: the tiny case in full,
window sweeps around tile edges, ragged lengths, partial / no RoPE, odd GQA
groups, no gate, large and steadily growing scores (the lazy rescale), the uniform-score window-count probe at full size, and the
full-size prefill workloads on seeded row samples."""
import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import api, configs, inputs
from gpu_helpers import (assert_close, bits, check_no_device_error, oracle_layer, prefill_rows_sample,
                         scaled_inv_freq)

pytestmark = pytest.mark.gpu


def _layer(c):
    return api.LayerParams(c.Hq, c.Hkv, 128, c.window, c.theta, c.rotary_dim)


def _check_all_rows(cuda_device, p, B, S, seed, gate=True):
    d = inputs.prefill_inputs(B, S, p.num_q_heads, p.num_kv_heads, 128, seed, with_gate=gate)
    dev = {k: (None if t is None else t.to(cuda_device)) for k, t in d.items()}
    out = api.attn_prefill(p, dev["q"], dev["k"], dev["v"], dev["gate"])
    torch.cuda.synchronize()
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]),
                         None if d["gate"] is None else d["gate"].numpy())
    return assert_close(out, ref, f"prefill B{B} S{S} W{p.window}")


def test_tiny_config_all_rows(cuda_device):
    c = configs.TINY
    stats = _check_all_rows(cuda_device, _layer(c), c.B, c.S, c.seed)
    assert stats["max_abs"] < 1e-2
    check_no_device_error()


@pytest.mark.parametrize("W", [1, 2, 63, 64, 65, 127, 128, 129, 300, -1])
@pytest.mark.parametrize("Hq", [4, 8])  # G = 2: one head pair per tile; G = 4: two pairs per (q-tile, kv-head)
def test_window_sweep(cuda_device, W, Hq):
    p = api.LayerParams(Hq, 2, 128, W, 1e4, 128)
    _check_all_rows(cuda_device, p, 1, 300, seed=100 + max(W, 0))
    check_no_device_error()


@pytest.mark.parametrize("W", [128, 256, 384, 512])
def test_band_edge_on_tile_boundary(cuda_device, W):
    """W a multiple of 128: for query tiles at or past position W the band's
    first key tile is visible exactly above each row's diagonal and the
    diagonal key tile exactly on and below it, the two masks complementary.
    Every row is checked, with a ragged last tile and two head pairs per
    kv-head."""
    p = api.LayerParams(8, 2, 128, W, 1e4, 128)
    _check_all_rows(cuda_device, p, 1, 1100, seed=900 + W)
    check_no_device_error()


@pytest.mark.parametrize("S", [1, 17, 128, 129, 255, 257, 640])
@pytest.mark.parametrize("W", [64, -1])
def test_ragged_lengths(cuda_device, S, W):
    p = api.LayerParams(4, 1, 128, W, 1e4, 128)
    _check_all_rows(cuda_device, p, 2, S, seed=200 + S)
    check_no_device_error()


@pytest.mark.parametrize("theta,r", [(5e6, 64), (0.0, 128), (5e5, 32), (1e4, 16), (1e4, 24), (1e4, 6), (1e4, 2),
                                     (1e4, 0), (1e4, 48), (1e4, 80), (5e5, 112)])
def test_rope_variants(cuda_device, theta, r):
    """Partial rotary widths through the in-kernel Q rotation: the vector form
    splits a row's 8-pair chunks between the two head slots (48, 80 and 112
    give the slots unequal counts; 16 leaves slot 1 none), widths not a
    multiple of 16 take the scalar form."""
    p = api.LayerParams(8, 2, 128, 200, theta, r)
    _check_all_rows(cuda_device, p, 1, 384, seed=300 + r)
    check_no_device_error()


@pytest.mark.parametrize("W,theta,r", [(-1, 5e6, 64), (200, 1e4, 128), (-1, 0.0, 32)])
def test_frequency_table(cuda_device, W, theta, r):
    """Caller-scaled RoPE (the full layers' long-context scaling) through the
    in-kernel Q rotation and the cos/sin table."""
    table = scaled_inv_freq(theta if theta > 0 else 1e4, r)
    p = api.LayerParams(8, 2, 128, W, theta, r, inv_freq=table)
    _check_all_rows(cuda_device, p, 1, 384, seed=350 + r)
    check_no_device_error()


@pytest.mark.parametrize("Hq,Hkv", [(6, 2), (2, 2), (3, 1), (16, 1), (8, 1), (12, 1)])
def test_gqa_groups(cuda_device, Hq, Hkv):
    p = api.LayerParams(Hq, Hkv, 128, 100, 1e4, 128)
    _check_all_rows(cuda_device, p, 3, 200, seed=400 + Hq)
    check_no_device_error()


def test_no_gate_and_custom_scale(cuda_device):
    _check_all_rows(cuda_device, api.LayerParams(4, 2, 128, 50, 1e4, 128), 2, 160, seed=501, gate=False)
    _check_all_rows(cuda_device, api.LayerParams(4, 2, 128, -1, 1e4, 128, softmax_scale=0.05), 1, 200, seed=502)
    check_no_device_error()


def _score_extreme_inputs(kind, B, S, Hq, Hkv, seed):
    """Inputs whose scores stress the online softmax.  'large': q and k times
    3, so scores have a standard deviation near 9 (natural units) and a few
    keys dominate each row.  'growing': every query and key points along one
    direction, keys lengthening linearly with position, so a row's running
    max climbs about 6 (log2 units) per 128-key tile -- under the kernel's
    rescale threshold of 8 for one tile, over it across two."""
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed)
    if kind == "large":
        d["q"] = (d["q"].float() * 3).to(torch.bfloat16)
        d["k"] = (d["k"].float() * 3).to(torch.bfloat16)
    else:
        ramp = torch.arange(S, dtype=torch.float32).view(1, S, 1, 1) / S
        d["q"] = (1.41 + 0.1 * d["q"].float()).to(torch.bfloat16)
        d["k"] = (1.41 * ramp + 0.1 * d["k"].float()).to(torch.bfloat16)
    return d


@pytest.mark.parametrize("kind,W,theta", [("large", 300, 1e4), ("large", -1, 1e4), ("growing", 300, 0.0),
                                          ("growing", -1, 0.0)])
def test_score_extremes(cuda_device, kind, W, theta):
    """The kernels round the rotated q and k to bf16 before their MMAs.  At
    these score magnitudes that rounding alone moves the exact attention
    output by up to about 6e-2 (the oracle fed rounded operands shows the same
    shift), so with RoPE on, the reference is the oracle's rotation rounded to
    bf16 and then attended without rotation; with theta = 0 both sides see
    identical operands and the reference is the plain oracle."""
    B, S, Hq, Hkv = 2, 700, 4, 2
    p = api.LayerParams(Hq, Hkv, 128, W, theta, 128)
    d = _score_extreme_inputs(kind, B, S, Hq, Hkv, seed=720 + (W > 0))
    dev = {k: t.to(cuda_device) for k, t in d.items()}
    out = api.attn_prefill(p, dev["q"], dev["k"], dev["v"], dev["gate"])
    torch.cuda.synchronize()
    q, k = bits(d["q"]), bits(d["k"])
    lay = oracle_layer(p)
    if theta > 0:
        pos = np.arange(S, dtype=np.int64)
        rot = lambda x: bits(torch.from_numpy(
            np.stack([oracle.rope(x[b], pos, theta, 128) for b in range(B)])).to(torch.bfloat16))
        q, k = rot(q), rot(k)
        lay = oracle.Layer(Hq, Hkv, 128, W, 0.0, 128)
    ref = oracle.prefill(lay, q, k, bits(d["v"]), d["gate"].numpy())
    assert_close(out, ref, f"prefill {kind} W{W}")
    check_no_device_error()


@pytest.mark.parametrize("W,theta,r,table", [(200, 1e4, 128, False), (-1, 5e6, 64, False), (-1, 5e6, 64, True),
                                             (96, 5e5, 24, False)])
def test_in_kernel_rotation_equals_rope_qk_bitwise(cuda_device, W, theta, r, table):
    """The in-kernel Q rotation and the key pre-pass round exactly as
    swa_rope_qk does: prefill with RoPE equals, bit for bit, prefill without
    rotation on q and k rotated beforehand by swa_rope_qk."""
    B, S, Hq, Hkv = 2, 333, 8, 2
    freq = scaled_inv_freq(theta, r) if table else None
    p = api.LayerParams(Hq, Hkv, 128, W, theta, r, inv_freq=freq)
    plain = api.LayerParams(Hq, Hkv, 128, W, 0.0, r)
    d = {k: t.to(cuda_device) for k, t in inputs.prefill_inputs(B, S, Hq, Hkv, 128, 780 + r).items()}
    out = api.attn_prefill(p, d["q"], d["k"], d["v"], d["gate"])
    q, k = d["q"].clone(), d["k"].clone()
    api.rope_qk(p, q=q, k=k)
    out_pre = api.attn_prefill(plain, q, k, d["v"], d["gate"])
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out_pre.view(torch.int16))
    check_no_device_error()


def test_saturated_gate_logits(cuda_device):
    """Gate logits of +-60 and +-1e4 saturate the sigmoid: the output is the
    ungated attention, about 1e-26 of it (sigmoid(-60)), or exactly zero
    (sigmoid(-1e4) underflows), never NaN."""
    B, S, Hq, Hkv = 1, 300, 8, 2
    p = api.LayerParams(Hq, Hkv, 128, 100, 1e4, 128)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, 760)
    levels = torch.tensor([60.0, -60.0, 1e4, -1e4, 0.0, 3.0, -3.0, 60.0])
    d["gate"] = levels.view(1, 1, Hq).expand(B, S, Hq).contiguous()
    dev = {k: t.to(cuda_device) for k, t in d.items()}
    out = api.attn_prefill(p, dev["q"], dev["k"], dev["v"], dev["gate"])
    torch.cuda.synchronize()
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]), d["gate"].numpy())
    assert_close(out, ref, "prefill saturated gates")
    assert bool((out[:, :, 3] == 0).all()) and bool((out[:, :, 1].float().abs() < 1e-20).all())
    check_no_device_error()


@pytest.mark.parametrize("cfg", [configs.STEP_SLIDING, configs.MUSE_SLIDING], ids=lambda c: c.name)
def test_uniform_score_probe_window_counts(cuda_device, cfg):
    """Q = 0 makes every score 0: each output row is sigmoid(g) times the mean
    of the visible values.  With one-hot values e_(j mod 128) every output dim
    counts visible keys, so an off-by-one anywhere in the band shows, at the
    full workload size."""
    B, S = min(cfg.B, 2), cfg.S
    p = _layer(cfg)
    q = torch.zeros(B, S, cfg.Hq, 128, dtype=torch.bfloat16, device=cuda_device)
    k = inputs.normal_bf16((B, S, cfg.Hkv, 128), cfg.seed, "k", cuda_device)
    v = torch.zeros(B, S, cfg.Hkv, 128, dtype=torch.bfloat16, device=cuda_device)
    j = torch.arange(S, device=cuda_device)
    v[:, j, :, j % 128] = 1.0
    gate = torch.zeros(B, S, cfg.Hq, device=cuda_device)
    out = api.attn_prefill(p, q, k, v, gate)
    torch.cuda.synchronize()
    W = cfg.window
    i = np.arange(S)
    lo = np.maximum(0, i - W + 1)
    n = i - lo + 1
    # count of j in [lo, i] with j % 128 == d, for every d
    d = np.arange(128)
    def count_upto(x):  # number of j in [0, x) with j % 128 == d
        return (x[:, None] // 128) + ((x[:, None] % 128) > d[None, :])
    counts = count_upto(i + 1) - count_upto(lo)
    expect = 0.5 * counts / n[:, None]                               # [S, 128]
    got = out.float().cpu().numpy()                                  # [B,S,Hq,128]
    # within one bf16 ulp: the kernel rounds 0.5/n and count*(0.5/n) in fp32
    # before bf16; one key too many or too few moves the dim that gains or
    # loses it by a whole count (>= 6% here)
    e = np.broadcast_to(expect[None, :, None, :], got.shape)
    bad = np.abs(got - e) > 2.0 ** -8 * np.abs(e)
    assert not bad.any(), f"window count mismatch at {np.argwhere(bad)[:5].tolist()}"
    check_no_device_error()


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [configs.STEP_SLIDING, configs.STEP_FULL, configs.MUSE_SLIDING,
                                 configs.MUSE_FULL], ids=lambda c: c.name)
def test_full_size_sampled_rows(cuda_device, cfg):
    p = _layer(cfg)
    d = inputs.prefill_inputs(cfg.B, cfg.S, cfg.Hq, cfg.Hkv, 128, cfg.seed)
    dev = {k: t.to(cuda_device) for k, t in d.items()}
    out = api.attn_prefill(p, dev["q"], dev["k"], dev["v"], dev["gate"])
    torch.cuda.synchronize()
    rows = prefill_rows_sample(cfg.B, cfg.S, cfg.Hq, cfg.window, cfg.seed)
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]), d["gate"].numpy(), rows=rows)
    got = out.cpu()[torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1]), torch.from_numpy(rows[:, 2])]
    assert_close(got, ref, cfg.name)
    check_no_device_error()


@pytest.mark.parametrize("Hq,Hkv,W,B", [(16, 2, 512, 4), (16, 2, -1, 4), (4, 2, 300, 8), (12, 1, 200, 8)],
                         ids=["pair-sliding", "pair-causal", "single-sliding", "pair-G12"])
def test_persistent_multi_tile(cuda_device, Hq, Hkv, W, B):
    """More work tiles than CTAs: every persistent CTA runs several tiles
    back to back, so tile boundaries inside one persistent CTA are checked."""
    S, seed = 2048, 700 + Hq + B
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed)
    dev = {k: t.to(cuda_device) for k, t in d.items()}
    out = api.attn_prefill(p, dev["q"], dev["k"], dev["v"], dev["gate"])
    torch.cuda.synchronize()
    rows = prefill_rows_sample(B, S, Hq, W, seed, n_random=160)
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]), d["gate"].numpy(), rows=rows)
    got = out.cpu()[torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1]), torch.from_numpy(rows[:, 2])]
    assert_close(got, ref, f"multi-tile Hq{Hq} Hkv{Hkv} W{W} B{B}")
    check_no_device_error()


@pytest.mark.slow
def test_q_and_out_beyond_2_31_elements(cuda_device):
    """Maximum-size indexing: B2 S69632 Hq128 puts 2^31 + 2^27 elements in q
    and out (4.6 GB each), so every 64-bit offset (rows, gate, cos/sin table,
    output) is exercised; a W64 band keeps the work small.  Sampled rows
    include the last rows of the second sequence."""
    B, S, Hq, Hkv, W = 2, 69632, 128, 8, 64
    assert B * S * Hq * 128 > 2 ** 31
    p = api.LayerParams(Hq, Hkv, 128, W, 5e5, 128)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=760, device=cuda_device)
    out = api.attn_prefill(p, d["q"], d["k"], d["v"], d["gate"])
    torch.cuda.synchronize()
    rows = prefill_rows_sample(B, S, Hq, W, 760, n_random=96)
    rows = np.concatenate([rows, np.array([(1, S - 1, Hq - 1), (1, S - 1, 0), (1, S - 129, 77)], np.int64)])
    got = out[torch.from_numpy(rows[:, 0]).to(cuda_device), torch.from_numpy(rows[:, 1]).to(cuda_device),
              torch.from_numpy(rows[:, 2]).to(cuda_device)].cpu()
    del out
    q = bits(d["q"].cpu())
    ref = oracle.prefill(oracle_layer(p), q, bits(d["k"].cpu()), bits(d["v"].cpu()), d["gate"].cpu().numpy(),
                         rows=rows)
    assert_close(got, ref, "q/out beyond 2^31 elements")
    check_no_device_error()


@pytest.mark.parametrize("S", [5, 37])
def test_many_short_sequences(cuda_device, S):
    """B = 300 sequences of a few tokens: one ragged 128-row tile per
    (sequence, head pair); the loads read zeros past S and the stores clip
    there, so neighbouring sequences are left intact."""
    B, Hq, Hkv = 300, 8, 2
    for W in (3, -1):
        p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
        d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=800 + S)
        dev = {k: t.to(cuda_device) for k, t in d.items()}
        out = api.attn_prefill(p, dev["q"], dev["k"], dev["v"], dev["gate"])
        torch.cuda.synchronize()
        rng = np.random.default_rng(S)
        rows = np.stack([rng.integers(0, B, 200), rng.integers(0, S, 200), rng.integers(0, Hq, 200)], 1)
        rows = np.concatenate([rows, np.array([(0, 0, 0), (B - 1, S - 1, Hq - 1)], np.int64)]).astype(np.int64)
        ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]), d["gate"].numpy(), rows=rows)
        got = out.cpu()[torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1]), torch.from_numpy(rows[:, 2])]
        assert_close(got, ref, f"B{B} S{S} W{W}")
    check_no_device_error()
