"""swa_attn_decode_mq on the GPU against the oracle: T new tokens per sequence
over ring and linear caches (empty, partial and full histories), every m-tile
count (T * G up to 64), single-split and split-K plans, NaN in slots outside
every band, the whole chain (chunked prefill writes the cache, RoPE of the new
tokens, multi-query decode) against whole-sequence prefill rows, and the
full-size Step workloads on seeded row samples."""
import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import api, configs, inputs
from gpu_helpers import assert_close, bits, check_no_device_error, oracle_layer

pytestmark = pytest.mark.gpu


def _run(cuda_device, p, B, T, C, lens, seed, gate=True, poison=False, scale=1.0):
    """Random cache of capacity C holding lens[b] - T earlier tokens, random
    (already rotated) new tokens; returns the GPU output and the oracle's.
    scale multiplies q and every key (scores grow with its square)."""
    d = inputs.decode_inputs(B, p.num_q_heads, p.num_kv_heads, 128, C, seed)
    new = inputs.prefill_inputs(B, T, p.num_q_heads, p.num_kv_heads, 128, seed + 1, with_gate=gate)
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    if scale != 1.0:
        new["q"] = (new["q"].float() * scale).to(torch.bfloat16)
        new["k"] = (new["k"].float() * scale).to(torch.bfloat16)
        kc = (kc.float() * scale).to(torch.bfloat16)
    if poison:   # slots outside every query's band hold NaN
        for b, L in enumerate(lens):
            L0 = L - T
            if p.window > 0:
                dead = [(L0 - p.window) % p.window] if L0 >= p.window else list(range(L0, p.window))
            else:
                dead = list(range(L0, C))
            kc[b, :, dead] = float("nan")
            vc[b, :, dead] = float("nan")
    lens_t = torch.tensor(lens, dtype=torch.int32)
    g = new["gate"]
    out = api.attn_decode_mq(p, new["q"].to(cuda_device), None if g is None else g.to(cuda_device),
                             new["k"].to(cuda_device), new["v"].to(cuda_device), kc.to(cuda_device),
                             vc.to(cuda_device), lens_t.to(cuda_device), max(lens))
    torch.cuda.synchronize()
    q64 = oracle.bf16_bits_to_f64(bits(new["q"]))
    ref = oracle.decode_mq(oracle_layer(p), q64, None if g is None else g.numpy(), bits(kc), bits(vc),
                           lens_t.numpy(), bits(new["k"]), bits(new["v"]))
    return out, ref


@pytest.mark.parametrize("T", [1, 2, 4])
@pytest.mark.parametrize("G", [1, 6, 12, 16])
@pytest.mark.parametrize("W", [32, 64, 100])
def test_sliding_ring(cuda_device, W, G, T):
    """Histories of 0, a few, W - 1, W, and many ring turns (every slot live,
    the oldest one outside every band)."""
    p = api.LayerParams(G * 2, 2, 128, W, 1e4, 128)
    lens = [T, T + 3, T + W - 1, T + W, T + 5 * W + 7]
    out, ref = _run(cuda_device, p, len(lens), T, W, lens, seed=2000 + W + 10 * G + T)
    assert_close(out, ref, f"mq ring W{W} G{G} T{T}")
    check_no_device_error()


@pytest.mark.parametrize("B,Hkv,G,W,T", [(1, 2, 8, 2048, 4), (2, 2, 8, 2048, 4), (39, 3, 4, 64, 3),
                                         (64, 1, 12, 512, 4)],
                         ids=["long-ring-splits", "long-and-short-ring", "many-rings", "full-rings"])
def test_ring_batches(cuda_device, B, Hkv, G, W, T):
    """Ring layers at other batch shapes: a long ring split over several CTAs
    (merged from their partials), a long and a short ring in one batch, many
    short rings, and a batch of full rings."""
    p = api.LayerParams(G * Hkv, Hkv, 128, W, 1e4, 128)
    rng = np.random.default_rng(2150 + B)
    if B == 1:
        lens = [T + 5000]
    elif B == 2:
        lens = [T + 5000, T + 100]
    else:
        lens = [int(x) for x in rng.integers(T, T + 5 * W, B)]
    out, ref = _run(cuda_device, p, B, T, W, lens, seed=2160 + B + W)
    assert_close(out, ref, f"mq ring batch B{B} Hkv{Hkv} G{G} W{W} T{T}")
    check_no_device_error()


@pytest.mark.parametrize("T", [1, 3, 4])
@pytest.mark.parametrize("G", [2, 8, 16])
def test_full_linear(cuda_device, G, T):
    """Linear cache, split-K plans (a short batch spreads 700 keys over
    several splits, so some splits hold no visible key for no row and the
    new tokens ride on the last one)."""
    p = api.LayerParams(G * 2, 2, 128, -1, 5e6, 64)
    lens = [T, T + 1, T + 299, 700]
    assert api.decode_mq_workspace_size(p, len(lens), T, max(lens)) > 0    # split-K plan
    out, ref = _run(cuda_device, p, len(lens), T, 700, lens, seed=2100 + G + T)
    assert_close(out, ref, f"mq linear G{G} T{T}")
    check_no_device_error()


@pytest.mark.parametrize("G,T", [(16, 4), (1, 16), (4, 16), (8, 8), (12, 5)])
def test_row_tiles(cuda_device, G, T):
    """One to four 16-row m-tiles, ragged last tiles, T up to 16."""
    for W, C in ((64, 64), (-1, 300)):
        p = api.LayerParams(G * 2, 2, 128, W, 1e4, 128)
        lens = [T, T + 40, T + 200] if W < 0 else [T + 1, T + 63, T + 64, T + 300]
        out, ref = _run(cuda_device, p, len(lens), T, C, lens, seed=2200 + G * T + max(W, 0))
        assert_close(out, ref, f"mq tiles G{G} T{T} W{W}")
    check_no_device_error()


def test_large_scores(cuda_device):
    for p, C, lens, seed in ((api.LayerParams(24, 2, 128, 64, 1e4, 128), 64, [4, 40, 68, 900], 830),
                             (api.LayerParams(16, 2, 128, -1, 5e6, 64), 9000, [4, 3000, 9000], 831)):
        out, ref = _run(cuda_device, p, len(lens), 4, C, lens, seed, scale=3.0)
        assert_close(out, ref, f"multi-query large scores W{p.window}")
    check_no_device_error()


def test_nan_outside_bands_and_no_gate(cuda_device):
    for W, C in ((64, 64), (-1, 500)):
        p = api.LayerParams(12, 1, 128, W, 1e4, 128)
        lens = [4, 9, 67, 68, 200] if W > 0 else [4, 9, 130, 404]
        out, ref = _run(cuda_device, p, len(lens), 4, C, lens, seed=2300 + max(W, 0), gate=False, poison=True)
        assert_close(out, ref, f"mq poison W{W}")
    check_no_device_error()


def test_one_query_matches_decode_after_append(cuda_device):
    """T = 1 is the one-query decode once the token is appended."""
    p = api.LayerParams(24, 2, 128, 64, 1e4, 128)
    B, lens = 4, [1, 20, 64, 300]
    d = inputs.decode_inputs(B, 24, 2, 128, 64, seed=2400)
    new = inputs.prefill_inputs(B, 1, 24, 2, 128, seed=2401)
    dev = {k: v.to(cuda_device) for k, v in new.items()}
    kc, vc = d["k_cache"].to(cuda_device), d["v_cache"].to(cuda_device)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    mq = api.attn_decode_mq(p, dev["q"], dev["gate"], dev["k"], dev["v"], kc, vc, lens_t, max(lens))
    pos = (lens_t - 1).reshape(B, 1)
    flat = api.LayerParams(24, 2, 128, 64, 0.0, 0)   # appends the given keys unchanged
    api.rope_qk(flat, k=dev["k"].clone(), pos=pos, v=dev["v"], k_cache=kc, v_cache=vc)
    one = api.attn_decode(p, dev["q"][:, 0].contiguous(), dev["gate"][:, 0].contiguous(), kc, vc, lens_t, max(lens))
    torch.cuda.synchronize()
    diff = (mq[:, 0].float() - one.float()).abs().max().item()
    assert diff <= 1e-2, diff
    check_no_device_error()


@pytest.mark.parametrize("W,theta,r", [(64, 1e4, 128), (-1, 5e6, 64)])
def test_chain_against_whole_sequence_prefill(cuda_device, W, theta, r):
    """Chunked prefill of the first L0 tokens writes the cache, swa_rope_qk
    rotates the T new tokens at L0 .. L0 + T - 1, multi-query decode attends:
    every row equals the whole-sequence prefill row at its position."""
    Hq, Hkv, B, L0, T = 12, 2, 2, 150, 4
    p = api.LayerParams(Hq, Hkv, 128, W, theta, r)
    L = L0 + T
    d = inputs.prefill_inputs(B, L, Hq, Hkv, 128, seed=2500 + max(W, 0))
    dev = {k: v.to(cuda_device) for k, v in d.items()}
    C = W if W > 0 else L
    kc = torch.zeros(B, Hkv, C, 128, dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    for a, b in ((0, 100), (100, L0)):
        api.attn_prefill_chunk(p, a, dev["q"][:, a:b].contiguous(), dev["k"][:, a:b].contiguous(),
                               dev["v"][:, a:b].contiguous(), dev["gate"][:, a:b].contiguous(), kc, vc)
    q = dev["q"][:, L0:].contiguous()
    k = dev["k"][:, L0:].contiguous()
    api.rope_qk(p, q=q, k=k, pos0=L0)
    lens = torch.full((B,), L, dtype=torch.int32, device=cuda_device)
    out = api.attn_decode_mq(p, q, dev["gate"][:, L0:].contiguous(), k, dev["v"][:, L0:].contiguous(), kc, vc,
                             lens, L)
    torch.cuda.synchronize()
    rows = np.array([(b, i, h) for b in range(B) for i in range(L0, L) for h in range(Hq)], np.int64)
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]), d["gate"].numpy(), rows=rows)
    assert_close(out.reshape(-1, 128), ref.reshape(-1, 128), f"mq chain W{W}")
    check_no_device_error()


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [configs.MQ_SLIDING, configs.MQ_FULL], ids=lambda c: c.name)
def test_full_size_sampled(cuda_device, cfg):
    """The multi-query decode workloads at full size (B64, T4, lengths
    U[4096, 131072]); the oracle checks a seeded sample of (b, t, h) rows."""
    p = api.LayerParams(cfg.Hq, cfg.Hkv, 128, cfg.window, cfg.theta, cfg.rotary_dim)
    lens = inputs.uniform_int(cfg.B, cfg.len_lo, cfg.len_hi, cfg.seed)
    d = inputs.decode_inputs(cfg.B, cfg.Hq, cfg.Hkv, 128, cfg.capacity, cfg.seed, device=cuda_device)
    new = inputs.prefill_inputs(cfg.B, cfg.T, cfg.Hq, cfg.Hkv, 128, cfg.seed + 1, device=cuda_device)
    out = api.attn_decode_mq(p, new["q"], new["gate"], new["k"], new["v"], d["k_cache"], d["v_cache"],
                             lens.to(cuda_device), int(lens.max()))
    torch.cuda.synchronize()
    rng = np.random.default_rng(cfg.seed)
    bsel = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] + list(rng.choice(cfg.B, 2, replace=False))))
    G = cfg.Hq // cfg.Hkv
    rows = np.array([(i, t, h) for i in range(len(bsel)) for t in range(cfg.T) for h in range(0, cfg.Hq, G // 2)],
                    np.int64)
    # copy only the sampled sequences' cached slots back for the oracle
    if cfg.window > 0:
        kc, vc, C = d["k_cache"][bsel].cpu(), d["v_cache"][bsel].cpu(), cfg.capacity
    else:
        C = max(int(lens[b]) - cfg.T for b in bsel)
        kc, vc = d["k_cache"][bsel, :, :C].cpu(), d["v_cache"][bsel, :, :C].cpu()
    q64 = oracle.bf16_bits_to_f64(bits(new["q"][bsel].cpu()))
    ref = oracle.decode_mq(oracle_layer(p), q64, new["gate"][bsel].cpu().numpy(), bits(kc), bits(vc),
                           lens[bsel].numpy(), bits(new["k"][bsel].cpu()), bits(new["v"][bsel].cpu()), rows=rows)
    bidx = torch.tensor([bsel[i] for i in rows[:, 0]])
    got = out.cpu()[bidx, torch.from_numpy(rows[:, 1]), torch.from_numpy(rows[:, 2])]
    assert_close(got, ref, cfg.name)
    check_no_device_error()
