"""swa_attn_decode on the GPU against the oracle: ring caches (sliding) and
linear caches (full), single-split and split-K paths, NaN in unused slots,
the rope+append+decode chain, and the full-size batched decode workload."""
import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import api, configs, inputs
from gpu_helpers import assert_close, bits, check_no_device_error, oracle_layer

pytestmark = pytest.mark.gpu


def _run(cuda_device, p, B, C, lens, seed, gate=True, poison=False, rows=None, scale=1.0):
    """scale multiplies q and the cached keys (scores grow with its square)."""
    d = inputs.decode_inputs(B, p.num_q_heads, p.num_kv_heads, 128, C, seed)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    if scale != 1.0:
        d["q"] = (d["q"].float() * scale).to(torch.bfloat16)
        kc = (kc.float() * scale).to(torch.bfloat16)
    if poison:   # slots nobody may read hold NaN
        for b, L in enumerate(lens):
            n = min(L, p.window) if p.window > 0 else L
            kc[b, :, n:] = float("nan")
            vc[b, :, n:] = float("nan")
    g = d["gate"] if gate else None
    out = api.attn_decode(p, d["q"].to(cuda_device), None if g is None else g.to(cuda_device),
                          kc.to(cuda_device), vc.to(cuda_device), lens_t.to(cuda_device), max(lens))
    torch.cuda.synchronize()
    q64 = oracle.bf16_bits_to_f64(bits(d["q"]))
    ref = oracle.decode(oracle_layer(p), q64, None if g is None else g.numpy(), bits(kc), bits(vc),
                        lens_t.numpy(), rows=rows)
    if rows is not None:
        got = out.cpu()[torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1])]
        return assert_close(got, ref, "decode rows")
    return assert_close(out, ref, "decode")


@pytest.mark.parametrize("G", [1, 6, 12, 16])
def test_sliding_ring(cuda_device, G):
    Hkv = 2
    p = api.LayerParams(G * Hkv, Hkv, 128, 64, 1e4, 128)
    _run(cuda_device, p, 6, 64, [1, 10, 63, 64, 65, 1000], seed=50 + G)
    check_no_device_error()


@pytest.mark.parametrize("G", [1, 8, 16])
def test_full_linear(cuda_device, G):
    p = api.LayerParams(G * 2, 2, 128, -1, 5e6, 64)
    _run(cuda_device, p, 5, 300, [1, 7, 64, 65, 300], seed=60 + G)
    check_no_device_error()


def test_split_k_paths(cuda_device):
    # long contexts with a small batch force several splits per sequence
    p = api.LayerParams(16, 2, 128, -1, 5e6, 64)
    lens = [1, 255, 256, 257, 4095, 9000, 20001]
    assert api.decode_workspace_size(p, len(lens), max(lens)) > 0
    _run(cuda_device, p, len(lens), 20480, lens, seed=70)
    pw = api.LayerParams(24, 2, 128, 2048, 5e5, 128)
    _run(cuda_device, pw, 3, 2048, [5, 2048, 100000], seed=71)
    check_no_device_error()


def test_large_scores(cuda_device):
    """q and keys times 3: a few keys dominate each row, and the split-K merge
    weighs partials whose maxima lie far apart."""
    _run(cuda_device, api.LayerParams(24, 2, 128, 64, 1e4, 128), 4, 64, [3, 64, 65, 700], seed=74, scale=3.0)
    _run(cuda_device, api.LayerParams(16, 2, 128, -1, 5e6, 64), 3, 12000, [9, 4097, 12000], seed=75, scale=3.0)
    check_no_device_error()


def test_unused_slots_may_hold_nan(cuda_device):
    p = api.LayerParams(8, 1, 128, 64, 1e4, 128)
    _run(cuda_device, p, 4, 64, [1, 5, 33, 63], seed=72, poison=True)
    pf = api.LayerParams(8, 1, 128, -1, 1e4, 128)
    _run(cuda_device, pf, 3, 500, [3, 129, 450], seed=73, poison=True, gate=False)
    check_no_device_error()


def test_rope_append_then_decode_matches_oracle(cuda_device):
    """The decode step as a user runs it: rotate q and the new k at position
    L-1, append k and v to the ring, then attend."""
    B, Hq, Hkv, W = 4, 24, 2, 32
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    lens = np.array([1, 20, 32, 77], np.int32)
    d = inputs.decode_inputs(B, Hq, Hkv, 128, W, seed=74)
    new = inputs.prefill_inputs(B, 1, Hq, Hkv, 128, seed=75)
    q = new["q"].to(cuda_device)
    k = new["k"].to(cuda_device)
    v = new["v"].to(cuda_device)
    kc, vc = d["k_cache"].to(cuda_device), d["v_cache"].to(cuda_device)
    pos = torch.from_numpy(lens - 1).reshape(B, 1).to(cuda_device)
    api.rope_qk(p, q=q, k=k, pos=pos, v=v, k_cache=kc, v_cache=vc)
    out = api.attn_decode(p, q[:, 0].contiguous(), d["gate"].to(cuda_device), kc, vc,
                          torch.from_numpy(lens).to(cuda_device), int(lens.max()))
    torch.cuda.synchronize()
    P = (lens - 1).astype(np.int64)
    q_rot = np.stack([oracle.rope(bits(new["q"][b]), P[b:b + 1], 1e4, 128)[0] for b in range(B)])
    k_rot = np.stack([oracle.rope(bits(new["k"][b]), P[b:b + 1], 1e4, 128)[0] for b in range(B)])
    v_new = oracle.bf16_bits_to_f64(bits(new["v"][:, 0]))
    ref = oracle.decode(oracle_layer(p), q_rot, d["gate"].numpy(), bits(d["k_cache"]), bits(d["v_cache"]), lens,
                        k_new=k_rot, v_new=v_new)
    assert_close(out, ref, "rope+append+decode")
    check_no_device_error()


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [configs.DECODE_SLIDING, configs.DECODE_FULL], ids=lambda c: c.name)
def test_full_size_decode_sampled(cuda_device, cfg):
    """The batched decode workload at full size (B=64, lengths U[4096,131072]);
    the oracle checks a seeded sample of (sequence, head) rows."""
    p = api.LayerParams(cfg.Hq, cfg.Hkv, 128, cfg.window, cfg.theta, cfg.rotary_dim)
    lens = inputs.uniform_int(cfg.B, cfg.len_lo, cfg.len_hi, cfg.seed)
    d = inputs.decode_inputs(cfg.B, cfg.Hq, cfg.Hkv, 128, cfg.capacity, cfg.seed, device=cuda_device)
    out = api.attn_decode(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens.to(cuda_device),
                          int(lens.max()))
    torch.cuda.synchronize()
    rng = np.random.default_rng(cfg.seed)
    bsel = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] + list(rng.choice(cfg.B, 2, replace=False))))
    G = cfg.Hq // cfg.Hkv
    rows = []
    for b in bsel:
        for h in range(0, cfg.Hq, max(1, G // 2)):
            rows.append((b, h))
    rows = np.array(rows, np.int64)
    # copy only the sampled sequences' visible slots back for the oracle
    sub_b = sorted(set(rows[:, 0].tolist()))
    remap = {b: i for i, b in enumerate(sub_b)}
    nmax = max(min(int(lens[b]), cfg.capacity) for b in sub_b)
    kc = d["k_cache"][sub_b, :, :nmax].cpu()
    vc = d["v_cache"][sub_b, :, :nmax].cpu()
    sub_lens = lens[sub_b].numpy().copy()
    C_sub = nmax if cfg.window < 0 else cfg.capacity
    if cfg.window > 0:
        kc = d["k_cache"][sub_b].cpu()
        vc = d["v_cache"][sub_b].cpu()
    q64 = oracle.bf16_bits_to_f64(bits(d["q"][sub_b]))
    lay = oracle_layer(p)
    sub_rows = np.array([(remap[b], h) for b, h in rows], np.int64)
    if cfg.window < 0:
        sub_lens = np.minimum(sub_lens, C_sub)
    ref = oracle.decode(lay, q64, d["gate"][sub_b].cpu().numpy(), bits(kc), bits(vc), sub_lens, rows=sub_rows)
    got = out.cpu()[torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1])]
    assert_close(got, ref, cfg.name)
    check_no_device_error()


@pytest.mark.slow
def test_large_batch(cuda_device):
    """B = 9000 sequences (72000 (sequence, kv-head) pairs: the batch sits on
    the grid's z axis), ring of 64; sampled sequences against the oracle."""
    B, Hq, Hkv, W = 9000, 16, 8, 64
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    lens = inputs.uniform_int(B, 1, 200, 4242)
    d = inputs.decode_inputs(B, Hq, Hkv, 128, W, 4242, device=cuda_device)
    out = api.attn_decode(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens.to(cuda_device), 200)
    torch.cuda.synchronize()
    bsel = [0, 1, 4095, 4096, 8191, 8192, 8999]
    sub = torch.tensor(bsel)
    ref = oracle.decode(oracle_layer(p), oracle.bf16_bits_to_f64(bits(d["q"][sub].cpu())), d["gate"][sub].cpu().numpy(),
                        bits(d["k_cache"][sub].cpu()), bits(d["v_cache"][sub].cpu()), lens[sub].numpy())
    assert_close(out[sub.to(cuda_device)], ref, "decode B9000")
    check_no_device_error()
