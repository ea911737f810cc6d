"""swa_attn_prefill_chunk on the GPU: a sequence prefilled in several chunks
against the KV cache gives the rows of the whole-sequence attention the
oracle computes, and leaves the cache exactly as appending every token with
swa_rope_qk would (ring: the last W positions; linear: all of them); the
bench's two continued-prefill workloads at full size on seeded rows."""
import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import api, configs, inputs
from gpu_helpers import (assert_close, bits, check_no_device_error, oracle_layer, prefill_rows_sample,
                         scaled_inv_freq)

pytestmark = pytest.mark.gpu


def _run_chunks(cuda_device, p, B, bounds, seed, C, gate=True, L_inputs=None):
    """Prefill positions bounds[0]..bounds[-1] chunk by chunk into a fresh
    cache; returns the inputs (CPU, L_inputs >= bounds[-1] tokens), the
    stacked outputs and the caches."""
    L = bounds[-1] if L_inputs is None else L_inputs
    d = inputs.prefill_inputs(B, L, p.num_q_heads, p.num_kv_heads, 128, seed, with_gate=gate)
    dev = {k: (None if t is None else t.to(cuda_device)) for k, t in d.items()}
    kc = torch.zeros(B, p.num_kv_heads, C, 128, dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    outs = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        sl = slice(a, b)
        g = None if dev["gate"] is None else dev["gate"][:, sl].contiguous()
        out = api.attn_prefill_chunk(p, a, dev["q"][:, sl].contiguous(), dev["k"][:, sl].contiguous(),
                                     dev["v"][:, sl].contiguous(), g, kc, vc)
        outs.append(out)
    torch.cuda.synchronize()
    return d, torch.cat(outs, dim=1), kc, vc


def _check(cuda_device, p, B, bounds, seed, C, gate=True):
    d, out, kc, vc = _run_chunks(cuda_device, p, B, bounds, seed, C, gate)
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]),
                         None if d["gate"] is None else d["gate"].numpy())
    assert_close(out, ref, f"chunks {bounds} W{p.window}")
    # the cache equals appending the whole sequence in one swa_rope_qk call
    L = bounds[-1]
    kref = torch.zeros_like(kc)
    vref = torch.zeros_like(vc)
    k_all = d["k"].to(cuda_device).contiguous()
    api.rope_qk(p, k=k_all, pos0=0, v=d["v"].to(cuda_device).contiguous(), k_cache=kref, v_cache=vref)
    torch.cuda.synchronize()
    slots = sorted({(pos % p.window) if p.window > 0 else pos for pos in range(max(0, L - (p.window if p.window > 0 else L)), L)})
    idx = torch.tensor(slots, device=cuda_device)
    assert torch.equal(kc[:, :, idx].view(torch.int16), kref[:, :, idx].view(torch.int16)), "k cache differs"
    assert torch.equal(vc[:, :, idx].view(torch.int16), vref[:, :, idx].view(torch.int16)), "v cache differs"
    check_no_device_error()


@pytest.mark.parametrize("bounds", [[0, 300], [0, 100, 137, 400], [0, 1, 2, 130, 131, 390], [0, 250, 640]],
                         ids=["one", "odd", "tiny-steps", "long-chunk"])
@pytest.mark.parametrize("W", [64, 100, 128, 200])
def test_sliding_chunks(cuda_device, bounds, W):
    """Ring cache: histories shorter than W - 1, chunks longer than W (only
    the last W positions stay in the ring), offsets off the 128 grid."""
    p = api.LayerParams(8, 2, 128, W, 1e4, 128)
    _check(cuda_device, p, 2, bounds, seed=900 + W, C=W)


@pytest.mark.parametrize("W,bounds", [(256, [0, 128, 640]), (512, [0, 384, 1000]), (384, [0, 256, 900])])
def test_sliding_chunks_tile_aligned_history(cuda_device, W, bounds):
    """A chunk whose history (the earlier tokens it attends to) is a multiple
    of 128 long puts its query tiles on key tile boundaries: for W a multiple
    of 128 the band's edges then fall exactly on key tile edges."""
    p = api.LayerParams(8, 2, 128, W, 1e4, 128)
    _check(cuda_device, p, 2, bounds, seed=950 + W, C=W)


@pytest.mark.parametrize("bounds", [[0, 300], [0, 100, 137, 400], [0, 1, 2, 130, 131, 390], [0, 256, 640]],
                         ids=["one", "odd", "tiny-steps", "aligned"])
@pytest.mark.parametrize("theta,r", [(5e6, 64), (0.0, 128)])
def test_full_chunks(cuda_device, bounds, theta, r):
    """Linear cache read in place: partial and no RoPE, offsets off the grid."""
    p = api.LayerParams(8, 2, 128, -1, theta, r)
    _check(cuda_device, p, 2, bounds, seed=950 + r, C=700)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (12, 1), (6, 2)])
def test_chunk_gqa_groups_no_gate(cuda_device, Hq, Hkv):
    _check(cuda_device, api.LayerParams(Hq, Hkv, 128, 96, 5e5, 32), 1, [0, 77, 300], seed=980 + Hq, C=96,
           gate=False)
    _check(cuda_device, api.LayerParams(Hq, Hkv, 128, -1, 1e4, 128), 1, [0, 200, 333], seed=990 + Hq, C=400,
           gate=False)


@pytest.mark.parametrize("W", [96, -1])
def test_chunks_frequency_table(cuda_device, W):
    table = scaled_inv_freq(5e6, 64)
    p = api.LayerParams(8, 2, 128, W, 5e6, 64, inv_freq=table)
    _check(cuda_device, p, 2, [0, 70, 333], seed=1010 + max(W, 0), C=96 if W > 0 else 400)


@pytest.mark.parametrize("p,C", [(api.LayerParams(8, 2, 128, 100, 1e4, 128), 100),
                                 (api.LayerParams(8, 2, 128, -1, 5e6, 64, inv_freq=scaled_inv_freq(5e6, 64)), 320)],
                         ids=["sliding", "full-table"])
def test_decode_after_chunked_prefill(cuda_device, p, C):
    """The cache a chunked prefill leaves feeds decode: the next token's
    output equals the whole-sequence prefill's next row."""
    B, L = 2, 301
    d, _, kc, vc = _run_chunks(cuda_device, p, B, [0, 120, 300], seed=1234, C=C, L_inputs=L)
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]), d["gate"].numpy(),
                         rows=np.array([(b, L - 1, h) for b in range(B) for h in range(8)], np.int64))
    q = d["q"][:, L - 1:L].to(cuda_device).contiguous()
    k = d["k"][:, L - 1:L].to(cuda_device).contiguous()
    v = d["v"][:, L - 1:L].to(cuda_device).contiguous()
    api.rope_qk(p, q=q, k=k, pos0=L - 1, v=v, k_cache=kc, v_cache=vc)
    lens = torch.full((B,), L, dtype=torch.int32, device=cuda_device)
    out = api.attn_decode(p, q[:, 0].contiguous(), d["gate"][:, L - 1].to(cuda_device).contiguous(), kc, vc, lens, L)
    torch.cuda.synchronize()
    assert_close(out.reshape(B * 8, 128), ref.reshape(B * 8, 128), "decode after chunks")
    check_no_device_error()


@pytest.mark.parametrize("cc", [configs.CHUNK_SLIDING, configs.CHUNK_FULL], ids=lambda c: c.name)
def test_bench_chunk_workloads_sampled(cuda_device, cc):
    """The continued-prefill workloads the bench times, at full size: the
    history (positions < pos0) is appended to a fresh cache the way a
    caller's earlier steps would (swa_rope_qk), the chunk then runs as in the
    bench, and seeded rows of it (first, last, band and tile edges, random,
    every head) match the oracle's whole-sequence prefill."""
    p = api.LayerParams(cc.Hq, cc.Hkv, 128, cc.window, cc.theta, cc.rotary_dim)
    L = cc.pos0 + cc.S
    d = inputs.prefill_inputs(cc.B, L, cc.Hq, cc.Hkv, 128, cc.seed)
    C = cc.window if cc.window > 0 else L
    kc = torch.zeros(cc.B, cc.Hkv, C, 128, dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    hist, new = slice(0, cc.pos0), slice(cc.pos0, L)
    api.rope_qk(p, k=d["k"][:, hist].to(cuda_device).contiguous(), pos0=0,
                v=d["v"][:, hist].to(cuda_device).contiguous(), k_cache=kc, v_cache=vc)
    dev = {k: t[:, new].to(cuda_device).contiguous() for k, t in d.items()}
    out = api.attn_prefill_chunk(p, cc.pos0, dev["q"], dev["k"], dev["v"], dev["gate"], kc, vc)
    torch.cuda.synchronize()
    rows = prefill_rows_sample(cc.B, cc.S, cc.Hq, cc.window, seed=cc.seed, n_random=48)
    rows[:, 1] += cc.pos0                     # positions of the chunk's rows in the whole sequence
    ref = oracle.prefill(oracle_layer(p), bits(d["q"]), bits(d["k"]), bits(d["v"]), d["gate"].numpy(), rows=rows)
    idx = [torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1] - cc.pos0), torch.from_numpy(rows[:, 2])]
    assert_close(out.cpu()[idx[0], idx[1], idx[2]], ref, cc.name)
    check_no_device_error()
