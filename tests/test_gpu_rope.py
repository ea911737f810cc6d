"""swa_rope_qk on the GPU against the oracle's RoPE, and the KV-cache append
(ring slot p mod W on sliding layers, slot p on full layers)."""
import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import api, inputs
from gpu_helpers import assert_close, bits, check_no_device_error, scaled_inv_freq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("theta,r", [(1e4, 128), (5e6, 64), (5e5, 32), (1e4, 6), (0.0, 128), (1e4, 0)])
def test_rope_in_place_matches_oracle(cuda_device, theta, r):
    B, S, Hq, Hkv = 2, 37, 12, 2
    p = api.LayerParams(Hq, Hkv, 128, 64, theta, r)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=41)
    q = d["q"].to(cuda_device)
    k = d["k"].to(cuda_device)
    pos = torch.randint(0, 131072, (B, S), generator=torch.Generator().manual_seed(3), dtype=torch.int32)
    api.rope_qk(p, q=q, k=k, pos=pos.to(cuda_device))
    torch.cuda.synchronize()
    for name, src, got, H in (("q", d["q"], q, Hq), ("k", d["k"], k, Hkv)):
        ref = oracle.rope(bits(src).reshape(B * S, H, 128), pos.numpy().reshape(-1).astype(np.int64), theta, r)
        if theta == 0 or r == 0:
            assert torch.equal(got.cpu(), src), name    # untouched, bit for bit
        assert_close(got.reshape(B * S, H, 128), ref, f"rope {name}")
    check_no_device_error()


@pytest.mark.parametrize("theta,r", [(5e6, 64), (1e4, 128), (0.0, 32)])
def test_rope_frequency_table_matches_oracle(cuda_device, theta, r):
    """A caller table replaces theta^(-2k/r); with theta 0 the table still
    rotates.  Positions up to 2^20 exercise the fp64 angle reduction."""
    B, S, Hq, Hkv = 2, 29, 8, 2
    table = scaled_inv_freq(theta if theta > 0 else 1e4, r)
    p = api.LayerParams(Hq, Hkv, 128, -1, theta, r, inv_freq=table)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=47)
    q = d["q"].to(cuda_device)
    k = d["k"].to(cuda_device)
    pos = torch.randint(0, 1 << 20, (B, S), generator=torch.Generator().manual_seed(5), dtype=torch.int32)
    api.rope_qk(p, q=q, k=k, pos=pos.to(cuda_device))
    torch.cuda.synchronize()
    P = pos.numpy().reshape(-1).astype(np.int64)
    for name, src, got, H in (("q", d["q"], q, Hq), ("k", d["k"], k, Hkv)):
        ref = oracle.rope_table(bits(src).reshape(B * S, H, 128), P, np.array(table), r)
        assert_close(got.reshape(B * S, H, 128), ref, f"rope table {name}")
        assert not torch.equal(got.cpu(), src), name
    check_no_device_error()


def test_rope_pos0_equals_explicit_positions(cuda_device):
    B, S, Hq, Hkv = 3, 20, 8, 8
    p = api.LayerParams(Hq, Hkv, 128, -1, 5e6, 64)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=42)
    q1, k1 = d["q"].to(cuda_device), d["k"].to(cuda_device)
    q2, k2 = q1.clone(), k1.clone()
    api.rope_qk(p, q=q1, k=k1, pos0=1000)
    pos = (1000 + torch.arange(S, dtype=torch.int32)).repeat(B, 1).to(cuda_device)
    api.rope_qk(p, q=q2, k=k2, pos=pos)
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(k1, k2)


@pytest.mark.parametrize("window,C", [(16, 16), (-1, 300)])
def test_cache_append_slots(cuda_device, window, C):
    B, S, Hq, Hkv = 3, 5, 4, 2
    p = api.LayerParams(Hq, Hkv, 128, window, 1e4, 128)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=43)
    k = d["k"].to(cuda_device)
    v = d["v"].to(cuda_device)
    kc = torch.zeros(B, Hkv, C, 128, dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    # distinct slots within each sequence (one call never writes a slot twice)
    pos = torch.tensor([[0, 1, 2, 3, 4], [15, 16, 17, 18, 19], [100, 150, 200, 250, 299]], dtype=torch.int32)
    if window > 0:
        pos[2] = torch.tensor([33, 45, 48, 59, 63])
    api.rope_qk(p, k=k, pos=pos.to(cuda_device), v=v, k_cache=kc, v_cache=vc)
    torch.cuda.synchronize()
    kc, vc, k = kc.cpu(), vc.cpu(), k.cpu()
    for b in range(B):
        for s in range(S):
            slot = int(pos[b, s]) % window if window > 0 else int(pos[b, s])
            assert torch.equal(kc[b, :, slot], k[b, s]), (b, s)           # rotated key, bit for bit
            assert torch.equal(vc[b, :, slot], d["v"][b, s]), (b, s)      # raw value, bit for bit
    written = torch.zeros(B, C, dtype=torch.bool)
    for b in range(B):
        for s in range(S):
            written[b, int(pos[b, s]) % window if window > 0 else int(pos[b, s])] = True
    assert torch.all(kc[~written.unsqueeze(1).expand(B, Hkv, C)] == 0)
    check_no_device_error()
