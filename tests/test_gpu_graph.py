"""The entry points inside CUDA graphs: nothing in a call synchronises the host
or allocates, so a decode step (RoPE + cache append + attention), a
multi-query decode and a prefill can be captured once and replayed with new
inputs copied into the captured buffers.  Replays must equal eager calls on
the same inputs bit for bit (same kernels, same order), and one replay is
checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import api, inputs
from gpu_helpers import assert_close, bits, check_no_device_error, oracle_layer

pytestmark = pytest.mark.gpu


def _graph(fn, warmup=True):
    if warmup:        # first calls set kernel attributes; keep them out of the capture
        fn()
        torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_step_graph(cuda_device):
    """One decode step per replay: rotate q and the new k at their positions,
    append k / v to the ring, attend; the lengths advance on the device."""
    B, Hq, Hkv, W = 4, 24, 2, 64
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    cache = inputs.decode_inputs(B, Hq, Hkv, 128, W, seed=3100, device=cuda_device)
    kc, vc = cache["k_cache"], cache["v_cache"]
    kc_e, vc_e = kc.clone(), vc.clone()                      # eager twin
    lens0 = torch.tensor([1, 30, 64, 200], dtype=torch.int32, device=cuda_device)
    lens = lens0.clone()
    q = torch.empty(B, 1, Hq, 128, dtype=torch.bfloat16, device=cuda_device)
    k = torch.empty(B, 1, Hkv, 128, dtype=torch.bfloat16, device=cuda_device)
    v = torch.empty_like(k)
    gate = torch.empty(B, Hq, device=cuda_device)
    out = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device=cuda_device)
    max_len = 400
    ws = torch.empty(max(api.decode_workspace_size(p, B, max_len), 1), dtype=torch.uint8, device=cuda_device)

    def step(q, k, v, gate, kc, vc, lens, out):
        api.rope_qk(p, q=q, k=k, pos=(lens - 1).view(B, 1), v=v, k_cache=kc, v_cache=vc)
        api.attn_decode(p, q.view(B, Hq, 128), gate, kc, vc, lens, max_len, out=out, workspace=ws)

    # warm-up on throw-away buffers, then capture
    step(q.zero_(), k.zero_(), v.zero_(), gate.zero_(), kc.clone(), vc.clone(), lens0.clone(), out)
    torch.cuda.synchronize()
    g = _graph(lambda: step(q, k, v, gate, kc, vc, lens, out), warmup=False)
    lens_e = lens0.clone()
    for t in range(3):
        new = inputs.prefill_inputs(B, 1, Hq, Hkv, 128, seed=3110 + t, device=cuda_device)
        q_e, k_e = new["q"].clone(), new["k"].clone()
        q.copy_(new["q"]); k.copy_(new["k"]); v.copy_(new["v"]); gate.copy_(new["gate"][:, 0])
        g.replay()
        out_e = torch.empty_like(out)
        step(q_e, k_e, new["v"], new["gate"][:, 0].contiguous(), kc_e, vc_e, lens_e, out_e)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), out_e.view(torch.int16)), f"replay {t} differs from eager"
        assert torch.equal(kc.view(torch.int16), kc_e.view(torch.int16))
        lens += 1
        lens_e += 1
    check_no_device_error()


def test_multi_query_decode_graph(cuda_device):
    B, T, Hq, Hkv, W = 3, 4, 24, 2, 64
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    cache = inputs.decode_inputs(B, Hq, Hkv, 128, W, seed=3200, device=cuda_device)
    lens = torch.tensor([4, 50, 300], dtype=torch.int32, device=cuda_device)
    st = {n: torch.empty(s, dtype=dt, device=cuda_device) for n, s, dt in
          (("q", (B, T, Hq, 128), torch.bfloat16), ("k", (B, T, Hkv, 128), torch.bfloat16),
           ("v", (B, T, Hkv, 128), torch.bfloat16), ("gate", (B, T, Hq), torch.float32))}
    out = torch.empty(B, T, Hq, 128, dtype=torch.bfloat16, device=cuda_device)

    def call(d, o):
        api.attn_decode_mq(p, d["q"], d["gate"], d["k"], d["v"], cache["k_cache"], cache["v_cache"], lens, 300,
                           out=o)

    for t in st.values():
        t.zero_()
    g = _graph(lambda: call(st, out))
    for r in range(2):
        new = inputs.prefill_inputs(B, T, Hq, Hkv, 128, seed=3210 + r, device=cuda_device)
        for n in st:
            st[n].copy_(new[n])
        g.replay()
        out_e = torch.empty_like(out)
        call(new, out_e)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), out_e.view(torch.int16)), f"replay {r} differs from eager"
    ref = oracle.decode_mq(oracle_layer(p), oracle.bf16_bits_to_f64(bits(new["q"].cpu())), new["gate"].cpu().numpy(),
                           bits(cache["k_cache"].cpu()), bits(cache["v_cache"].cpu()), lens.cpu().numpy(),
                           bits(new["k"].cpu()), bits(new["v"].cpu()))
    assert_close(out, ref, "multi-query decode replay")
    check_no_device_error()


def test_prefill_graph(cuda_device):
    B, S, Hq, Hkv, W = 1, 700, 8, 2, 200
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    st = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=3300, device=cuda_device)
    out = torch.empty_like(st["q"])
    ws = torch.empty(api.prefill_workspace_size(p, B, S), dtype=torch.uint8, device=cuda_device)

    def call(d, o):
        api.attn_prefill(p, d["q"], d["k"], d["v"], d["gate"], out=o, workspace=ws)

    g = _graph(lambda: call(st, out))
    for r in range(2):
        new = inputs.prefill_inputs(B, S, Hq, Hkv, 128, seed=3310 + r, device=cuda_device)
        for n in st:
            st[n].copy_(new[n])
        g.replay()
        out_e = torch.empty_like(out)
        call(new, out_e)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), out_e.view(torch.int16)), f"replay {r} differs from eager"
    rows = np.array([(0, i, h) for i in (0, 1, 199, 200, 201, 511, 512, 699) for h in (0, 5)], np.int64)
    ref = oracle.prefill(oracle_layer(p), bits(new["q"].cpu()), bits(new["k"].cpu()), bits(new["v"].cpu()),
                         new["gate"].cpu().numpy(), rows=rows)
    got = out.cpu()[torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1]), torch.from_numpy(rows[:, 2])]
    assert_close(got, ref, "prefill replay")
    check_no_device_error()
