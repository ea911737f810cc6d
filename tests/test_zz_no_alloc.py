"""swa_attn_decode_no_alloc against the oracle and against swa_attn_decode.

The no-alloc entry point serves callers that cannot allocate device memory
when they call (an engine that hands its plugins no allocator, a host
callback, a serving loop that must not stall on an allocation): its split-K
partials live in a static device array inside libswa.so instead of a caller
workspace.  These tests call it through the C ABI twice in a row, with
different data, and check each result against the fp64 oracle on sampled
(sequence, q-head) rows and against the workspace entry point's output on
every element, within the parity tolerance of the other GPU tests
(1e-2 + 1e-2 * |reference|).  This file is collected last so that a failure
here leaves every other test already run.
"""
import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import api, inputs
from gpu_helpers import ATOL, RTOL, assert_close, bits, check_no_device_error, oracle_layer

pytestmark = pytest.mark.gpu


def _case(dev, p, B, C, lens, seed):
    d = inputs.decode_inputs(B, p.num_q_heads, p.num_kv_heads, 128, C, seed, device=dev)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=dev)
    return d, lens_t


def _compare(a, b):
    a = a.float().cpu().numpy()
    b = b.float().cpu().numpy()
    assert np.all(np.isfinite(a))
    assert np.all(np.abs(a - b) <= ATOL + RTOL * np.abs(b)), float(np.abs(a - b).max())


def _oracle_rows(p, d, lens, out, seed, n_seq=4):
    """The oracle on every q-head of a seeded sample of sequences (always the
    longest and the shortest); only those sequences' visible slots are copied
    back to the host."""
    lens = np.asarray(lens, np.int64)
    B = len(lens)
    rng = np.random.default_rng(seed)
    sub = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] +
                     rng.choice(B, min(n_seq, B), replace=False).tolist()))
    C = d["k_cache"].shape[2]
    n = C if p.window > 0 else max(int(lens[b]) for b in sub)
    kc = d["k_cache"][sub, :, :n].cpu()
    vc = d["v_cache"][sub, :, :n].cpu()
    rows = np.array([(i, h) for i in range(len(sub)) for h in range(p.num_q_heads)], np.int64)
    ref = oracle.decode(oracle_layer(p), oracle.bf16_bits_to_f64(bits(d["q"][sub])), d["gate"][sub].cpu().numpy(),
                        bits(kc), bits(vc), lens[sub].astype(np.int32), rows=rows)
    got = out[sub].cpu()[torch.from_numpy(rows[:, 0]), torch.from_numpy(rows[:, 1])]
    assert_close(got, ref, "no-alloc decode rows vs oracle")


@pytest.mark.parametrize("shrink", [False, True])
def test_no_alloc_decode_matches_oracle_and_workspace_decode_twice(cuda_device, shrink):
    if shrink:
        # the usual split-K partials (B*Hq rows x many splits) exceed the
        # static array, so the call must use fewer, longer splits
        p = api.LayerParams(128, 8, 128, -1, 5e6, 64)
        B, C = 64, 16384
        lens = inputs.uniform_int(B, 1024, C, seed=81).tolist()
        assert api.decode_workspace_size(p, B, max(lens)) > api.NO_ALLOC_SCRATCH_BYTES
    else:
        p = api.LayerParams(16, 2, 128, -1, 5e6, 64)
        B, C = 5, 20480
        lens = [1, 300, 4097, 9000, 20480]
        assert 0 < api.decode_workspace_size(p, B, max(lens)) <= api.NO_ALLOC_SCRATCH_BYTES
    for call, seed in enumerate((82, 83)):        # two calls in a row, different data
        d, lens_t = _case(cuda_device, p, B, C, lens, seed + 10 * shrink)
        ref = api.attn_decode(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens_t, max(lens))
        out = torch.full_like(ref, float("nan"))
        api.attn_decode_no_alloc(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens_t, max(lens), out)
        torch.cuda.synchronize()
        _oracle_rows(p, d, lens, out, seed)
        _compare(out, ref)
    check_no_device_error()


def test_no_alloc_single_split_sliding(cuda_device):
    p = api.LayerParams(96, 8, 128, 512, 1e4, 128)
    B, lens = 8, [3, 511, 512, 513, 4096, 70000, 100, 131072]
    for seed in (84, 85):
        d, lens_t = _case(cuda_device, p, B, 512, lens, seed)
        ref = api.attn_decode(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens_t, max(lens))
        out = torch.empty_like(ref)
        api.attn_decode_no_alloc(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens_t, max(lens), out)
        torch.cuda.synchronize()
        _oracle_rows(p, d, lens, out, seed, n_seq=8)
        _compare(out, ref)
    check_no_device_error()


def test_no_alloc_one_split_when_two_do_not_fit(cuda_device):
    # 16 q-heads x 1024 sequences = 16384 rows: two splits need 17 MB > 16 MiB,
    # so every row runs as one split, which needs no scratch at all
    p = api.LayerParams(16, 1, 128, -1, 5e6, 64)
    B, C = 1024, 8192
    lens = inputs.uniform_int(B, 1, C, seed=86).tolist()
    lens[0] = C
    assert B * 16 * 2 * 520 + 512 > api.NO_ALLOC_SCRATCH_BYTES
    for seed in (87, 88):
        d, lens_t = _case(cuda_device, p, B, C, lens, seed)
        ref = api.attn_decode(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens_t, max(lens))
        out = torch.full_like(ref, float("nan"))
        api.attn_decode_no_alloc(p, d["q"], d["gate"], d["k_cache"], d["v_cache"], lens_t, max(lens), out)
        torch.cuda.synchronize()
        _oracle_rows(p, d, lens, out, seed)
        _compare(out, ref)
        del d
    check_no_device_error()
