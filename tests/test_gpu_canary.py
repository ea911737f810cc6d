"""Out-of-bounds and stray-write checks on the GPU without a sanitizer: every
buffer a call writes (outputs, workspaces, KV caches) sits between guard bands
of a known byte pattern that must survive the call; read-only inputs must be
bit-identical afterwards; cache slots a call must not write keep their bytes.
Shapes are odd on purpose (ragged tiles, partial rings, split-K)."""
import pytest
import torch

from full_gqa_attention_swa_b200 import api, inputs
from gpu_helpers import check_no_device_error

pytestmark = pytest.mark.gpu

GUARD = 65536   # bytes on each side; a multiple of 256 keeps every view aligned
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape` / `dtype` in the middle of a byte buffer whose
    guard bands hold PATTERN."""

    def __init__(self, shape, dtype, device, fill=None):
        n = torch.empty(shape, dtype=dtype).numel() * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.buf = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device=device)
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def check(self, what):
        assert bool((self.buf[:GUARD] == PATTERN).all()), f"{what}: write before the buffer"
        assert bool((self.buf[GUARD + self.n:] == PATTERN).all()), f"{what}: write past the buffer"


def _ws(nbytes, device):
    return Guarded((max(nbytes, 16),), torch.uint8, device) if nbytes > 0 else None


def _same(a, b, what):
    assert torch.equal(a.view(torch.uint8) if a.dtype != torch.uint8 else a,
                       b.view(torch.uint8) if b.dtype != torch.uint8 else b), f"{what} changed"


@pytest.mark.parametrize("W", [64, -1])
def test_prefill(cuda_device, W):
    B, S, Hq, Hkv = 2, 333, 6, 2
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    d = {k: t.to(cuda_device) for k, t in inputs.prefill_inputs(B, S, Hq, Hkv, 128, 6000).items()}
    before = {k: t.clone() for k, t in d.items()}
    out = Guarded((B, S, Hq, 128), torch.bfloat16, cuda_device)
    ws = _ws(api.prefill_workspace_size(p, B, S), cuda_device)
    api.attn_prefill(p, d["q"], d["k"], d["v"], d["gate"], out=out.t, workspace=None if ws is None else ws.t)
    torch.cuda.synchronize()
    out.check("prefill out")
    if ws is not None:
        ws.check("prefill workspace")
    for k in d:
        _same(d[k], before[k], f"prefill input {k}")
    check_no_device_error()


@pytest.mark.parametrize("W,C", [(64, 64), (-1, 600)])
def test_prefill_chunk(cuda_device, W, C):
    B, S, pos0, Hq, Hkv = 2, 150, 201, 8, 2
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    d = {k: t.to(cuda_device) for k, t in inputs.prefill_inputs(B, S, Hq, Hkv, 128, 6100).items()}
    before = {k: t.clone() for k, t in d.items()}
    cache = inputs.decode_inputs(B, Hq, Hkv, 128, C, 6101, device=cuda_device)
    kc = Guarded((B, Hkv, C, 128), torch.bfloat16, cuda_device, cache["k_cache"])
    vc = Guarded((B, Hkv, C, 128), torch.bfloat16, cuda_device, cache["v_cache"])
    out = Guarded((B, S, Hq, 128), torch.bfloat16, cuda_device)
    ws = _ws(api.prefill_chunk_workspace_size(p, B, S, pos0), cuda_device)
    api.attn_prefill_chunk(p, pos0, d["q"], d["k"], d["v"], d["gate"], kc.t, vc.t, out=out.t,
                           workspace=None if ws is None else ws.t)
    torch.cuda.synchronize()
    for g, what in ((out, "chunk out"), (kc, "k cache"), (vc, "v cache")):
        g.check(what)
    if ws is not None:
        ws.check("chunk workspace")
    for k in d:
        _same(d[k], before[k], f"chunk input {k}")
    # slots of positions outside pos0 .. pos0 + S - 1 (ring: outside its last W) keep their bytes
    written = set((pos % W) if W > 0 else pos for pos in range(max(pos0, pos0 + S - (W if W > 0 else S)), pos0 + S))
    keep = torch.tensor([s for s in range(C) if s not in written], device=cuda_device)
    if keep.numel():
        _same(kc.t[:, :, keep], cache["k_cache"][:, :, keep], "k cache slots not written by the chunk")
        _same(vc.t[:, :, keep], cache["v_cache"][:, :, keep], "v cache slots not written by the chunk")
    check_no_device_error()


@pytest.mark.parametrize("W,C,max_len", [(64, 64, 300), (-1, 3000, 3000)])
def test_decode_and_multi_query(cuda_device, W, C, max_len):
    """One-query decode (split-K on the long linear cache) and multi-query
    decode write only their outputs / workspaces; caches and inputs stay."""
    B, Hq, Hkv, T = 3, 24, 2, 4
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    cache = inputs.decode_inputs(B, Hq, Hkv, 128, C, 6200, device=cuda_device)
    kc0, vc0 = cache["k_cache"].clone(), cache["v_cache"].clone()
    lens = torch.tensor([T, max_len // 2, max_len], dtype=torch.int32, device=cuda_device)
    q0, g0 = cache["q"].clone(), cache["gate"].clone()
    out = Guarded((B, Hq, 128), torch.bfloat16, cuda_device)
    ws = _ws(api.decode_workspace_size(p, B, max_len), cuda_device)
    api.attn_decode(p, cache["q"], cache["gate"], cache["k_cache"], cache["v_cache"], lens, max_len, out=out.t,
                    workspace=None if ws is None else ws.t)
    new = {k: t.to(cuda_device) for k, t in inputs.prefill_inputs(B, T, Hq, Hkv, 128, 6201).items()}
    new0 = {k: t.clone() for k, t in new.items()}
    out_mq = Guarded((B, T, Hq, 128), torch.bfloat16, cuda_device)
    ws_mq = _ws(api.decode_mq_workspace_size(p, B, T, max_len), cuda_device)
    api.attn_decode_mq(p, new["q"], new["gate"], new["k"], new["v"], cache["k_cache"], cache["v_cache"], lens, max_len,
                       out=out_mq.t, workspace=None if ws_mq is None else ws_mq.t)
    torch.cuda.synchronize()
    out.check("decode out")
    out_mq.check("multi-query out")
    for w, what in ((ws, "decode workspace"), (ws_mq, "multi-query workspace")):
        if w is not None:
            w.check(what)
    _same(cache["k_cache"], kc0, "k cache")
    _same(cache["v_cache"], vc0, "v cache")
    _same(cache["q"], q0, "decode q")
    _same(cache["gate"], g0, "decode gate")
    for k in new:
        _same(new[k], new0[k], f"multi-query input {k}")
    check_no_device_error()


def test_rope_append(cuda_device):
    """swa_rope_qk rotates q / k inside their buffers and writes exactly the
    slots of the given positions."""
    B, S, Hq, Hkv, W = 3, 5, 12, 2, 16
    p = api.LayerParams(Hq, Hkv, 128, W, 1e4, 128)
    d = inputs.prefill_inputs(B, S, Hq, Hkv, 128, 6300)
    q = Guarded((B, S, Hq, 128), torch.bfloat16, cuda_device, d["q"].to(cuda_device))
    k = Guarded((B, S, Hkv, 128), torch.bfloat16, cuda_device, d["k"].to(cuda_device))
    cache = inputs.decode_inputs(B, Hq, Hkv, 128, W, 6301, device=cuda_device)
    kc = Guarded((B, Hkv, W, 128), torch.bfloat16, cuda_device, cache["k_cache"])
    vc = Guarded((B, Hkv, W, 128), torch.bfloat16, cuda_device, cache["v_cache"])
    pos = torch.tensor([[0, 1, 2, 3, 4], [20, 21, 22, 23, 24], [7, 9, 11, 13, 15]], dtype=torch.int32)
    api.rope_qk(p, q=q.t, k=k.t, pos=pos.to(cuda_device), v=d["v"].to(cuda_device), k_cache=kc.t, v_cache=vc.t)
    torch.cuda.synchronize()
    for g, what in ((q, "q"), (k, "k"), (kc, "k cache"), (vc, "v cache")):
        g.check(what)
    for b in range(B):
        keep = torch.tensor([s for s in range(W) if s not in set(int(x) % W for x in pos[b])], device=cuda_device)
        _same(kc.t[b, :, keep], cache["k_cache"][b, :, keep], f"k cache slots of sequence {b} not written")
        _same(vc.t[b, :, keep], cache["v_cache"][b, :, keep], f"v cache slots of sequence {b} not written")
    check_no_device_error()
