"""Host-side checks of the C ABI (no GPU needed): the library builds and
loads, exports every function include/swa.h declares, sizes workspaces and
KV caches, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from full_gqa_attention_swa_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "swa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SWA_API\s+[\w\s\*]+?\b(swa_\w+)\s*\(", text)))


def _P(**kw):
    base = dict(num_q_heads=8, num_kv_heads=2, head_dim=128, window=64, rope_theta=1e4, rotary_dim=128,
                softmax_scale=0.0)
    base.update(kw)
    return ctypes.byref(api._Params(**base))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert len(declared) == len(api.SYMBOLS) == 15
    assert sorted(api.SYMBOLS) == declared
    for name in declared:
        assert hasattr(lib, name), name
    assert "sm_100a" in api.version()


def test_status_strings(lib):
    for code, name in api.STATUS_NAMES.items():
        assert lib.swa_status_string(code).decode() == name


def test_kv_cache_bytes_matches_page_arithmetic(lib):
    # Muse explainer, GQA section: 128K context, 2 KV heads, 52 layers ~ 6.5 GiB
    full = api.LayerParams(32, 2, 128, api.WINDOW_FULL, 0.0, 128)
    assert 52 * api.kv_cache_bytes(full, 1, 131072) == 6.5 * 2 ** 30
    mha = api.LayerParams(32, 32, 128, api.WINDOW_FULL, 0.0, 128)
    assert 52 * api.kv_cache_bytes(mha, 1, 131072) == 104 * 2 ** 30
    # a sliding layer's ring keeps W slots however long the context
    sl = api.LayerParams(32, 2, 128, 2048, 5e5, 128)
    assert api.kv_cache_bytes(sl, 1, 131072) == 2048 * 2 * 128 * 2 * 2
    assert api.kv_cache_bytes(sl, 3, 100) == 3 * 100 * 2 * 128 * 2 * 2
    assert lib.swa_kv_cache_bytes(_P(head_dim=64), 1, 1) == -1


def test_workspace_sizes(lib):
    p = api.LayerParams(96, 8, 128, 512, 1e4, 128)
    ws = api.prefill_workspace_size(p, 1, 8192)
    k_bytes = 8192 * 8 * 128 * 2
    table = 8192 * 64 * 8
    assert ws == k_bytes + table
    # the table holds whole groups of 32 positions and whole couples of pairs:
    # S = 100 -> 4 groups, r = 6 -> 3 pairs -> 2 couples of 32 x 16 bytes
    odd = api.LayerParams(4, 2, 128, -1, 1e4, 6)
    k_odd = (1 * 100 * 2 * 128 * 2 + 255) // 256 * 256
    assert api.prefill_workspace_size(odd, 1, 100) == k_odd + 4 * 2 * 512
    assert api.prefill_workspace_size(api.LayerParams(32, 2, 128, -1, 0.0, 128), 4, 16384) == 0
    # sliding decode: one split, no workspace; full decode: split-K partials
    assert api.decode_workspace_size(p, 64, 131072) == 0
    full = api.LayerParams(64, 8, 128, -1, 5e6, 64)
    assert api.decode_workspace_size(full, 64, 131072) > 0


NULL = None
FAKE = 1 << 20          # aligned, never dereferenced: every case fails validation first
MIS = (1 << 20) + 8     # 8-byte aligned only


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_heads=8, num_kv_heads=3), 1),
    (dict(num_kv_heads=0), 1),
    (dict(head_dim=64), 2),
    (dict(window=0), 1),
    (dict(window=-2), 1),
    (dict(rotary_dim=3), 1),
    (dict(rotary_dim=130), 1),
    (dict(rope_theta=-1.0), 1),
    (dict(rope_theta=float("inf")), 1),
    (dict(softmax_scale=float("nan")), 1),
])
def test_bad_layer_params(lib, kw, status):
    st = lib.swa_attn_prefill(_P(**kw), 1, 128, FAKE, FAKE, FAKE, NULL, FAKE, FAKE, 1 << 30, NULL)
    assert st == status
    assert lib.swa_last_error_detail().decode() != ""


def test_prefill_argument_errors(lib):
    p = _P()
    assert lib.swa_attn_prefill(None, 1, 128, FAKE, FAKE, FAKE, NULL, FAKE, FAKE, 1 << 30, NULL) == 1
    assert lib.swa_attn_prefill(p, -1, 128, FAKE, FAKE, FAKE, NULL, FAKE, FAKE, 1 << 30, NULL) == 1
    assert lib.swa_attn_prefill(p, 1, 128, NULL, FAKE, FAKE, NULL, FAKE, FAKE, 1 << 30, NULL) == 1
    assert lib.swa_attn_prefill(p, 1, 128, FAKE, FAKE, FAKE, NULL, NULL, FAKE, 1 << 30, NULL) == 1
    assert lib.swa_attn_prefill(p, 1, 128, MIS, FAKE, FAKE, NULL, FAKE, FAKE, 1 << 30, NULL) == 1
    assert lib.swa_attn_prefill(p, 1, 128, FAKE, FAKE, FAKE, MIS, FAKE, FAKE, 1 << 30, NULL) == 1
    assert lib.swa_attn_prefill(p, 1, 128, FAKE, FAKE, FAKE, NULL, FAKE, NULL, 0, NULL) == 3
    assert lib.swa_attn_prefill(p, 1, 128, FAKE, FAKE, FAKE, NULL, FAKE, FAKE, 100, NULL) == 3
    assert lib.swa_attn_prefill(p, 1, 128, FAKE, FAKE, FAKE, NULL, FAKE, FAKE + 16, 1 << 30, NULL) == 3
    # empty inputs: nothing to do, nothing launched
    assert lib.swa_attn_prefill(p, 0, 128, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == 0
    assert lib.swa_attn_prefill(p, 2, 0, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == 0


def test_decode_argument_errors(lib):
    sl = _P(num_q_heads=96, num_kv_heads=8, window=512)
    full = _P(num_q_heads=64, num_kv_heads=8, window=-1, rope_theta=5e6, rotary_dim=64)
    args = lambda C, max_len: (FAKE, NULL, FAKE, FAKE, C, FAKE, max_len, FAKE, FAKE, 1 << 34, NULL)
    assert lib.swa_attn_decode(sl, 4, *args(256, 100)) == 1             # ring capacity != W
    assert lib.swa_attn_decode(full, 4, *args(1000, 2000)) == 1         # max_len > capacity
    assert lib.swa_attn_decode(full, 4, *args(1000, 0)) == 1            # max_len < 1
    assert lib.swa_attn_decode(_P(num_q_heads=34, num_kv_heads=2), 4, *args(64, 10)) == 2  # G > 16
    a = list(args(4096, 4096))
    a[0] = MIS
    assert lib.swa_attn_decode(full, 4, *a) == 1
    a = list(args(131072, 131072))
    a[8] = NULL                                                         # workspace missing
    assert lib.swa_attn_decode(full, 64, *a) == 3
    assert lib.swa_attn_decode(sl, 0, *args(512, 512)) == 0              # empty batch
    assert lib.swa_attn_decode(sl, 70000, *args(512, 512)) == 2          # B beyond the grid's z limit


def test_decode_no_alloc_argument_errors(lib):
    """The no-alloc decode's host checks, which all run before it touches the
    device (no GPU needed): the same rules as swa_attn_decode, with out
    required."""
    sl = _P(num_q_heads=96, num_kv_heads=8, window=512)
    full = _P(num_q_heads=64, num_kv_heads=8, window=-1, rope_theta=5e6, rotary_dim=64)
    # (q, gate, k_cache, v_cache, C, seq_lens, max_len, out, stream)
    args = lambda C, max_len: [FAKE, NULL, FAKE, FAKE, C, FAKE, max_len, FAKE, NULL]
    f = lib.swa_attn_decode_no_alloc
    assert f(sl, 4, *args(256, 100)) == 1                                # ring capacity != W
    assert f(full, 4, *args(1000, 2000)) == 1                            # max_len > capacity
    assert f(full, 4, *args(1000, 0)) == 1                               # max_len < 1
    assert f(full, 4, *args(0, 10)) == 1                                 # capacity < 1
    assert f(_P(num_q_heads=34, num_kv_heads=2), 4, *args(64, 10)) == 2  # G > 16
    assert f(sl, 70000, *args(512, 512)) == 2                            # B beyond the grid's z limit
    assert f(sl, -1, *args(512, 512)) == 1                               # negative batch
    assert f(sl, 0, *args(512, 512)) == 0                                # empty batch: nothing launched
    assert f(None, 4, *args(512, 512)) == 1                              # no parameters
    for i, name in ((0, "q"), (2, "k_cache"), (3, "v_cache"), (5, "seq_lens"), (7, "out")):
        a = args(512, 512)
        a[i] = NULL
        assert f(sl, 4, *a) == 1, name                                   # required pointer missing
        a[i] = MIS
        assert f(sl, 4, *a) == 1, name                                   # misaligned pointer
    a = args(512, 512)
    a[1] = MIS
    assert f(sl, 4, *a) == 1                                             # misaligned gate
    assert b"aligned" in lib.swa_last_error_detail()


def test_rope_argument_errors(lib):
    p = _P(window=16)
    assert lib.swa_rope_qk(p, 2, 4, FAKE, FAKE, NULL, 0, FAKE, FAKE, NULL, 16, NULL) == 1   # one cache only
    assert lib.swa_rope_qk(p, 2, 4, FAKE, NULL, NULL, 0, FAKE, FAKE, FAKE, 16, NULL) == 1   # cache needs k
    assert lib.swa_rope_qk(p, 2, 4, FAKE, FAKE, NULL, 0, FAKE, FAKE, FAKE, 8, NULL) == 1    # capacity != W
    assert lib.swa_rope_qk(p, 2, 4, FAKE, FAKE, NULL, -1, NULL, NULL, NULL, 0, NULL) == 1   # negative pos0
    assert lib.swa_rope_qk(p, 2, 4, MIS, FAKE, NULL, 0, NULL, NULL, NULL, 0, NULL) == 1
    assert lib.swa_rope_qk(p, 0, 4, FAKE, FAKE, NULL, 0, NULL, NULL, NULL, 0, NULL) == 0
    assert lib.swa_rope_qk(p, 2, 4, NULL, NULL, NULL, 0, NULL, NULL, NULL, 0, NULL) == 0


def test_prefill_chunk_argument_errors(lib):
    sl = _P(num_q_heads=8, num_kv_heads=2, window=512)
    full = _P(num_q_heads=8, num_kv_heads=2, window=-1, rope_theta=5e6, rotary_dim=64)
    # (B, S, pos0, q, k, v, gate, k_cache, v_cache, C, out, ws, ws_bytes, stream)
    args = lambda C, pos0: (1, 256, pos0, FAKE, FAKE, FAKE, NULL, FAKE, FAKE, C, FAKE, FAKE, 1 << 34, NULL)
    assert lib.swa_attn_prefill_chunk(sl, *args(256, 100)) == 1          # ring capacity != W
    assert lib.swa_attn_prefill_chunk(full, *args(300, 100)) == 1        # capacity < pos0 + S
    assert lib.swa_attn_prefill_chunk(full, 1, 256, -1, *args(4096, 0)[3:]) == 1   # negative pos0
    assert lib.swa_attn_prefill_chunk(full, 1, 256, 0x7FFFFF00, *args(4096, 0)[3:]) == 1  # positions past 2^31
    a = list(args(512, 100))
    a[7] = NULL                                                          # k_cache missing
    assert lib.swa_attn_prefill_chunk(sl, *a) == 1
    a = list(args(512, 100))
    a[8] = MIS                                                           # misaligned v_cache
    assert lib.swa_attn_prefill_chunk(sl, *a) == 1
    a = list(args(512, 100))
    a[11], a[12] = NULL, 0                                               # workspace missing
    assert lib.swa_attn_prefill_chunk(sl, *a) == 3
    # nothing to do: returns before touching anything
    assert lib.swa_attn_prefill_chunk(sl, 1, 0, 100, *([NULL] * 6), 512, NULL, NULL, 0, NULL) == 0


def test_prefill_chunk_workspace_sizes(lib):
    # sliding W 512, r 128: history min(pos0, 511) rows + the chunk, keys and
    # values [B, h + S, Hkv, D] bf16 each, plus the table of S positions
    sl = api.LayerParams(8, 2, 128, 512, 1e4, 128)
    row = 2 * 128 * 2
    up = lambda n: (n + 255) // 256 * 256
    table = lambda S, half: ((S + 31) // 32) * ((half + 1) // 2) * 512
    assert api.prefill_chunk_workspace_size(sl, 2, 300, 1000) == 2 * up(2 * (511 + 300) * row) + up(table(300, 64))
    assert api.prefill_chunk_workspace_size(sl, 2, 300, 10) == 2 * up(2 * (10 + 300) * row) + up(table(300, 64))
    # full layer: rotated chunk keys + table; without RoPE nothing at all
    full = api.LayerParams(8, 2, 128, -1, 5e6, 64)
    assert api.prefill_chunk_workspace_size(full, 2, 300, 5000) == up(2 * 300 * row) + up(table(300, 32))
    assert api.prefill_chunk_workspace_size(api.LayerParams(8, 2, 128, -1, 0.0, 128), 2, 300, 5000) == 0


def test_frequency_table(lib):
    """A caller table makes a theta-0 layer rotate (workspace for keys and
    the cos/sin table appears); a non-finite or negative entry is rejected
    before any launch; the binding checks the table's length."""
    table = tuple(0.5 ** k for k in range(32))
    with_table = api.LayerParams(8, 2, 128, -1, 0.0, 64, inv_freq=table)
    plain = api.LayerParams(8, 2, 128, -1, 0.0, 64)
    assert api.prefill_workspace_size(plain, 1, 100) == 0
    assert api.prefill_workspace_size(with_table, 1, 100) == (100 * 2 * 128 * 2 + 255) // 256 * 256 + 4 * 16 * 512
    # rotary_dim 0 never rotates, table or not
    assert api.prefill_workspace_size(api.LayerParams(8, 2, 128, -1, 0.0, 0, inv_freq=()), 1, 100) == 0
    for bad in (float("nan"), float("inf"), -1e-3):
        prm = api.LayerParams(8, 2, 128, -1, 1e4, 64, inv_freq=table[:31] + (bad,)).c()
        st = lib.swa_attn_prefill(ctypes.byref(prm), 1, 128, FAKE, FAKE, FAKE, NULL, FAKE, FAKE, 1 << 30, NULL)
        assert st == 1
        assert "inv_freq[31]" in lib.swa_last_error_detail().decode()
    with pytest.raises(ValueError):
        api.LayerParams(8, 2, 128, -1, 1e4, 64, inv_freq=table[:30]).c()


def test_decode_mq_argument_errors(lib):
    sl = _P(num_q_heads=96, num_kv_heads=8, window=512)
    full = _P(num_q_heads=64, num_kv_heads=8, window=-1, rope_theta=5e6, rotary_dim=64)
    # (B, T, q, gate, k_new, v_new, k_cache, v_cache, C, seq_lens, max_len, out, ws, ws_bytes, stream)
    args = lambda T, C, max_len: (4, T, FAKE, NULL, FAKE, FAKE, FAKE, FAKE, C, FAKE, max_len, FAKE, FAKE,
                                  1 << 34, NULL)
    assert lib.swa_attn_decode_mq(sl, *args(4, 256, 600)) == 1             # ring capacity != W
    assert lib.swa_attn_decode_mq(full, *args(4, 1000, 1005)) == 1         # max_len - T > capacity
    assert lib.swa_attn_decode_mq(full, *args(4, 1000, 3)) == 1            # max_len < T
    assert lib.swa_attn_decode_mq(full, *args(0, 1000, 10)) == 1           # T < 1
    assert lib.swa_attn_decode_mq(full, *args(9, 1000, 100)) == 2          # T * G = 72 > 64
    assert lib.swa_attn_decode_mq(sl, *args(17, 512, 100)) == 2            # T > 16
    assert lib.swa_attn_decode_mq(_P(num_q_heads=34, num_kv_heads=1), *args(2, 64, 10)) == 2   # 68 rows
    a = list(args(4, 1000, 1004))
    a[4] = MIS                                                             # misaligned k_new
    assert lib.swa_attn_decode_mq(full, *a) == 1
    a = list(args(4, 1000, 1004))
    a[5] = NULL                                                            # v_new missing
    assert lib.swa_attn_decode_mq(full, *a) == 1
    a = list(args(4, 131072, 131072))
    a[12], a[13] = NULL, 0                                                 # workspace missing
    assert lib.swa_attn_decode_mq(full, *a) == 3
    assert lib.swa_attn_decode_mq(sl, 0, 4, *([NULL] * 6), 512, NULL, 600, NULL, NULL, 0, NULL) == 0


def test_decode_mq_workspace_sizes(lib):
    # sliding B64 (one split: 512 (sequence, kv-head) pairs fill the SM slots)
    sl = api.LayerParams(96, 8, 128, 512, 1e4, 128)
    assert api.decode_mq_workspace_size(sl, 64, 4, 131072) == 0
    # full B64 T4: split-K partials for B * T * Hq rows
    full = api.LayerParams(64, 8, 128, -1, 5e6, 64)
    ws = api.decode_mq_workspace_size(full, 64, 4, 131072)
    rows = 64 * 4 * 64
    splits = ws // (rows * (128 * 4 + 8))
    assert splits >= 2 and ws == rows * splits * 128 * 4 + rows * splits * 8
    assert api.decode_mq_workspace_size(full, 64, 17, 131072) == 0    # unsupported T
    assert api.decode_mq_workspace_size(full, 64, 4, 3) == 0           # max_len < T


def test_binding_requires_one_device():
    """The binding refuses tensors spread over several GPUs (a pointer into
    another GPU's memory must never reach a kernel) and a stream of another
    device; no GPU is needed to check the rule."""
    from types import SimpleNamespace as NS

    import torch

    d0, d1 = torch.device("cuda", 0), torch.device("cuda", 1)
    assert api._device(NS(device=d0), None, NS(device=d0)) == d0
    with pytest.raises(ValueError):
        api._device(NS(device=d0), NS(device=d1))
    with pytest.raises(ValueError):
        api._device(NS(device=d1), stream=NS(device=d0))
