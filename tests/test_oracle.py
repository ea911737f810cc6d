"""Pins for the fp64 oracle: each test ties it to something other than itself.

Checks (page title, section they follow):
* torch's own scaled-dot-product attention (fp64, CPU) with the band built
  from torch.tril/triu and RoPE written as complex multiplication -- the
  whole prefill definition, "Step-3.7-Flash-oQ3e" explainer secs. 2.2-2.3.
* closed forms: rotation angle of a unit vector at known frequencies
  (theta^0 = 1, 10000^-0.5 = 0.01), the window-1 and zero-query special
  cases, gate logits 0 and +40, the KV-cache footprint the Muse explainer
  prints (GQA section).
* invariants: streaming == materialised matrix, softmax rows sum to one and
  vanish off the band, W >= S == full, RoPE composition / norm / relativity,
  GQA == MHA with repeated KV heads, decode == last prefill row, ring order
  irrelevant.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from full_gqa_attention_swa_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(t):
    return inputs.as_bits(t)


def _f64(t):
    return t.to(torch.float64)


def _rope_complex(x, pos, theta, r, freq=None):
    """RoPE as multiplication of z_k = x_k + i x_{k+r/2} by exp(i p w_k),
    w_k = theta^(-2k/r) or freq[k]."""
    if (theta == 0 and freq is None) or r == 0:
        return x.clone()
    half = r // 2
    k = torch.arange(half, dtype=torch.float64)
    w = (torch.tensor(float(theta), dtype=torch.float64) ** (-2.0 * k / r) if freq is None
         else torch.tensor(np.asarray(freq, np.float64)))
    ang = pos.to(torch.float64)[:, None] * w[None, :]                      # [S, half]
    rot = torch.polar(torch.ones_like(ang), ang)                             # e^{i ang}
    z = torch.complex(x[..., :half], x[..., half:r])                        # [..., S, H, half]
    z = z * rot[:, None, :]
    y = x.clone()
    y[..., :half] = z.real
    y[..., half:r] = z.imag
    return y


def _sdpa_reference(q, k, v, gate, window, theta, r, freq=None):
    """Library attention on the same inputs: torch SDPA in fp64 with an
    explicit boolean band mask from tril/triu; KV heads repeated per group."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    pos = torch.arange(S)
    qr = _rope_complex(_f64(q), pos, theta, r, freq)
    kr = _rope_complex(_f64(k), pos, theta, r, freq)
    G = Hq // Hkv
    kr = kr.repeat_interleave(G, dim=2)
    vv = _f64(v).repeat_interleave(G, dim=2)
    ones = torch.ones(S, S, dtype=torch.bool)
    mask = ones.tril() if window < 0 else ones.tril() & ones.triu(-(window - 1))
    o = torch.nn.functional.scaled_dot_product_attention(
        qr.transpose(1, 2), kr.transpose(1, 2), vv.transpose(1, 2), attn_mask=mask,
        scale=1.0 / math.sqrt(D))
    o = o.transpose(1, 2)
    if gate is not None:
        o = o * torch.sigmoid(_f64(gate))[..., None]
    return o.numpy()


CASES = [
    # B, S, Hq, Hkv, D, W, theta, r
    (1, 33, 4, 2, 16, 5, 1e4, 16),
    (2, 40, 6, 3, 32, 1, 1e4, 32),
    (1, 29, 4, 1, 16, -1, 5e6, 8),
    (1, 48, 8, 2, 16, 16, 0.0, 16),
    (2, 17, 2, 2, 8, 100, 5e5, 0),
    (1, 64, 4, 4, 128, 32, 1e4, 64),
]


@pytest.mark.parametrize("B,S,Hq,Hkv,D,W,theta,r", CASES)
def test_prefill_matches_torch_sdpa(B, S, Hq, Hkv, D, W, theta, r):
    d = inputs.prefill_inputs(B, S, Hq, Hkv, D, seed=11 + S)
    lay = oracle.Layer(Hq, Hkv, D, W, theta, r)
    got = oracle.prefill(lay, _bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    ref = _sdpa_reference(d["q"], d["k"], d["v"], d["gate"], W, theta, r)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("B,S,Hq,Hkv,D,W,theta,r", CASES)
def test_streaming_equals_materialised(B, S, Hq, Hkv, D, W, theta, r):
    d = inputs.prefill_inputs(B, S, Hq, Hkv, D, seed=23 + S)
    lay = oracle.Layer(Hq, Hkv, D, W, theta, r)
    args = (_bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    a = oracle.prefill(lay, *args)
    b, w = oracle.prefill_materialised(lay, *args, want_weights=True)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    # softmax rows: sum to one, zero exactly off the band, support = window
    np.testing.assert_allclose(w.sum(-1), 1.0, rtol=0, atol=1e-14)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    band = (j <= i) if W < 0 else ((j <= i) & (j > i - W))
    assert np.all(w[..., ~band] == 0.0)
    assert np.all(w[..., band] > 0.0)
    expect = np.minimum(np.arange(S) + 1, S if W < 0 else W)
    assert np.array_equal((w > 0).sum(-1)[0, 0], expect)


def test_rows_subset_matches_all_rows():
    d = inputs.prefill_inputs(2, 50, 4, 2, 16, seed=5)
    lay = oracle.Layer(4, 2, 16, 7, 1e4, 16)
    args = (_bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    full = oracle.prefill(lay, *args)
    rows = np.array([[0, 0, 0], [1, 49, 3], [0, 6, 1], [1, 7, 2], [0, 25, 3]], np.int64)
    sub = oracle.prefill(lay, *args, rows=rows)
    for t, (b, i, h) in enumerate(rows):
        assert np.array_equal(sub[t], full[b, i, h])


def test_window_at_least_S_is_full_causal_bitwise():
    d = inputs.prefill_inputs(1, 45, 4, 2, 32, seed=3)
    args = (_bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    full = oracle.prefill(oracle.Layer(4, 2, 32, -1, 1e4, 32), *args)
    for W in (45, 46, 1000):
        got = oracle.prefill(oracle.Layer(4, 2, 32, W, 1e4, 32), *args)
        assert np.array_equal(got, full)


def test_window_one_returns_gated_value():
    d = inputs.prefill_inputs(2, 30, 6, 2, 16, seed=9)
    lay = oracle.Layer(6, 2, 16, 1, 1e4, 16)
    got = oracle.prefill(lay, _bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    v = oracle.bf16_bits_to_f64(_bits(d["v"]))                     # [B,S,Hkv,D]
    g = 1.0 / (1.0 + np.exp(-d["gate"].numpy().astype(np.float64)))  # [B,S,Hq]
    expect = g[..., None] * np.repeat(v, 3, axis=2)
    np.testing.assert_allclose(got, expect, rtol=1e-15, atol=0)


def test_gate_limits():
    d = inputs.prefill_inputs(1, 20, 4, 2, 16, seed=4)
    lay = oracle.Layer(4, 2, 16, 6, 1e4, 16)
    args = (_bits(d["q"]), _bits(d["k"]), _bits(d["v"]))
    ungated = oracle.prefill(lay, *args, None)
    big = oracle.prefill(lay, *args, np.full((1, 20, 4), 40.0, np.float32))
    zero = oracle.prefill(lay, *args, np.zeros((1, 20, 4), np.float32))
    assert np.array_equal(big, ungated)          # sigmoid(40) rounds to 1 in fp64
    assert np.array_equal(zero, 0.5 * ungated)   # sigmoid(0) = 1/2 exactly


@pytest.mark.parametrize("W", [1, 3, 64, 127, 128, 129, -1])
def test_uniform_score_probe_counts(W):
    """Q = 0 makes every score 0, so each output is the gate times the mean of
    the visible values; with one-hot values e_(j mod D) every output dim is a
    count of visible keys -- an exact window-size check."""
    B, S, Hq, Hkv, D = 1, 300, 2, 1, 128
    q = torch.zeros(B, S, Hq, D, dtype=torch.bfloat16)
    k = inputs.normal_bf16((B, S, Hkv, D), 1, "k")
    v = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16)
    v[0, torch.arange(S), 0, torch.arange(S) % D] = 1.0
    gate = torch.zeros(B, S, Hq)                                    # sigmoid = 1/2
    lay = oracle.Layer(Hq, Hkv, D, W, 1e4, 128)
    got = oracle.prefill(lay, _bits(q), _bits(k), _bits(v), gate.numpy())
    for i in (0, 1, 2, 63, 64, 65, 127, 128, 129, 200, 299):
        lo = 0 if W < 0 else max(0, i - W + 1)
        n = i - lo + 1
        counts = np.zeros(D)
        for j in range(lo, i + 1):
            counts[j % D] += 1
        np.testing.assert_allclose(got[0, i, 0], 0.5 * counts / n, rtol=1e-15, atol=1e-16)
        assert oracle.visible_count(i, W) == n


def test_gqa_contiguous_groups_equal_repeated_mha():
    B, S, Hq, Hkv, D = 1, 24, 8, 2, 16
    d = inputs.prefill_inputs(B, S, Hq, Hkv, D, seed=8)
    gqa = oracle.prefill(oracle.Layer(Hq, Hkv, D, 9, 1e4, 16), _bits(d["q"]), _bits(d["k"]),
                         _bits(d["v"]), d["gate"].numpy())
    krep = d["k"].repeat_interleave(Hq // Hkv, dim=2)
    vrep = d["v"].repeat_interleave(Hq // Hkv, dim=2)
    mha = oracle.prefill(oracle.Layer(Hq, Hq, D, 9, 1e4, 16), _bits(d["q"]), _bits(krep),
                         _bits(vrep), d["gate"].numpy())
    assert np.array_equal(gqa, mha)
    # an interleaved head mapping (h % Hkv) gives a different answer
    kint = d["k"].repeat(1, 1, Hq // Hkv, 1)
    vint = d["v"].repeat(1, 1, Hq // Hkv, 1)
    other = oracle.prefill(oracle.Layer(Hq, Hq, D, 9, 1e4, 16), _bits(d["q"]), _bits(kint),
                           _bits(vint), d["gate"].numpy())
    assert not np.allclose(gqa, other)
    # permuting q-heads within a group permutes the outputs
    perm = torch.tensor([1, 0, 3, 2, 5, 4, 7, 6])
    gp = oracle.prefill(oracle.Layer(Hq, Hkv, D, 9, 1e4, 16), _bits(d["q"][:, :, perm]),
                        _bits(d["k"]), _bits(d["v"]), d["gate"][:, :, perm].numpy())
    assert np.array_equal(gp, gqa[:, :, perm.numpy()])


# ---------------------------------------------------------------- RoPE pins

def test_rope_identity_cases():
    x = np.random.default_rng(0).standard_normal(128)
    assert np.array_equal(oracle.rope_f64(x, 1234, 0.0, 128), x)     # theta 0: no rotation
    assert np.array_equal(oracle.rope_f64(x, 1234, 1e4, 0), x)       # no rotary dims
    assert np.array_equal(oracle.rope_f64(x, 0, 1e4, 128), x)        # position 0
    y = oracle.rope_f64(x, 77, 5e6, 64)                               # partial rotary
    assert np.array_equal(y[64:], x[64:])
    assert not np.allclose(y[:64], x[:64])


@pytest.mark.parametrize("r,k,theta,omega", [
    (128, 0, 1e4, 1.0),        # theta^0 = 1
    (128, 32, 1e4, 0.01),      # 10000^(-64/128) = 1/100
    (64, 16, 1e4, 0.01),       # 10000^(-32/64)  = 1/100 (frequency uses rotary_dim)
    (64, 0, 5e6, 1.0),
    (8, 2, 1e4, 0.01),
])
def test_rope_unit_vector_angle(r, k, theta, omega):
    """e_k at position p turns into cos(p w) e_k + sin(p w) e_(k + r/2)."""
    D = 128
    for p in (1, 3, 100, 4097):
        e = np.zeros(D)
        e[k] = 1.0
        y = oracle.rope_f64(e, p, theta, r)
        expect = np.zeros(D)
        expect[k] = math.cos(p * omega)
        expect[k + r // 2] = math.sin(p * omega)
        np.testing.assert_allclose(y, expect, atol=1e-12)


def test_rope_group_norm_and_relativity():
    rng = np.random.default_rng(1)
    D, r, th = 128, 64, 5e6
    x = rng.standard_normal(D)
    # composition: rotating by p1 then p2 equals rotating by p1 + p2
    a = oracle.rope_f64(oracle.rope_f64(x, 300, th, r), 4000, th, r)
    b = oracle.rope_f64(x, 4300, th, r)
    np.testing.assert_allclose(a, b, atol=1e-10)
    # per-pair norms are preserved
    y = oracle.rope_f64(x, 131071, th, r)
    h = r // 2
    np.testing.assert_allclose(y[:h] ** 2 + y[h:r] ** 2, x[:h] ** 2 + x[h:r] ** 2, rtol=1e-12)
    # scores depend only on i - j
    q = rng.standard_normal(D)
    kk = rng.standard_normal(D)
    for delta in (0, 1, 17, 511):
        s = [oracle.rope_f64(q, j + delta, 1e4, 128) @ oracle.rope_f64(kk, j, 1e4, 128)
             for j in (0, 5, 1000, 60000)]
        np.testing.assert_allclose(s, s[0], rtol=0, atol=1e-9)


def test_rope_tensor_matches_vector_form():
    x = inputs.normal_bf16((5, 3, 128), 2, "q")
    pos = np.array([0, 1, 511, 4096, 131071])
    got = oracle.rope(_bits(x), pos, 1e4, 128)
    xf = oracle.bf16_bits_to_f64(_bits(x))
    for t in range(5):
        for h in range(3):
            assert np.array_equal(got[t, h], oracle.rope_f64(xf[t, h], pos[t], 1e4, 128))


# ---------------------------------------------------------- KV-cache sizing

def test_kv_cache_footprint_matches_page():
    g = json.load(open(os.path.join(GOLDEN, "kv_cache_footprint.json")))
    for c in g["cases"]:
        n = oracle.kv_cache_bytes(g["tokens"], c["kv_heads"], g["head_dim"], g["bytes_per_elem"],
                                  g["layers"])
        assert n == c["gib_printed"] * 2 ** 30      # exactly 6.5 GiB and 104 GiB


# ------------------------------------------------------------------ decode

def _ring_cache(k_rot, v, W, perm=None):
    """Place positions S-min(S,W)..S-1 at ring slot p mod W (fp64)."""
    S, Hkv, D = k_rot.shape
    kc = np.zeros((1, Hkv, W, D))
    vc = np.zeros((1, Hkv, W, D))
    for p in range(max(0, S - W), S):
        slot = p % W if perm is None else perm[p % W]
        kc[0, :, slot] = k_rot[p]
        vc[0, :, slot] = v[p]
    return kc, vc


@pytest.mark.parametrize("S,W", [(40, 8), (40, 40), (7, 16), (33, 1)])
def test_decode_equals_last_prefill_row(S, W):
    Hq, Hkv, D, th, r = 6, 2, 32, 1e4, 32
    d = inputs.prefill_inputs(1, S, Hq, Hkv, D, seed=31)
    lay = oracle.Layer(Hq, Hkv, D, W, th, r)
    pre = oracle.prefill(lay, _bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    pos = np.arange(S)
    k_rot = oracle.rope(_bits(d["k"][0]), pos, th, r)          # [S,Hkv,D]
    v = oracle.bf16_bits_to_f64(_bits(d["v"][0]))
    q_rot = oracle.rope(_bits(d["q"][0, S - 1:]), pos[S - 1:], th, r)   # [1,Hq,D]
    kc, vc = _ring_cache(k_rot, v, W)
    dec = oracle.decode_f64(lay, q_rot, d["gate"][:, S - 1].numpy(), kc, vc, np.array([S]))
    np.testing.assert_allclose(dec[0], pre[0, S - 1], rtol=1e-12, atol=1e-13)
    # ring slot order does not matter
    perm = inputs.permutation(W, 5).numpy()
    kc2, vc2 = _ring_cache(k_rot, v, W, perm)
    if S < W:   # only the first S slots are live; keep them in place
        kc2, vc2 = kc, vc
    dec2 = oracle.decode_f64(lay, q_rot, d["gate"][:, S - 1].numpy(), kc2, vc2, np.array([S]))
    np.testing.assert_allclose(dec2, dec, rtol=1e-12, atol=1e-13)
    # full layer: linear cache of capacity >= S
    full = oracle.Layer(Hq, Hkv, D, -1, th, r)
    pre_f = oracle.prefill(full, _bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    C = S + 5
    kcl = np.zeros((1, Hkv, C, D))
    vcl = np.zeros((1, Hkv, C, D))
    kcl[0, :, :S] = k_rot.transpose(1, 0, 2)
    vcl[0, :, :S] = v.transpose(1, 0, 2)
    dec_f = oracle.decode_f64(full, q_rot, d["gate"][:, S - 1].numpy(), kcl, vcl, np.array([S]))
    np.testing.assert_allclose(dec_f[0], pre_f[0, S - 1], rtol=1e-12, atol=1e-13)


def test_decode_bf16_cache_matches_f64_cache():
    B, Hq, Hkv, D, C = 3, 8, 2, 64, 50
    d = inputs.decode_inputs(B, Hq, Hkv, D, C, seed=12)
    lens = np.array([1, 37, 50], np.int32)
    lay = oracle.Layer(Hq, Hkv, D, -1, 5e6, 32)
    q = oracle.bf16_bits_to_f64(_bits(d["q"]))
    a = oracle.decode(lay, q, d["gate"].numpy(), _bits(d["k_cache"]), _bits(d["v_cache"]), lens)
    b = oracle.decode_f64(lay, q, d["gate"].numpy(), oracle.bf16_bits_to_f64(_bits(d["k_cache"])),
                          oracle.bf16_bits_to_f64(_bits(d["v_cache"])), lens)
    assert np.array_equal(a, b)
    rows = np.array([[2, 7], [0, 0], [1, 4]], np.int64)
    sub = oracle.decode(lay, q, d["gate"].numpy(), _bits(d["k_cache"]), _bits(d["v_cache"]), lens,
                        rows=rows)
    for t, (bb, h) in enumerate(rows):
        assert np.array_equal(sub[t], a[bb, h])
    # sliding ring: seq longer than W uses all W slots, shorter uses the first L
    W = 16
    ds = inputs.decode_inputs(2, Hq, Hkv, D, W, seed=13)
    lens_s = np.array([5, 1000], np.int32)
    lay_s = oracle.Layer(Hq, Hkv, D, W, 1e4, 64)
    qs = oracle.bf16_bits_to_f64(_bits(ds["q"]))
    got = oracle.decode(lay_s, qs, None, _bits(ds["k_cache"]), _bits(ds["v_cache"]), lens_s)
    kf = oracle.bf16_bits_to_f64(_bits(ds["k_cache"]))
    vf = oracle.bf16_bits_to_f64(_bits(ds["v_cache"]))
    for b, n in ((0, 5), (1, 16)):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            s = kf[b, kv, :n] @ qs[b, h] / math.sqrt(D)
            w = np.exp(s - s.max())
            w /= w.sum()
            np.testing.assert_allclose(got[b, h], w @ vf[b, kv, :n], rtol=1e-12, atol=1e-14)


def test_decode_new_token_override():
    B, Hq, Hkv, D, W = 1, 4, 2, 16, 8
    d = inputs.decode_inputs(B, Hq, Hkv, D, W, seed=14)
    lens = np.array([21], np.int32)                 # current position 20 -> slot 4
    lay = oracle.Layer(Hq, Hkv, D, W, 1e4, 16)
    q = oracle.bf16_bits_to_f64(_bits(d["q"]))
    kn = np.random.default_rng(2).standard_normal((B, Hkv, D))
    vn = np.random.default_rng(3).standard_normal((B, Hkv, D))
    got = oracle.decode(lay, q, d["gate"].numpy(), _bits(d["k_cache"]), _bits(d["v_cache"]), lens,
                        k_new=kn, v_new=vn)
    kc = oracle.bf16_bits_to_f64(_bits(d["k_cache"]))
    vc = oracle.bf16_bits_to_f64(_bits(d["v_cache"]))
    kc[:, :, 20 % W] = kn
    vc[:, :, 20 % W] = vn
    ref = oracle.decode_f64(lay, q, d["gate"].numpy(), kc, vc, lens)
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)


# ---- caller-supplied frequency tables (the full layers' YaRN scaling of the
# Step explainer's section 2.3, whose parameters the page leaves open)

def _scaled_table(theta, r, factor=2.0, keep_above=0.05, scale_below=0.002):
    """A long-context table of the kind a caller passes: high frequencies
    kept, low ones divided by `factor`, a linear blend in between."""
    k = np.arange(r // 2, dtype=np.float64)
    w = theta ** (-2.0 * k / r)
    t = np.clip((np.log(w) - np.log(scale_below)) / (np.log(keep_above) - np.log(scale_below)), 0.0, 1.0)
    return w / (factor * (1.0 - t) + t)


def test_rope_table_of_theta_frequencies_is_theta_rope():
    theta, r = 5e6, 64
    table = theta ** (-2.0 * np.arange(r // 2) / r)
    d = inputs.prefill_inputs(1, 40, 4, 2, 128, seed=71)
    x = _bits(d["k"])[0]
    pos = np.arange(40, dtype=np.int64)
    np.testing.assert_allclose(oracle.rope_table(x, pos, table, r), oracle.rope(x, pos, theta, r),
                               rtol=1e-12, atol=1e-12)
    a = oracle.prefill(oracle.Layer(4, 2, 128, -1, theta, r), _bits(d["q"]), _bits(d["k"]), _bits(d["v"]),
                       d["gate"].numpy())
    b = oracle.prefill(oracle.Layer(4, 2, 128, -1, theta, r, inv_freq=tuple(table)), _bits(d["q"]),
                       _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    np.testing.assert_allclose(b, a, rtol=1e-11, atol=1e-12)


def test_rope_table_half_frequency_is_half_position():
    """Halving every frequency turns a vector at position p exactly as the
    unhalved table turns it at p / 2 (p even: both angles are one rounding
    of p * w / 2)."""
    rng = np.random.default_rng(3)
    table = rng.uniform(1e-6, 1.0, 32)
    for p in (2, 100, 4096, 131070):
        x = rng.standard_normal(128)
        np.testing.assert_array_equal(oracle.rope_f64_table(x, p, table / 2, 64),
                                      oracle.rope_f64_table(x, p // 2, table, 64))


@pytest.mark.parametrize("k", [0, 7, 31])
def test_rope_table_unit_vector_angle(k):
    """e_k turns by p * table[k] into the plane (e_k, e_(k + r/2))."""
    table = _scaled_table(5e6, 64)
    for p in (1, 17, 8191, 100003):
        e = np.zeros(128)
        e[k] = 1.0
        y = oracle.rope_f64_table(e, p, table, 64)
        expect = np.zeros(128)
        expect[k] = math.cos(p * table[k])
        expect[k + 32] = math.sin(p * table[k])
        np.testing.assert_allclose(y, expect, atol=1e-12)


@pytest.mark.parametrize("W", [-1, 24])
def test_prefill_with_table_matches_torch_sdpa(W):
    table = _scaled_table(5e6, 64)
    d = inputs.prefill_inputs(2, 48, 6, 2, 128, seed=73)
    lay = oracle.Layer(6, 2, 128, W, 5e6, 64, inv_freq=tuple(table))
    got = oracle.prefill(lay, _bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    ref = _sdpa_reference(d["q"], d["k"], d["v"], d["gate"], W, 5e6, 64, freq=table)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


# ---- multi-query decode (T new tokens per sequence: the MTP layers' drafts
# checked in one call; Step spec card config dump, Step explainer section 2.2)

def _mq_setup(L, T, W, C=None, seed=81, Hq=6, Hkv=2, D=32):
    """Inputs of one sequence of L tokens without RoPE (theta 0, so cached
    keys are the raw bf16 keys); the cache holds the first L - T tokens."""
    d = inputs.prefill_inputs(1, L, Hq, Hkv, D, seed=seed)
    L0 = L - T
    C = (W if W > 0 else L0 + 3) if C is None else C
    kb, vb = _bits(d["k"])[0], _bits(d["v"])[0]            # [L, Hkv, D] uint16
    kc = np.zeros((1, Hkv, C, D), np.uint16)
    vc = np.zeros((1, Hkv, C, D), np.uint16)
    for p in range(max(0, L0 - W) if W > 0 else 0, L0):
        slot = p % W if W > 0 else p
        kc[0, :, slot] = kb[p]
        vc[0, :, slot] = vb[p]
    return d, kc, vc, kb[None, L0:], vb[None, L0:]


@pytest.mark.parametrize("L,T,W", [(40, 4, 8), (40, 3, 40), (7, 4, 16), (33, 2, 1), (5, 5, 8), (12, 4, 3),
                                   (50, 1, 16), (64, 4, -1), (4, 4, -1)])
def test_decode_mq_equals_prefill_rows(L, T, W):
    """Each of the T queries equals the whole-sequence prefill's row at its
    position: the cache part, the new-token part and the per-query band."""
    Hq, Hkv, D = 6, 2, 32
    d, kc, vc, kn, vn = _mq_setup(L, T, W)
    lay = oracle.Layer(Hq, Hkv, D, W, 0.0, 0)
    pre = oracle.prefill(lay, _bits(d["q"]), _bits(d["k"]), _bits(d["v"]), d["gate"].numpy())
    q = oracle.bf16_bits_to_f64(_bits(d["q"]))[:, L - T:]
    got = oracle.decode_mq(lay, q, d["gate"][:, L - T:].numpy(), kc, vc, np.array([L]), kn, vn)
    np.testing.assert_allclose(got[0], pre[0, L - T:], rtol=1e-12, atol=1e-13)
    rows = np.array([[0, T - 1, 5], [0, 0, 0], [0, T // 2, 3]], np.int64)
    sub = oracle.decode_mq(lay, q, d["gate"][:, L - T:].numpy(), kc, vc, np.array([L]), kn, vn, rows=rows)
    for i, (b, t, h) in enumerate(rows):
        assert np.array_equal(sub[i], got[b, t, h])


@pytest.mark.parametrize("W", [8, 16])
def test_decode_mq_ignores_slots_outside_every_band(W):
    """The oldest ring entry (position L0 - W) is outside every query's band,
    and unfilled slots of a short ring are never read: NaN there changes
    nothing."""
    for L, T in ((40, 3), (9, 4)):
        d, kc, vc, kn, vn = _mq_setup(L, T, W)
        lay = oracle.Layer(6, 2, 32, W, 0.0, 0)
        q = oracle.bf16_bits_to_f64(_bits(d["q"]))[:, L - T:]
        ref = oracle.decode_mq(lay, q, None, kc, vc, np.array([L]), kn, vn)
        L0 = L - T
        nan = np.uint16(0x7FC0)
        kc2, vc2 = kc.copy(), vc.copy()
        dead = [(L0 - W) % W] if L0 >= W else list(range(L0, W))
        for slot in dead:
            kc2[0, :, slot] = nan
            vc2[0, :, slot] = nan
        got = oracle.decode_mq(lay, q, None, kc2, vc2, np.array([L]), kn, vn)
        assert np.array_equal(got, ref)


def test_decode_mq_one_query_is_decode_after_append():
    """T = 1: the same result as appending the token to the cache and running
    the one-query decode (ring and linear caches, several lengths)."""
    B, Hq, Hkv, D, W = 3, 8, 2, 32, 16
    lens = np.array([1, 16, 45], np.int32)
    for window, C in ((W, W), (-1, 50)):
        dd = inputs.decode_inputs(B, Hq, Hkv, D, C, seed=83)
        new = inputs.prefill_inputs(B, 1, Hq, Hkv, D, seed=84)
        kc, vc = _bits(dd["k_cache"]).copy(), _bits(dd["v_cache"]).copy()
        kn, vn = _bits(new["k"]), _bits(new["v"])
        lay = oracle.Layer(Hq, Hkv, D, window, 1e4, 32)
        q = oracle.bf16_bits_to_f64(_bits(new["q"]))                 # [B,1,Hq,D]
        got = oracle.decode_mq(lay, q, new["gate"].numpy(), kc, vc, lens, kn, vn)
        for b, Lb in enumerate(lens):
            slot = (Lb - 1) % W if window > 0 else Lb - 1
            kc[b, :, slot] = kn[b, 0]
            vc[b, :, slot] = vn[b, 0]
        ref = oracle.decode(lay, q[:, 0], new["gate"][:, 0].numpy(), kc, vc, lens)
        np.testing.assert_allclose(got[:, 0], ref, rtol=1e-13, atol=1e-14)


def test_decode_mq_rejects_bad_lengths():
    d, kc, vc, kn, vn = _mq_setup(10, 4, 8)
    lay = oracle.Layer(6, 2, 32, 8, 0.0, 0)
    q = oracle.bf16_bits_to_f64(_bits(d["q"]))[:, 6:]
    with pytest.raises(ValueError):
        oracle.decode_mq(lay, q, None, kc, vc, np.array([3]), kn, vn)          # fewer tokens than T
    with pytest.raises(ValueError):
        oracle.decode_mq(lay, q, None, kc[:, :, :4], vc[:, :, :4], np.array([10]), kn, vn)   # ring != W
