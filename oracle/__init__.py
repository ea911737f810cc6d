"""fp64 CPU oracle for banded/causal GQA attention with RoPE and a head gate.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its binding) never calls it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over independent
rows); this module only builds that file with gcc, loads it with ctypes and
marshals numpy arrays.  Passages followed (page title, section):

* "Step-3.7-Flash-oQ3e" explainer, section 2.2 -- full layers use a plain
  causal mask, sliding layers a sliding-window causal mask and keep the last
  512 tokens of KV cache.  Reading: query i sees key j iff i-W < j <= i.
* same page, section 2.3 -- per-layer rope_theta, partial rotary on full
  layers, per-head sigmoid output gate.  Readings: first ``rotary_dim`` dims,
  rotate-half pairs, frequency theta^(-2k/rotary_dim); one gate logit per
  (token, q-head) multiplying the normalised attention output.
* "Step-3.7-Flash" spec card, config dump -- 64 q-heads in 8 attention
  groups (GQA); reading: kv head = h // (Hq // Hkv).
* "Muse-Glimmer-30B-6bit" explainer, RoPE section -- rope theta 0 means no
  rotary encoding; GQA section -- KV-cache footprint arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

WINDOW_FULL = -1


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("rope_theta", ctypes.c_double),
        ("rotary_dim", ctypes.c_int32),
        ("softmax_scale", ctypes.c_double),
        ("inv_freq", ctypes.c_void_p),
    ]


@dataclass(frozen=True)
class Layer:
    """One attention layer's parameters as the pages state them.

    window: W >= 1 for a sliding layer (W keys including self), -1 for full.
    rope_theta: 0 means no rotary encoding.  softmax_scale <= 0: 1/sqrt(D).
    inv_freq: rotary_dim/2 angular frequencies replacing theta^(-2k/r)
    (caller-scaled RoPE, e.g. the full layers' YaRN of the Step explainer's
    section 2.3), or None.
    """

    num_q_heads: int
    num_kv_heads: int
    head_dim: int = 128
    window: int = WINDOW_FULL
    rope_theta: float = 10000.0
    rotary_dim: int = 128
    softmax_scale: float = 0.0
    inv_freq: tuple = None

    def __post_init__(self):
        freq = None
        if self.inv_freq is not None:
            freq = np.ascontiguousarray(self.inv_freq, dtype=np.float64)
            assert freq.shape == (self.rotary_dim // 2,)
        object.__setattr__(self, "_freq", freq)  # kept alive with the layer

    def _c(self) -> _Layer:
        return _Layer(self.num_q_heads, self.num_kv_heads, self.head_dim, self.window,
                      float(self.rope_theta), self.rotary_dim, float(self.softmax_scale),
                      None if self._freq is None else self._freq.ctypes.data)


_lib = None


def _configure(lib):
    """Set the argument and result types of every oracle entry point on a
    loaded library (the built liboracle.so, or a test's variant of it)."""
    P = ctypes.POINTER
    lib.oracle_rope.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                ctypes.c_void_p, ctypes.c_double, ctypes.c_int32, ctypes.c_void_p]
    lib.oracle_rope.restype = ctypes.c_int
    lib.oracle_rope_table.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    lib.oracle_rope_table.restype = ctypes.c_int
    lib.oracle_rope_vec_table.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double]
    lib.oracle_rope_vec_table.restype = None
    lib.oracle_prefill.argtypes = [P(_Layer), ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32]
    lib.oracle_prefill.restype = ctypes.c_int
    lib.oracle_prefill_materialised.argtypes = [P(_Layer), ctypes.c_int32, ctypes.c_int32,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.oracle_prefill_materialised.restype = ctypes.c_int
    lib.oracle_decode.argtypes = [P(_Layer), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_int32]
    lib.oracle_decode.restype = ctypes.c_int
    lib.oracle_decode_f64.argtypes = [P(_Layer), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                      ctypes.c_void_p, ctypes.c_void_p]
    lib.oracle_decode_f64.restype = ctypes.c_int
    lib.oracle_decode_mq.argtypes = [P(_Layer), ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32]
    lib.oracle_decode_mq.restype = ctypes.c_int
    lib.oracle_kv_cache_bytes.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_int32]
    lib.oracle_kv_cache_bytes.restype = ctypes.c_int64
    lib.oracle_visible_count.argtypes = [ctypes.c_int64, ctypes.c_int32]
    lib.oracle_visible_count.restype = ctypes.c_int64
    lib.oracle_rope_vec.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                    ctypes.c_double]
    lib.oracle_rope_vec.restype = None
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(build()))
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 data as its raw 16-bit patterns (numpy has no bf16 type)."""
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        a = a.view(np.uint16) if a.dtype.itemsize == 2 else None
    if a is None:
        raise TypeError("expected bf16 bit patterns as a uint16/int16 array")
    return a


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def rope(x_bf16, pos, theta: float, rotary_dim: int) -> np.ndarray:
    """RoPE of x[T, H, D] (bf16 bits) with token t at position pos[t]; fp64 out."""
    x = _u16(x_bf16)
    T, H, D = x.shape
    p = np.ascontiguousarray(pos, dtype=np.int64)
    assert p.shape == (T,)
    out = np.empty((T, H, D), np.float64)
    _check(_load().oracle_rope(_ptr(x), T, H, D, _ptr(p), float(theta), rotary_dim, _ptr(out)), "rope")
    return out


def rope_table(x_bf16, pos, inv_freq, rotary_dim: int) -> np.ndarray:
    """RoPE of x[T, H, D] (bf16 bits) at positions pos[t] with pair k turned
    at frequency inv_freq[k]; fp64 out."""
    x = _u16(x_bf16)
    T, H, D = x.shape
    p = np.ascontiguousarray(pos, dtype=np.int64)
    f = np.ascontiguousarray(inv_freq, dtype=np.float64)
    assert p.shape == (T,) and f.shape == (rotary_dim // 2,)
    out = np.empty((T, H, D), np.float64)
    _check(_load().oracle_rope_table(_ptr(x), T, H, D, _ptr(p), _ptr(f), rotary_dim, _ptr(out)), "rope_table")
    return out


def rope_f64_table(x, p: float, inv_freq, rotary_dim: int) -> np.ndarray:
    """Table-frequency RoPE of one fp64 head vector x[D] at position p."""
    y = np.array(x, dtype=np.float64, copy=True)
    f = np.ascontiguousarray(inv_freq, dtype=np.float64)
    assert y.ndim == 1 and f.shape == (rotary_dim // 2,)
    _load().oracle_rope_vec_table(_ptr(y), rotary_dim, _ptr(f), float(p))
    return y


def rope_f64(x, p: float, theta: float, rotary_dim: int) -> np.ndarray:
    """RoPE of one fp64 head vector x[D] at position p (returns a copy)."""
    y = np.array(x, dtype=np.float64, copy=True)
    assert y.ndim == 1
    _load().oracle_rope_vec(_ptr(y), y.shape[0], rotary_dim, float(theta), float(p))
    return y


def prefill(layer: Layer, q, k, v, gate=None, rows=None, threads: int = 0) -> np.ndarray:
    """Prefill attention at positions 0..S-1 on un-rotated bf16 q/k/v.

    q [B,S,Hq,D], k/v [B,S,Hkv,D] as bf16 bits; gate [B,S,Hq] float32 or None.
    rows: int64 array [n, 3] of (b, i, h), or None for every row.
    Returns fp64 [B,S,Hq,D] (rows None) or [n, D].
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, S, Hq, D = q.shape
    assert Hq == layer.num_q_heads and D == layer.head_dim
    assert k.shape == v.shape == (B, S, layer.num_kv_heads, D)
    g = None if gate is None else np.ascontiguousarray(gate, dtype=np.float32)
    if g is not None:
        assert g.shape == (B, S, Hq)
    if rows is None:
        r, n = None, 0
        out = np.empty((B, S, Hq, D), np.float64)
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
        n = r.shape[0]
        out = np.empty((n, D), np.float64)
    lay = layer._c()
    _check(_load().oracle_prefill(ctypes.byref(lay), B, S, _ptr(q), _ptr(k), _ptr(v), _ptr(g), n,
                                  _ptr(r), _ptr(out), threads), "prefill")
    return out


def prefill_materialised(layer: Layer, q, k, v, gate=None, want_weights: bool = False):
    """Tiny-input variant: full S x S masked score matrix, row softmax, @ V.

    Returns out [B,S,Hq,D] and, if asked, the probability matrices
    [B,Hq,S,S].
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, S, Hq, D = q.shape
    g = None if gate is None else np.ascontiguousarray(gate, dtype=np.float32)
    out = np.empty((B, S, Hq, D), np.float64)
    w = np.empty((B, Hq, S, S), np.float64) if want_weights else None
    lay = layer._c()
    _check(_load().oracle_prefill_materialised(ctypes.byref(lay), B, S, _ptr(q), _ptr(k), _ptr(v),
                                               _ptr(g), _ptr(out), _ptr(w)), "prefill_materialised")
    return (out, w) if want_weights else out


def decode(layer: Layer, q_rot, gate, k_cache, v_cache, seq_lens, k_new=None, v_new=None,
           rows=None, threads: int = 0) -> np.ndarray:
    """One-query decode over a bf16 cache [B,Hkv,C,D] (rotated K, raw V).

    q_rot [B,Hq,D] fp64 (after RoPE); gate [B,Hq] float32 or None;
    seq_lens [B] counts the current token (query position L_b - 1).
    k_new/v_new [B,Hkv,D] fp64 optionally replace the current token's slot.
    rows: int64 [n, 2] of (b, h) or None.  Returns fp64 [B,Hq,D] or [n, D].
    """
    kc, vc = _u16(k_cache), _u16(v_cache)
    B, Hkv, C, D = kc.shape
    q = np.ascontiguousarray(q_rot, dtype=np.float64)
    assert q.shape == (B, layer.num_q_heads, D)
    g = None if gate is None else np.ascontiguousarray(gate, dtype=np.float32)
    L = np.ascontiguousarray(seq_lens, dtype=np.int32)
    kn = None if k_new is None else np.ascontiguousarray(k_new, dtype=np.float64)
    vn = None if v_new is None else np.ascontiguousarray(v_new, dtype=np.float64)
    if rows is None:
        r, n = None, 0
        out = np.empty((B, layer.num_q_heads, D), np.float64)
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
        n = r.shape[0]
        out = np.empty((n, D), np.float64)
    lay = layer._c()
    _check(_load().oracle_decode(ctypes.byref(lay), B, _ptr(q), _ptr(g), _ptr(kc), _ptr(vc), C,
                                 _ptr(L), _ptr(kn), _ptr(vn), n, _ptr(r), _ptr(out), threads), "decode")
    return out


def decode_f64(layer: Layer, q_rot, gate, k_cache, v_cache, seq_lens) -> np.ndarray:
    """decode() with an fp64 cache (tiny self-checks only)."""
    kc = np.ascontiguousarray(k_cache, dtype=np.float64)
    vc = np.ascontiguousarray(v_cache, dtype=np.float64)
    B, Hkv, C, D = kc.shape
    q = np.ascontiguousarray(q_rot, dtype=np.float64)
    g = None if gate is None else np.ascontiguousarray(gate, dtype=np.float32)
    L = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.empty((B, layer.num_q_heads, D), np.float64)
    lay = layer._c()
    _check(_load().oracle_decode_f64(ctypes.byref(lay), B, _ptr(q), _ptr(g), _ptr(kc), _ptr(vc), C,
                                     _ptr(L), _ptr(out)), "decode_f64")
    return out


def decode_mq(layer: Layer, q_rot, gate, k_cache, v_cache, seq_lens, k_new, v_new, rows=None,
              threads: int = 0) -> np.ndarray:
    """Multi-query decode: T new tokens per sequence at positions
    L_b - T .. L_b - 1 (L_b = seq_lens[b]); the bf16 cache [B,Hkv,C,D] holds
    the L_b - T earlier tokens (ring slot p mod W, or slot p), the new
    tokens' rotated keys / raw values are k_new / v_new [B,T,Hkv,D] bf16.

    q_rot [B,T,Hq,D] fp64 (after RoPE); gate [B,T,Hq] float32 or None.
    rows: int64 [n, 3] of (b, t, h) or None.  Returns fp64 [B,T,Hq,D] or [n, D].
    """
    kc, vc = _u16(k_cache), _u16(v_cache)
    kn, vn = _u16(k_new), _u16(v_new)
    B, Hkv, C, D = kc.shape
    T = kn.shape[1]
    assert kn.shape == (B, T, Hkv, D) and vn.shape == kn.shape
    q = np.ascontiguousarray(q_rot, dtype=np.float64)
    assert q.shape == (B, T, layer.num_q_heads, D)
    g = None if gate is None else np.ascontiguousarray(gate, dtype=np.float32)
    L = np.ascontiguousarray(seq_lens, dtype=np.int32)
    if rows is None:
        r, n = None, 0
        out = np.empty((B, T, layer.num_q_heads, D), np.float64)
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
        n = r.shape[0]
        out = np.empty((n, D), np.float64)
    lay = layer._c()
    _check(_load().oracle_decode_mq(ctypes.byref(lay), B, T, _ptr(q), _ptr(g), _ptr(kc), _ptr(vc), C, _ptr(L),
                                    _ptr(kn), _ptr(vn), n, _ptr(r), _ptr(out), threads), "decode_mq")
    return out


def kv_cache_bytes(tokens: int, kv_heads: int, head_dim: int, bytes_per_elem: int, layers: int) -> int:
    """tokens x kv_heads x head_dim x 2 (K and V) x bytes x layers."""
    return int(_load().oracle_kv_cache_bytes(tokens, kv_heads, head_dim, bytes_per_elem, layers))


def visible_count(i: int, window: int) -> int:
    """Number of keys query position i sees under window W (-1: full)."""
    return int(_load().oracle_visible_count(i, window))


def bf16_bits_to_f64(a) -> np.ndarray:
    """Exact value of bf16 bit patterns as fp64 (for comparisons)."""
    u = _u16(a).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
