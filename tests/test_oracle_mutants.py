"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a copy of oracle/oracle.c (an
off-by-one band edge, a flipped rotation or gate sign, an interleaved GQA
mapping, a dropped scale or normalisation, a wrong cache slot, ...), builds
the copy with the oracle's own compiler flags, swaps it in for the real
library and runs the pins of tests/test_oracle.py against it: at least one
pin must fail.  The unmodified copy, built the same way, must pass them all,
so a failure is the planted mistake and nothing else.  oracle.c itself is
never changed; everything happens on the CPU.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "oracle.c")

# name -> edits (text in oracle.c, replacement, occurrences replaced: None for all)
MUTANTS = {
    # band edge one key too wide in the streaming prefill: W + 1 keys per row
    "prefill band off by one": [("? ri - (int64_t)L->window + 1 : 0;", "? ri - (int64_t)L->window : 0;", None)],
    # the visibility predicate used by the materialised prefill and the multi-query decode
    "visible() off by one": [("return j > i - (int64_t)W;", "return j >= i - (int64_t)W;", None)],
    # rotation sign of the first element of each pair
    "rope sign": [("x[k] = a * c - b * s;", "x[k] = a * c + b * s;", 1)],
    # positions counted from 1 (invisible to relativity, visible to absolute angles)
    "rope position off by one": [("double phi = p * freq;", "double phi = (p + 1.0) * freq;", None)],
    # q-head h reads kv-head h mod Hkv instead of h / G (prefill and decode)
    "gqa interleaved": [("rh / G == kvh", "rh % Hkv == kvh", None), ("rh / G != kvh", "rh % Hkv != kvh", None)],
    "gate sign": [("return 1.0 / (1.0 + exp(-g));", "return 1.0 / (1.0 + exp(g));", None)],
    "softmax scale dropped": [("        s *= scale;\n", "", None)],
    "softmax not normalised": [("double w = scratch[j] / denom;", "double w = scratch[j];", None)],
    "keys used as values": [("out[d] += w * vals[j * D + d];", "out[d] += w * keys[j * D + d];", None)],
    "decode token in the next slot": [("(Lb - 1) % L->window : Lb - 1;", "Lb % L->window : Lb - 1;", None)],
    "multi-query ring slot shifted": [("const int64_t slot = W > 0 ? j % W : j;",
                                       "const int64_t slot = W > 0 ? (j + 1) % W : j;", None)],
    "bf16 low mantissa bits dropped": [("uint32_t u = ((uint32_t)b) << 16;",
                                        "uint32_t u = ((uint32_t)(b & 0xFF80u)) << 16;", None)],
}


def _battery():
    """The pins, with fixed parameters, as (label, callable) pairs."""
    out = [(f"sdpa {c}", (lambda c=c: pins.test_prefill_matches_torch_sdpa(*c))) for c in pins.CASES]
    out += [(f"streaming == materialised {c}", (lambda c=c: pins.test_streaming_equals_materialised(*c)))
            for c in pins.CASES]
    out += [(f"uniform-score probe W={w}", (lambda w=w: pins.test_uniform_score_probe_counts(w))) for w in (3, 64, -1)]
    out += [
        ("row subset == all rows", pins.test_rows_subset_matches_all_rows),
        ("window one", pins.test_window_one_returns_gated_value),
        ("gate limits", pins.test_gate_limits),
        ("gqa == repeated mha", pins.test_gqa_contiguous_groups_equal_repeated_mha),
        ("rope angle theta^0", lambda: pins.test_rope_unit_vector_angle(128, 0, 1e4, 1.0)),
        ("rope angle 1/100", lambda: pins.test_rope_unit_vector_angle(128, 32, 1e4, 0.01)),
        ("rope identity", pins.test_rope_identity_cases),
        ("rope norm / relativity", pins.test_rope_group_norm_and_relativity),
        ("decode == last prefill row", lambda: pins.test_decode_equals_last_prefill_row(40, 8)),
        ("decode new-token override", pins.test_decode_new_token_override),
        ("multi-query == prefill rows", lambda: pins.test_decode_mq_equals_prefill_rows(40, 4, 8)),
        ("multi-query dead slot", lambda: pins.test_decode_mq_ignores_slots_outside_every_band(8)),
    ]
    return out


def _failures():
    failed = []
    for label, fn in _battery():
        try:
            fn()
        except (AssertionError, RuntimeError, ValueError) as e:  # a wrong value, or the oracle refusing
            failed.append((label, type(e).__name__))
    return failed


def _build(tmp_path, name, text):
    c = tmp_path / f"{name}.c"
    c.write_text(text)
    so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", str(so), str(c), "-lm"], check=True,
                   capture_output=True)
    return oracle._configure(ctypes.CDLL(str(so)))


def test_unmodified_copy_passes_every_pin(tmp_path, monkeypatch):
    monkeypatch.setattr(oracle, "_lib", _build(tmp_path, "copy", open(SRC).read()))
    assert _failures() == []


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, monkeypatch, name):
    src = open(SRC).read()
    mutant = src
    for old, new, count in MUTANTS[name]:
        assert old in mutant, f"mutation site of '{name}' not found in oracle.c"
        mutant = mutant.replace(old, new) if count is None else mutant.replace(old, new, count)
    assert mutant != src
    monkeypatch.setattr(oracle, "_lib", _build(tmp_path, "mutant", mutant))
    failed = _failures()
    assert failed, f"no pin catches '{name}'"
