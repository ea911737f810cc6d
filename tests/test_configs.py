"""The workloads in configs.py carry the values the pages print
(tests/golden/layer_configs.json, each entry with its citation): head
counts, windows, rope thetas, partial rotary factors, and the number of MTP
layers behind the multi-query decode's T."""
import json
import os

from full_gqa_attention_swa_b200 import configs

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "layer_configs.json")))


def test_step_layers():
    g = GOLDEN["step37"]
    D = g["head_dim"]
    Hkv = g["num_attention_groups"]
    for c in (configs.STEP_SLIDING, configs.DECODE_SLIDING, configs.CHUNK_SLIDING, configs.MQ_SLIDING):
        assert (c.Hq, c.Hkv, c.D, c.window) == (g["sliding_q_heads"], Hkv, D, g["sliding_window"]), c.name
        assert (c.theta, c.rotary_dim) == (g["rope_theta_sliding"], int(g["partial_rotary_sliding"] * D)), c.name
    for c in (configs.STEP_FULL, configs.DECODE_FULL, configs.CHUNK_FULL, configs.MQ_FULL):
        assert (c.Hq, c.Hkv, c.D, c.window) == (g["num_attention_heads"], Hkv, D, configs.WINDOW_FULL), c.name
        assert (c.theta, c.rotary_dim) == (g["rope_theta_full"], int(g["partial_rotary_full"] * D)), c.name


def test_muse_layers():
    g = GOLDEN["muse"]
    for c in (configs.MUSE_SLIDING, configs.MUSE_FULL):
        assert (c.Hq, c.Hkv, c.D) == (g["num_attention_heads"], g["num_kv_heads"], g["head_dim"]), c.name
    assert (configs.MUSE_SLIDING.window, configs.MUSE_SLIDING.theta) == (g["sliding_window"], g["rope_theta_sliding"])
    assert (configs.MUSE_FULL.window, configs.MUSE_FULL.theta) == (configs.WINDOW_FULL, g["rope_theta_full"])


def test_multi_query_decode_checks_every_mtp_draft():
    """T = the token being decoded plus one draft per MTP layer."""
    for c in configs.MULTI_QUERY.values():
        assert c.T == GOLDEN["step37"]["mtp_layers"] + 1, c.name
