"""Byte accounting pinned to the worked KV-cache example printed on the architecture
evolution page (walkthrough steps 4 and 5) and to the cache-size formula of the
compressed-sparse-attention comparison article (part 3.1)."""
import json
import os

from compressed_sparse_kv_fp32_b200 import accounting

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_cache_size_example.json")


def test_worked_kv_cache_example():
    g = json.load(open(GOLDEN))
    per_pos_layer = accounting.kv_cache_bytes(1, 1, g["kv_heads"], g["head_dim"], g["head_dim"],
                                              g["bytes_per_value"])
    assert per_pos_layer // g["bytes_per_value"] == g["numbers_per_position_per_layer"]
    per_pos = accounting.kv_cache_bytes(1, g["layers"], g["kv_heads"], g["head_dim"],
                                        g["head_dim"], g["bytes_per_value"])
    assert per_pos == g["bytes_per_position"]
    assert per_pos // g["bytes_per_value"] == g["numbers_per_position"]
    total = accounting.kv_cache_bytes(g["positions"], g["layers"], g["kv_heads"], g["head_dim"],
                                      g["head_dim"], g["bytes_per_value"])
    assert abs(total / 1e9 - g["total_gb_approx"]) / g["total_gb_approx"] < 0.06
    ungrouped = accounting.kv_cache_bytes(g["positions"], g["layers"], g["ungrouped_heads"],
                                          g["head_dim"], g["head_dim"], g["bytes_per_value"])
    assert ungrouped == 8 * total
    assert abs(ungrouped / 1e9 - g["ungrouped_total_gb_approx"]) / 320 < 0.06


def test_decode_step_bytes_128k_budget_1024():
    b = accounting.decode_step_bytes([131072], Hq=32, Hkv=32, budget=1024)
    assert b["codes"] == 128 * 2**20
    assert b["kv_rows"] == 16 * 2**20
    assert b["q"] == 32 * 128 * 2
    assert b["total"] == 144 * 2**20 + 8192


def test_decode_step_bytes_short_sequences_cap_rows():
    b = accounting.decode_step_bytes([10, 0], Hq=4, Hkv=2, budget=64)
    assert b["kv_rows"] == 4 * 10 * 512
    assert b["codes"] == 2 * 10 * 32


def test_encode_bytes_per_vector():
    assert accounting.encode_bytes_per_vector() == 288
