"""Host-side helpers of bench.py, pinned to the pages' worked KV-size example."""
import json
import os

import bench

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_size_llama3_70b_100k.json")


def test_dense_kv_bytes_matches_worked_example():
    g = json.load(open(GOLDEN))
    b = bench.dense_kv_bytes(g["layers"], g["kv_heads"], g["head_dim"], g["tokens"], g["elem_bytes"])
    assert b == g["bytes_exact"]
    assert round(b / 1e9, 1) == g["printed_gb"]


def test_token_bytes_of_the_64k_workload():
    # tier ranks 16 / 32 / 64, s = 16 int4: 2 * (2r + 16 + 8 + 2)
    assert [bench.token_bytes(r, 16, 4) for r in (16, 32, 64)] == [116, 180, 308]
    # expected bytes per (layer, kv-head) token at tier probabilities 0.6 / 0.3 / 0.1
    mean = 0.6 * 116 + 0.3 * 180 + 0.1 * 308
    assert abs(mean - 154.4) < 1e-9


def test_measured_peaks_is_read():
    p = bench.measured_peaks()
    assert p["hbm_gbs"] > 1000
