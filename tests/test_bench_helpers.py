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


def test_pack_step_inputs_round_trips_with_aligned_parts():
    import torch
    steps = 3
    k = torch.randn(steps, 4, 1, 8, 128).to(torch.bfloat16)
    q = torch.randn(steps, 4, 1, 32, 128).to(torch.bfloat16)
    t = torch.randint(0, 3, (steps, 2, 1, 5), dtype=torch.uint8)       # 10 bytes: forces padding
    c = torch.randn(steps, 3).to(torch.bfloat16)
    block, offs, sizes = bench.pack_step_inputs((k, t, q, c))
    assert all(o % 16 == 0 for o in offs)
    assert block.shape == (steps, offs[-1] + sizes[-1])
    for i in range(steps):
        row = block[i]
        assert torch.equal(row[offs[0]:offs[0] + sizes[0]].view(torch.bfloat16).view(k.shape[1:]), k[i])
        assert torch.equal(row[offs[1]:offs[1] + sizes[1]].view(t.shape[1:]), t[i])
        assert torch.equal(row[offs[2]:offs[2] + sizes[2]].view(torch.bfloat16).view(q.shape[1:]), q[i])
        assert torch.equal(row[offs[3]:offs[3] + sizes[3]].view(torch.bfloat16).view(c.shape[1:]), c[i])


def test_fp32_alu_peak_from_unit_counts_and_clock():
    # 148 SMs x 128 fp32 lanes x 2 flops (one FMA) x 1965 MHz
    assert abs(bench.fp32_alu_peak_tflops(1965.0) - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9
    assert abs(bench.fp32_alu_peak_tflops(1965.0) - 74.45) < 0.01
