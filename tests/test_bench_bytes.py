"""The algorithmic bytes behind the bench's achieved GB/s (the roofline numerator), derived by
hand per call: packed sign bits N*K/8, the 4-byte tensor scale alpha, x bf16 (2 bytes, read once
per call), y fp32 (4 bytes per row)."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_bitnet_layer_fused_bytes(N, K):
    assert bench.layer_bytes("bitnet", N, K)["fused"] == N * K // 8 + 4 + 2 * K + 4 * N


def test_grouped_calls_read_x_once():
    # q, k, v: three 4096x4096 weight sets, three alphas, three y, one x
    assert bench.call_bytes([4096] * 3, 4096) == 3 * (4096 * 4096 // 8 + 4 + 4 * 4096) + 2 * 4096
    assert bench.call_bytes([4096], 4096) == bench.layer_bytes("bitnet", 4096, 4096)["fused"]


def test_decode_step_bytes_match_the_traffic_record():
    """Per call type, the numerator equals the algorithmic bytes stored beside the DRAM counters,
    and the 32-layer step totals about 816 MB (far above the 126 MB L2)."""
    shapes = {n: (N, K) for n, N, K in bench.LLAMA7B}
    per_call = {}
    for names in bench.LLAMA7B_CALLS:
        K = shapes[names[0]][1]
        assert all(shapes[n][1] == K for n in names)          # a group shares its input
        per_call[names] = bench.call_bytes([shapes[n][0] for n in names], K)
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))["bitnet_fused_llama7b_grouped"]
    stored = rec["per_call_algorithmic_bytes"]
    assert sorted(stored.values()) == sorted(per_call.values())
    step = 32 * sum(per_call.values())
    assert 815e6 < step < 817e6
    # the record's per-launch DRAM figure is the mean over the four call types
    assert rec["dram_bytes_per_launch"] == sum(rec["per_call_dram_bytes"].values()) / 4
