"""The roofline arithmetic bench.py reports, on the CPU.

The algorithmic bytes are K and V of every KV head for each visible key row
(visible prefix rows plus the S suffix rows), bf16: 4 KV heads x 2 x 256 x
2 B = 4096 B per row.  The FLOPs are QK^T plus PV, 2 flops per MAC:
4 * Hq * S * D per visible key.  The expected values below are counted
from the workload definitions, independently of bench.py.
"""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gqa_prefix_suffix_b200 import inputs as gen  # noqa: E402


@pytest.mark.parametrize("name,visible_prefix,S", [
    ("libero_tiny", 512, 10),     # P = 576, valid 512, no mask
    ("base_chunk", 900, 50),      # P = 1024, valid 900, no mask
])
def test_bytes_and_flops_of_the_single_sample_workloads(name, visible_prefix, S):
    inp = bench.workload_inputs(name)
    kv, flops = bench.algorithmic_bytes(inp)
    rows = visible_prefix + S
    assert kv == 4096 * rows
    assert flops == 4 * 8 * S * 256 * rows


def test_base_chunk_figures():
    kv, flops = bench.algorithmic_bytes(bench.workload_inputs("base_chunk"))
    assert kv == 3_891_200
    assert flops == 389_120_000


def test_history_loop_figures():
    kv, _ = bench.algorithmic_bytes(bench.workload_inputs("history_loop"))
    assert kv == 7_987_200        # 1900 visible rows + 50 suffix rows


def test_batched_counts_only_visible_rows():
    inp = gen.batched_mask()
    kv, flops = bench.algorithmic_bytes(inp)
    vis = 0
    for b in range(inp.B):
        vl = int(inp.prefix_valid_len[b])
        vis += int(torch.count_nonzero(inp.prefix_mask[b, :vl]))
    rows = vis + inp.B * inp.S
    assert kv == 4096 * rows
    assert flops == 4 * 8 * inp.S * 256 * rows
    # hidden rows inside the valid range are excluded: fewer bytes than the valid range
    valid_rows = int(inp.prefix_valid_len.sum()) + inp.B * inp.S
    assert kv < 4096 * valid_rows


def test_whole_bucket_without_valid_len():
    inp = gen.make_inputs(2, 8, 4, 128, 10, 256, 5, valid_len=None)
    kv, _ = bench.algorithmic_bytes(inp)
    assert kv == 4096 * 2 * (128 + 10)
