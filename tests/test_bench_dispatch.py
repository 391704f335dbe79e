"""Host-side (no GPU): the kernel family AUTO dispatches each benchmark
workload to, as bench.py reports it next to the per-workload timings."""
from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

S = pytest.importorskip("attention_sdpa_fwd_b200")

EXPECTED = {
    "tiny_relpos_f32": "exact",            # fp32 I/O
    "sam_global": "tcgen05",               # 16 query blocks x 12 heads < two per SM
    "sam_windowed": "tc_persistent",       # 1200 windows x heads of two key tiles each
    "decoder_token_to_image": "split_kv",  # 8 rows against 4096 keys, head_dim 16
    "decoder_image_to_token": "small_d",
    "decoder_self": "small_d",
    "gqa_causal": "tcgen05",
    "gqa_sliding": "tcgen05",
    "gqa_float_mask": "tcgen05",
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_auto_dispatch_of_benchmark_workloads(name):
    import bench
    from attention_sdpa_fwd_b200 import workloads as W
    assert bench.auto_path_name(S, W.SPECS[name]) == EXPECTED[name]
