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


# head_dim-16 shapes on either side of the split-KV rule (Tkv >= 1024 and
# Tq <= Tkv / 16), as (B, H, Tq, Tkv) -> family
D16_RULE = [((4, 8, 8, 4096), "split_kv"), ((4, 8, 100, 8192), "split_kv"), ((4, 8, 64, 1024), "split_kv"),
            ((4, 8, 128, 2048), "split_kv"), ((4, 8, 129, 2048), "small_d"), ((4, 8, 128, 1024), "small_d"),
            ((4, 8, 8, 1023), "small_d"), ((4, 8, 4096, 8), "small_d"), ((4, 8, 512, 4096), "small_d")]


@pytest.mark.parametrize("shape,family", D16_RULE)
def test_auto_dispatch_head_dim_16(shape, family):
    import bench
    import torch
    from attention_sdpa_fwd_b200 import workloads as W
    B, H, Tq, Tkv = shape
    sp = W.Spec("d16_rule", torch.bfloat16, B, H, H, Tq, Tkv, 16, 0.25, seed=0)
    assert bench.auto_path_name(S, sp) == family


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_auto_dispatch_of_benchmark_workloads(name):
    import bench
    from attention_sdpa_fwd_b200 import workloads as W
    assert bench.auto_path_name(S, W.SPECS[name]) == EXPECTED[name]
