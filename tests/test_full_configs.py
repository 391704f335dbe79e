"""GPU parity at the benchmark workloads' full sizes, in the launch
configuration the benchmark times (the AUTO path): every output for the
smaller workloads, a deterministic row sample (edge, window-boundary and
tile-boundary rows included) for the large ones, where the oracle computes the
sampled rows exactly."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from attention_sdpa_fwd_b200 import workloads as W
from helpers import assert_gates, gpu_run, oracle_ref, sample_rows

pytestmark = pytest.mark.gpu

FULL = {"tiny_relpos_f32", "sam_windowed", "decoder_token_to_image", "decoder_image_to_token", "decoder_self"}
ALL = list(W.SPECS.values()) + list(W.STRONG_SPECS.values())


@pytest.mark.parametrize("sp", ALL, ids=[s.name for s in ALL])
def test_full_size(sp):
    wl = W.make(sp)
    out, _ = gpu_run(wl)
    if sp.name in FULL:
        ref = oracle_ref(wl)
        got = out.double().numpy()
    else:
        # 128 rows per (b, h) at T = 8192 (edge, window-boundary and tile-boundary rows included)
        n = 128 if sp.Tq >= 8192 else 256
        rows = sample_rows(sp.Tq, n, seed=sp.seed, must=(sp.window - 2, sp.window - 1, sp.window,
                                                          sp.window + 1) if sp.window else ())
        ref = oracle_ref(wl, rows=rows)
        got = out[:, :, rows].double().numpy()
    assert_gates(got, ref.out, sp.dtype, sp.name, strong=sp.name.endswith("_strong"))
