"""Negative controls of the GPU gates: results that are wrong in ways a
kernel could plausibly be wrong must FAIL the gates against the true oracle,
while the kernel's correct result passes them on the same inputs.  Every wrong
result is the kernel's own output on deliberately mis-arranged inputs, so the
gates are shown to reject the mistakes at the sizes and value distributions
of the stated workloads:

  * an all-zero output;
  * rel_h and rel_w swapped (the tables handed over the other way round);
  * the patch grid read transposed (heights and widths exchanged);
  * GQA kv heads tiled (head h reads kv head h % Hkv) instead of repeated
    consecutively (h / (Hq/Hkv)).

The bias is the decomposed rel-pos term of the SAM image encoder's attention
(mlx-examples issue "segment_anything: fuse attention ..."); GQA repeats
key/value heads to match the query heads (Axon PR "Add
scaled_dot_product_attention", GQA item)."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from attention_sdpa_fwd_b200 import workloads as W
from helpers import GATES, assert_gates, oracle_ref, passes, stats

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16
# the SAM global attention distribution at a reduced size: q, k, v ~ N(0, 1/2),
# tables N(0, 0.02^2), scale 1/8, head_dim 64
SQUARE = W.Spec("negctl_square_32x32", BF16, 1, 4, 4, 1024, 1024, 64, 0.125, seed=90,
                qkv_std=1.0 / math.sqrt(2.0), q_hw=(32, 32), k_hw=(32, 32), rel_std=0.02)
OBLONG = W.Spec("negctl_oblong_16x64", BF16, 1, 4, 4, 1024, 1024, 64, 0.125, seed=91,
                qkv_std=1.0 / math.sqrt(2.0), q_hw=(16, 64), k_hw=(16, 64), rel_std=0.02)
GQA = W.Spec("negctl_gqa", BF16, 2, 8, 2, 512, 512, 128, 1.0 / math.sqrt(128.0), seed=92,
             mask_kind=W.MASK_CAUSAL)


def _run(sp, q, k, v, rh=None, rw=None, q_hw=None, k_hw=None):
    import attention_sdpa_fwd_b200 as S
    out = S.sdpa(q.cuda(), k.cuda(), v.cuda(), sp.scale, mask_kind=sp.mask_kind, offset=sp.offset,
                 window=sp.window, rel_pos_h=None if rh is None else rh.cuda(),
                 rel_pos_w=None if rw is None else rw.cuda(), q_hw=q_hw, k_hw=k_hw)
    torch.cuda.synchronize()
    assert S.sdpa_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    return out.cpu().double().numpy()


def _must_fail(got, ref, what):
    s = stats(got, ref)
    assert not passes(s, BF16), f"{what} passes the gates {GATES[BF16]}: {s}"


def test_zero_output_fails():
    wl = W.make(SQUARE)
    ref = oracle_ref(wl).out
    _must_fail(np.zeros_like(ref), ref, "all-zero output")


def test_swapped_rel_tables_fail():
    sp = SQUARE
    wl = W.make(sp)
    ref = oracle_ref(wl).out
    good = _run(sp, wl.q, wl.k, wl.v, wl.rel_pos_h, wl.rel_pos_w, sp.q_hw, sp.k_hw)
    assert_gates(good, ref, BF16, "correct tables")
    bad = _run(sp, wl.q, wl.k, wl.v, wl.rel_pos_w, wl.rel_pos_h, sp.q_hw, sp.k_hw)
    _must_fail(bad, ref, "rel_h / rel_w swapped")


def test_transposed_grid_fails():
    sp = OBLONG
    wl = W.make(sp)
    ref = oracle_ref(wl).out
    good = _run(sp, wl.q, wl.k, wl.v, wl.rel_pos_h, wl.rel_pos_w, sp.q_hw, sp.k_hw)
    assert_gates(good, ref, BF16, "correct grid")
    # the same tokens read as a 64 x 16 grid (tables exchanged so their sizes fit it)
    tq, tk = sp.q_hw[::-1], sp.k_hw[::-1]
    bad = _run(sp, wl.q, wl.k, wl.v, wl.rel_pos_w, wl.rel_pos_h, tq, tk)
    _must_fail(bad, ref, "patch grid transposed")


def test_tiled_gqa_fails():
    sp = GQA
    wl = W.make(sp)
    ref = oracle_ref(wl).out
    good = _run(sp, wl.q, wl.k, wl.v)
    assert_gates(good, ref, BF16, "consecutive repetition")
    # permute the query heads so that the kernel's consecutive mapping reads kv
    # head h % Hkv for original head h, then put the heads back in order
    g = sp.Hq // sp.Hkv
    perm = [a * sp.Hkv + r for r in range(sp.Hkv) for a in range(g)]  # new head r*g + a <- original a*Hkv + r
    inv = np.argsort(perm)
    bad = _run(sp, wl.q[:, perm], wl.k, wl.v)[:, inv]
    for h in range(sp.Hq):  # the permutation really emulates h -> h % Hkv
        assert perm[inv[h]] == h and inv[h] // g == h % sp.Hkv
    _must_fail(bad, ref, "GQA kv heads tiled")
