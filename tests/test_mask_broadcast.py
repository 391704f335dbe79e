"""GPU parity of mask tensors broadcast over the batch and over the heads
([1, 1, Tq, Tkv], [1, Hq, Tq, Tkv], [B, 1, Tq, Tkv]: a size-1 axis has stride
0), on every kernel family that takes the problem: at head_dim 128 with 16-byte
mask rows the tensor-core kernel brings the mask tiles in by TMA, whose map
then has extent-1 head / batch axes; other key counts take the per-row loads.
Float and bool masks, against the fp64 oracle given the same broadcast mask."""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

from attention_sdpa_fwd_b200 import workloads as W
from helpers import assert_gates, oracle_ref
from test_parity import PATHS, applicable

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16

# (name, B, Hq, Hkv, Tq, Tkv, d, mask kind, broadcast over batch, broadcast over heads)
CASES = [
    ("float_tma_bcast_batch_heads", 3, 4, 2, 200, 320, 128, W.MASK_FLOAT, True, True),
    ("float_tma_bcast_batch", 2, 4, 4, 150, 200, 128, W.MASK_FLOAT, True, False),
    ("bool_tma_bcast_batch_heads", 2, 2, 1, 130, 272, 128, W.MASK_BOOL, True, True),
    ("float_rows_bcast_batch", 2, 2, 2, 100, 301, 128, W.MASK_FLOAT, True, False),
    ("float_d64_bcast_batch_heads", 2, 4, 2, 260, 256, 64, W.MASK_FLOAT, True, True),
    ("bool_d16_bcast_batch", 3, 2, 2, 40, 96, 16, W.MASK_BOOL, True, False),
]


def _spec(seed, name, B, Hq, Hkv, Tq, Tkv, d, mk, bb, bh):
    return W.Spec(name, BF16, B, Hq, Hkv, Tq, Tkv, d, 1.0 / np.sqrt(d), seed=seed,
                  mask_kind=mk, mask_std=1.0, mask_neg_inf_frac=0.3 if mk == W.MASK_BOOL else 0.15,
                  mask_heads=1 if bh else Hq)


@pytest.mark.parametrize("i", range(len(CASES)), ids=[c[0] for c in CASES])
def test_broadcast_mask(i):
    import attention_sdpa_fwd_b200 as S
    case = CASES[i]
    name, B, Hq, Hkv, Tq, Tkv, d, mk, bb, bh = case
    sp = _spec(300 + i, *case)
    wl = W.make(sp)
    mask = wl.mask[:1].contiguous() if bb else wl.mask  # [1, Hm, Tq, Tkv]: one mask for every batch
    wl = dataclasses.replace(wl, mask=mask)
    ref = oracle_ref(wl)
    dev = lambda x: None if x is None else x.cuda()
    for path in ["auto"] + [p for p in PATHS if applicable(p, sp)]:
        out = S.sdpa(dev(wl.q), dev(wl.k), dev(wl.v), sp.scale, mask_kind=mk, mask=dev(mask), path=path)
        torch.cuda.synchronize()
        assert S.sdpa_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
        assert_gates(out.double().cpu().numpy(), ref.out, BF16, f"{name}/{path}")
