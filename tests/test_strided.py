"""GPU parity for strided tensors (sdpa_fwd_strided): the "bshd" layout
[B, T, H, d] that the Axon PR takes by default, used in place through
transposed views, on every path; plus row strides that the TMA / 16-byte
paths cannot take, which AUTO must route to the exact kernel."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import attention_sdpa_fwd_b200 as S
from attention_sdpa_fwd_b200 import workloads as W
from helpers import assert_gates, oracle_ref

pytestmark = pytest.mark.gpu

F32, BF16 = torch.float32, torch.bfloat16


def S_(name, dtype, B, Hq, Hkv, Tq, Tkv, d, **kw):
    kw.setdefault("scale", 1.0 / math.sqrt(d))
    return W.Spec(name, dtype, B, Hq, Hkv, Tq, Tkv, d, **kw)


CASES = [
    ("tcgen05", S_("bshd_relpos_d64_12x16", BF16, 2, 3, 3, 192, 192, 64, q_hw=(12, 16), k_hw=(12, 16),
                   rel_std=0.5, seed=70)),
    ("tcgen05", S_("bshd_causal_gqa_d128", BF16, 1, 8, 2, 300, 300, 128, mask_kind=W.MASK_CAUSAL, seed=71)),
    ("tcgen05", S_("bshd_none_d64_ragged", BF16, 2, 4, 2, 333, 260, 64, seed=72)),
    ("small_d", S_("bshd_d16_rows", BF16, 2, 4, 2, 300, 40, 16, seed=73)),
    ("split_kv", S_("bshd_d16_long_kv", BF16, 2, 4, 4, 8, 1500, 16, seed=74)),
    ("exact", S_("bshd_f32_relpos_d16", F32, 1, 2, 2, 64, 64, 16, scale=0.25, q_hw=(8, 8), k_hw=(8, 8),
                 rel_std=0.5, seed=75)),
    ("exact", S_("bshd_bf16_float_mask_d64", BF16, 1, 2, 1, 130, 150, 64, mask_kind=W.MASK_FLOAT, mask_std=1.0,
                 mask_neg_inf_frac=0.2, mask_heads=2, seed=76)),
]


def bshd(x):
    """A [B, T, H, d]-contiguous copy of the bhsd tensor x, returned as its
    [B, H, T, d] view (strides {T*H*d, d, H*d, 1})."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


def run(wl, path, out_bshd):
    sp = wl.spec
    dv = lambda x: None if x is None else x.cuda()
    q, k, v = (bshd(dv(t)) for t in (wl.q, wl.k, wl.v))
    assert not q.is_contiguous() and q.stride(3) == 1
    out = bshd(torch.zeros_like(dv(wl.q))) if out_bshd else None
    res = S.sdpa(q, k, v, sp.scale, mask_kind=sp.mask_kind, offset=sp.offset, window=sp.window,
                 mask=dv(wl.mask), rel_pos_h=dv(wl.rel_pos_h), rel_pos_w=dv(wl.rel_pos_w), q_hw=sp.q_hw,
                 k_hw=sp.k_hw, out=out, path=path)
    torch.cuda.synchronize()
    return res


@pytest.mark.parametrize("path,sp", CASES, ids=[c[1].name for c in CASES])
@pytest.mark.parametrize("out_bshd", [False, True], ids=["out_bhsd", "out_bshd"])
def test_bshd_parity(path, sp, out_bshd):
    wl = W.make(sp)
    res = run(wl, path, out_bshd)
    ref = oracle_ref(wl)
    assert_gates(res.cpu().double().numpy(), ref.out, sp.dtype, f"{sp.name}/{path}")
    # same bytes as the dense call on the same path
    dense = S.sdpa(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), sp.scale, mask_kind=sp.mask_kind, offset=sp.offset,
                   window=sp.window, mask=None if wl.mask is None else wl.mask.cuda(),
                   rel_pos_h=None if wl.rel_pos_h is None else wl.rel_pos_h.cuda(),
                   rel_pos_w=None if wl.rel_pos_w is None else wl.rel_pos_w.cuda(), q_hw=sp.q_hw,
                   k_hw=sp.k_hw, path=path)
    torch.cuda.synchronize()
    assert torch.equal(res.contiguous(), dense)


def test_unaligned_row_stride_goes_to_exact():
    """A token stride of 68 elements (136 bytes) is no multiple of 16 bytes:
    the tensor-core path refuses it (MISALIGNED), AUTO still computes it."""
    sp = S_("padded_rows_d64", BF16, 1, 1, 1, 200, 180, 64, seed=77)
    wl = W.make(sp)

    def padded(x):
        B, H, T, d = x.shape
        buf = torch.zeros(B, H, T, d + 4, dtype=x.dtype, device="cuda")
        buf[..., :d] = x.cuda()
        return buf[..., :d]

    q, k, v = padded(wl.q), padded(wl.k), padded(wl.v)
    assert q.stride(2) == 68
    with pytest.raises(S.SdpaError) as e:
        S.sdpa(q, k, v, sp.scale, path="tcgen05")
    assert e.value.status == -3
    assert S.sdpa_select_path  # the binding exposes the selector too
    res = S.sdpa(q, k, v, sp.scale)
    torch.cuda.synchronize()
    ref = oracle_ref(wl)
    assert_gates(res.cpu().double().numpy(), ref.out, sp.dtype, sp.name)
