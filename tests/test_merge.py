"""GPU parity of sdpa_merge: element by element against the oracle's merge,
and end to end -- attention over a key axis cut into chunks (each chunk run
through the library with its lse output, on strided K/V views) and merged
must match the oracle's attention over the whole axis."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import attention_sdpa_fwd_b200 as S
import oracle
from attention_sdpa_fwd_b200 import workloads as W
from helpers import assert_gates, oracle_ref

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,d,n", [(torch.bfloat16, 64, 3), (torch.bfloat16, 16, 5), (torch.bfloat16, 128, 1),
                                       (torch.float32, 64, 4), (torch.float32, 16, 2)])
def test_merge_matches_oracle(dtype, d, n):
    g = torch.Generator().manual_seed(d * 10 + n)
    B, H, T = 2, 3, 77
    outs = [torch.randn(B, H, T, d, generator=g).to(dtype) for _ in range(n)]
    lses = [torch.randn(B, H, T, generator=g) * 3 for _ in range(n)]
    for i in range(n):
        lses[i][0, 0, i % T] = -math.inf            # a part without keys for some row
    for i in range(n):
        lses[i][1, 2, 5] = -math.inf                # a row without keys anywhere
    out, lse = S.merge([o.cuda() for o in outs], [x.cuda() for x in lses])
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.merge(outs, lses)
    got = out.cpu().double().numpy()
    if dtype == torch.float32:
        assert np.max(np.abs(got - ref_out)) < 1e-5
    else:
        assert np.max(np.abs(got - ref_out)) <= 2.0 ** -8 * np.max(np.abs(ref_out)) + 1e-6
    fin = np.isfinite(ref_lse)
    gl = lse.cpu().double().numpy()
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) < 1e-5
    assert torch.all(out[1, 2, 5] == 0)


def test_merge_in_place_equals_out_of_place():
    g = torch.Generator().manual_seed(5)
    outs = [torch.randn(1, 4, 300, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(3)]
    lses = [torch.randn(1, 4, 300, generator=g).cuda() for _ in range(3)]
    ref_o, ref_l = S.merge(outs, lses)
    o0, l0 = outs[0].clone(), lses[0].clone()
    S.merge([o0] + outs[1:], [l0] + lses[1:], out=o0, lse=l0)
    torch.cuda.synchronize()
    assert torch.equal(o0, ref_o) and torch.equal(l0, ref_l)


CASES = [
    W.Spec("chunked_none_d64", torch.bfloat16, 2, 4, 2, 260, 1000, 64, scale=0.125, seed=80),
    W.Spec("chunked_causal_d128", torch.bfloat16, 1, 4, 4, 300, 300, 128, scale=1 / math.sqrt(128),
           mask_kind=W.MASK_CAUSAL, seed=81),
    W.Spec("chunked_d16_long_kv", torch.bfloat16, 2, 4, 4, 8, 3000, 16, scale=0.25, seed=82),
]


@pytest.mark.parametrize("sp", CASES, ids=[c.name for c in CASES])
def test_chunked_attention_merged_equals_full(sp):
    wl = W.make(sp)
    q, k, v = wl.q.cuda(), wl.k.cuda(), wl.v.cuda()
    edges = [0, sp.Tkv // 3, sp.Tkv // 3 + 17, sp.Tkv]
    outs, lses = [], []
    for a, b in zip(edges[:-1], edges[1:]):
        lse = torch.empty(sp.B, sp.Hq, sp.Tq, device="cuda")
        kw = {}
        if sp.mask_kind == W.MASK_CAUSAL:
            kw = dict(mask_kind=W.MASK_CAUSAL, offset=sp.offset - a)  # chunk key j is key a + j
        outs.append(S.sdpa(q, k[:, :, a:b], v[:, :, a:b], sp.scale, lse=lse, **kw))
        lses.append(lse)
    out, _ = S.merge(outs, lses)
    torch.cuda.synchronize()
    ref = oracle_ref(wl)
    assert_gates(out.cpu().double().numpy(), ref.out, sp.dtype, sp.name)
