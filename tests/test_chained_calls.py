"""Consecutive calls on one stream that depend on each other.

The tensor-core and persistent kernels are launched with programmatic stream
serialization: a grid's CTAs may be scheduled while the previous grid in the
stream still runs, and wait for its completion before they touch global
memory.  These tests enqueue dependent calls back to back with no host
synchronisation between them, on shapes of several waves (so that CTAs of the
second grid do start while the first one runs), and check each result
against the fp64 oracle on sampled rows:

* read after write: the second call's queries are the first call's output;
* write after read: a call writes its output over the previous call's
  queries;
* both calls share the split-KV workspace (the SAM global shape at batch 1
  splits its last wave's key ranges), so a second grid that wrote its
  partials early would corrupt the first one's merge.
"""
import numpy as np
import pytest
import torch

import oracle
from attention_sdpa_fwd_b200 import workloads as W
from helpers import assert_gates

pytestmark = pytest.mark.gpu


def _rows(Tq, n=40):
    return sorted(set(list(range(0, Tq, max(1, Tq // n))) + [Tq - 1]))


def _ref(sp, q, k, v, rh, rw, rows):
    kw = dict(rows=rows)
    if sp.rel:
        kw.update(rel_pos_h=rh.cpu(), rel_pos_w=rw.cpu(), q_hw=sp.q_hw, k_hw=sp.k_hw)
    return oracle.sdpa(q.cpu(), k.cpu(), v.cpu(), sp.scale, **kw).out


def _call(S, sp, q, k, v, rh, rw, out):
    kw = dict(out=out)
    if sp.rel:
        kw.update(rel_pos_h=rh, rel_pos_w=rw, q_hw=sp.q_hw, k_hw=sp.k_hw)
    return S.sdpa(q, k, v, sp.scale, **kw)


CASES = [
    # name, spec, batch subset kept for the oracle
    ("sam_global", W.SPECS["sam_global"], 1),
    ("sam_windowed", W.scaled(W.SPECS["sam_windowed"], B=48), 2),
    ("gqa_d128_no_mask", W.Spec("gqa_d128_no_mask", torch.bfloat16, 2, 16, 4, 2048, 2048, 128, 128 ** -0.5,
                                seed=5), 1),
]


@pytest.mark.parametrize("name,sp,nb", CASES, ids=[c[0] for c in CASES])
def test_read_after_write_and_write_after_read(name, sp, nb):
    import attention_sdpa_fwd_b200 as S
    wl = W.make(sp, seed=sp.seed + 31)
    dev = lambda x: None if x is None else x.cuda().contiguous()
    q, k, v, rh, rw = dev(wl.q), dev(wl.k), dev(wl.v), dev(wl.rel_pos_h), dev(wl.rel_pos_w)
    q2 = dev(W.make(sp, seed=sp.seed + 32).q)
    q_orig = q.clone()
    x, y, z = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    torch.cuda.synchronize()
    # read after write: x = attn(q), then y = attn(x), no sync in between
    _call(S, sp, q, k, v, rh, rw, x)
    _call(S, sp, x, k, v, rh, rw, y)
    torch.cuda.synchronize()
    # write after read: z = attn(q), then q = attn(q2) over the queries the
    # previous grid reads, no sync in between
    _call(S, sp, q, k, v, rh, rw, z)
    _call(S, sp, q2, k, v, rh, rw, q)
    torch.cuda.synchronize()
    assert S.sdpa_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
    rows = _rows(sp.Tq)
    sl = slice(0, nb)
    got = lambda t: t[sl][:, :, rows].double().cpu().numpy()
    ref_x = _ref(sp, q_orig[sl], k[sl], v[sl], rh, rw, rows)
    assert_gates(got(x), ref_x, sp.dtype, f"{name}: first call")
    assert_gates(got(y), _ref(sp, x[sl], k[sl], v[sl], rh, rw, rows), sp.dtype,
                 f"{name}: call reading the previous call's output")
    assert_gates(got(z), ref_x, sp.dtype, f"{name}: call whose queries the next call overwrites")
    assert_gates(got(q), _ref(sp, q2[sl], k[sl], v[sl], rh, rw, rows), sp.dtype,
                 f"{name}: call writing over the previous call's queries")
