"""The gates can tell a missing bias apart: for every workload with a bias or
mask, the oracle with the bias removed must FAIL the gates against the true
oracle (otherwise a kernel that ignores the bias would pass).  Oracle only,
on a row sample; no GPU."""
from __future__ import annotations

import pytest

from attention_sdpa_fwd_b200 import workloads as W
from helpers import oracle_ref, passes, sample_rows, stats

BIASED = [s for s in list(W.SPECS.values()) + list(W.STRONG_SPECS.values())
          if s.rel or s.mask_kind != W.MASK_NONE]


@pytest.mark.parametrize("sp", BIASED, ids=[s.name for s in BIASED])
def test_dropping_bias_fails_gates(sp):
    if sp.Tq * sp.Tkv * sp.B * sp.Hq > 4096 * 4096 * 12:
        # the large GQA workloads: two batches x a few heads are enough to decide
        sp = W.scaled(sp, B=1, Hq=4, Hkv=1)
    if sp.B > 8:
        sp = W.scaled(sp, B=4)
    wl = W.make(sp)
    rows = sample_rows(sp.Tq, 32, seed=1) if sp.Tq > 256 else None
    true = oracle_ref(wl, rows=rows)
    nob = oracle_ref(wl, rows=rows, drop_bias=True)
    s = stats(nob.out, true.out)
    assert not passes(s, sp.dtype), f"{sp.name}: bias undiscriminated by the gates {s}"
