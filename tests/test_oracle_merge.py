"""Pins of the oracle's split-key merge against the oracle's own full
attention: attention over a key axis cut into chunks, combined with
``oracle.merge``, must equal attention over the whole axis (no mask, causal
with an offset, a float mask with -inf entries, GQA), and a single part must
come back unchanged."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _chunks(n, cuts):
    edges = [0] + list(cuts) + [n]
    return [(a, b) for a, b in zip(edges[:-1], edges[1:])]


@pytest.mark.parametrize("case", ["none", "causal", "float_mask", "gqa"])
def test_merge_of_key_chunks_equals_full_attention(case):
    B, Hq, Hkv, Tq, Tkv, d = 2, 4, 4, 19, 37, 8
    if case == "gqa":
        Hkv = 2
    q, k, v = _rand((B, Hq, Tq, d), 1), _rand((B, Hkv, Tkv, d), 2), _rand((B, Hkv, Tkv, d), 3)
    kw, mask = {}, None
    if case == "causal":
        kw = dict(mask_kind=oracle.MASK_CAUSAL, offset=9)
    if case == "float_mask":
        mask = _rand((B, 1, Tq, Tkv), 4)
        mask[mask > 1.2] = -np.inf
        kw = dict(mask_kind=oracle.MASK_FLOAT)
    full = oracle.sdpa(q, k, v, 0.3, mask=mask, **kw)
    outs, lses = [], []
    for a, b in _chunks(Tkv, (5, 6, 20, 33)):
        ckw = dict(kw)
        if case == "causal":
            ckw["offset"] = kw["offset"] - a  # key j of the chunk is key a + j of the whole axis
        part = oracle.sdpa(q, k[:, :, a:b], v[:, :, a:b], 0.3,
                           mask=None if mask is None else mask[..., a:b].contiguous(), **ckw)
        outs.append(part.out)
        lses.append(part.lse)
    if case == "causal":
        assert np.isneginf(np.stack(lses)).any(), "some chunk must be fully masked for some row"
    out, lse = oracle.merge(outs, lses)
    fin = np.isfinite(full.lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.max(np.abs(out - full.out)) < 1e-12
    assert np.max(np.abs(lse[fin] - full.lse[fin])) < 1e-12


def test_merge_single_part_is_identity_and_empty_rows_are_zero():
    o = _rand((2, 3, 5, 4), 7).numpy()
    s = _rand((2, 3, 5), 8).numpy()
    out, lse = oracle.merge([o], [s])
    assert np.max(np.abs(out - o)) < 1e-15 and np.max(np.abs(lse - s)) < 1e-15
    s2 = np.full_like(s, -np.inf)
    out, lse = oracle.merge([o, o], [s2, s2])
    assert np.all(out == 0) and np.all(np.isneginf(lse))
