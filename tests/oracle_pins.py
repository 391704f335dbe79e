"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Each ``pin_*`` takes a bound oracle library and raises AssertionError when the
oracle disagrees with: a worked example derived by hand (``golden/``), a closed
form, an invariant of softmax attention, a hand-enumerated index table, or an
independent library routine (torch's float64 scaled_dot_product_attention,
which is the mlx-examples issue's own proposal: the bias handed to a fused
SDPA as its additive mask).  ``test_oracle_pins.py`` runs them on the shipped
oracle; ``test_oracle_plants.py`` runs them on copies with planted mistakes and
checks each copy fails at least one pin.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle
from oracle import MASK_BOOL, MASK_CAUSAL, MASK_FLOAT, MASK_NONE, MASK_SLIDING

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _num(x):
    if isinstance(x, str):
        table = {"ln2": math.log(2.0), "ln3": math.log(3.0), "ln4": math.log(4.0),
                 "-ln2": -math.log(2.0), "2ln3": 2.0 * math.log(3.0), "-inf": -math.inf,
                 "ln(9/2)": math.log(4.5), "ln(7/2)": math.log(3.5)}
        if x in table:
            return table[x]
        num, den = x.split("/")  # an exact fraction "a/b"
        return float(num) / float(den)
    if isinstance(x, list):
        return [_num(y) for y in x]
    return float(x)


def _arr(x):
    return np.asarray(_num(x), dtype=np.float64)


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin), f"{what}: non-finite pattern differs"
    assert np.array_equal(a[~fin], b[~fin]), f"{what}: infinities differ"
    err = float(np.max(np.abs(a[fin] - b[fin]))) if fin.any() else 0.0
    assert err <= tol * max(1.0, float(np.max(np.abs(b[fin]))) if fin.any() else 1.0), \
        f"{what}: max |diff| {err:.3e} > {tol:.1e}"


def _rand_problem(seed, B=1, Hq=2, Hkv=1, Tq=6, Tkv=6, d=4, hw=(2, 3), rel=True, rel_std=0.7):
    r = _rng(seed)
    p = dict(q=r.standard_normal((B, Hq, Tq, d)), k=r.standard_normal((B, Hkv, Tkv, d)),
             v=r.standard_normal((B, Hkv, Tkv, d)))
    if rel:
        p["rel_pos_h"] = r.standard_normal((2 * hw[0] - 1, d)) * rel_std
        p["rel_pos_w"] = r.standard_normal((2 * hw[1] - 1, d)) * rel_std
        p["q_hw"] = hw
        p["k_hw"] = hw
    return p


def _bias_from_index_table(q, Rh, Rw):
    """Bias [B,H,6,6] of the 2x3 grid from the hand-enumerated index table."""
    rows = np.loadtxt(os.path.join(GOLDEN, "relpos_index_2x3.txt"), dtype=np.int64, comments="#")
    bias = np.zeros(q.shape[:2] + (6, 6))
    for i, j, ih, iw in rows:
        bias[:, :, i, j] = q[:, :, i, :] @ Rh[ih] + q[:, :, i, :] @ Rw[iw]
    return bias


def _bias_from_index_table_q2x3_k3x2(q, Rh, Rw):
    """Bias [B,H,6,6] of query grid 2x3 against key grid 3x2 from the
    hand-enumerated index table."""
    rows = np.loadtxt(os.path.join(GOLDEN, "relpos_index_q2x3_k3x2.txt"), dtype=np.int64, comments="#")
    bias = np.zeros(q.shape[:2] + (6, 6))
    for i, j, ih, iw in rows:
        bias[:, :, i, j] = q[:, :, i, :] @ Rh[ih] + q[:, :, i, :] @ Rw[iw]
    return bias


# ---------------------------------------------------------------------------
def pin_hand_cases(lib):
    """Worked examples whose outputs were derived by hand (golden/hand_cases.json)."""
    with open(os.path.join(GOLDEN, "hand_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        kw = dict(mask_kind=c.get("mask_kind", 0), offset=c.get("offset", 0), window=c.get("window", 0))
        if "mask" in c:
            m = _arr(c["mask"])
            kw["mask"] = m if c["mask_kind"] == MASK_FLOAT else m.astype(np.uint8)
        if "rel_pos_h" in c:
            kw.update(rel_pos_h=_arr(c["rel_pos_h"]), rel_pos_w=_arr(c["rel_pos_w"]),
                      q_hw=c["q_hw"], k_hw=c["k_hw"])
        r = oracle.sdpa(_arr(c["q"]), _arr(c["k"]), _arr(c["v"]), c["scale"], lib=lib, **kw)
        _close(r.out, _arr(c["out"]), 1e-12, c["name"] + " out")
        if "lse" in c:
            _close(r.lse, _arr(c["lse"]), 1e-12, c["name"] + " lse")


def pin_weights_sum_to_one(lib):
    """Every softmax row sums to 1 (and weights are non-negative)."""
    p = _rand_problem(1, Hq=2, Hkv=2)
    for kind, extra in [(MASK_NONE, {}), (MASK_CAUSAL, {"offset": 1}), (MASK_SLIDING, {"window": 3})]:
        r = oracle.sdpa(p["q"], p["k"], p["v"], 0.4, mask_kind=kind, want_weights=True, lib=lib,
                        rel_pos_h=p["rel_pos_h"], rel_pos_w=p["rel_pos_w"], q_hw=p["q_hw"], k_hw=p["k_hw"], **extra)
        s = r.weights.sum(-1)
        assert np.all(np.abs(s - 1.0) < 1e-12), f"mask {kind}: row sums {s}"
        assert np.all(r.weights >= 0.0)


def pin_zero_tables_equal_plain(lib):
    """Zero rel-pos tables reduce to plain SDPA."""
    p = _rand_problem(2)
    a = oracle.sdpa(p["q"], p["k"], p["v"], 0.3, rel_pos_h=np.zeros_like(p["rel_pos_h"]),
                    rel_pos_w=np.zeros_like(p["rel_pos_w"]), q_hw=p["q_hw"], k_hw=p["k_hw"], lib=lib)
    b = oracle.sdpa(p["q"], p["k"], p["v"], 0.3, lib=lib)
    _close(a.out, b.out, 1e-13, "zero tables")


def pin_row_constant_bias_shift(lib):
    """A per-row constant added to every score leaves the output unchanged: a
    constant float mask, and the same vector u added to every row of Rh (which
    adds q_i.u to row i's scores)."""
    p = _rand_problem(3, Hq=2, Hkv=2)
    base = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, rel_pos_h=p["rel_pos_h"], rel_pos_w=p["rel_pos_w"],
                       q_hw=p["q_hw"], k_hw=p["k_hw"], lib=lib)
    u = _rng(30).standard_normal(p["q"].shape[-1])
    shifted = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, rel_pos_h=p["rel_pos_h"] + u,
                          rel_pos_w=p["rel_pos_w"], q_hw=p["q_hw"], k_hw=p["k_hw"], lib=lib)
    _close(shifted.out, base.out, 1e-12, "Rh + u")
    shifted = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, rel_pos_h=p["rel_pos_h"],
                          rel_pos_w=p["rel_pos_w"] - 2.0 * u, q_hw=p["q_hw"], k_hw=p["k_hw"], lib=lib)
    _close(shifted.out, base.out, 1e-12, "Rw - 2u")
    m = _rng(31).standard_normal((1, 1, 6, 6))
    a = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, mask_kind=MASK_FLOAT, mask=m, lib=lib)
    b = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, mask_kind=MASK_FLOAT, mask=m + 3.25, lib=lib)
    _close(a.out, b.out, 1e-12, "mask + c")


def pin_constant_values(lib):
    """V constant over the keys returns that constant, with any bias or mask."""
    p = _rand_problem(4)
    c = np.array([1.5, -2.0, 0.25, 7.0])
    v = np.broadcast_to(c, p["v"].shape).copy()
    r = oracle.sdpa(p["q"], p["k"], v, 0.9, rel_pos_h=p["rel_pos_h"], rel_pos_w=p["rel_pos_w"],
                    q_hw=p["q_hw"], k_hw=p["k_hw"], mask_kind=MASK_SLIDING, window=2, lib=lib)
    _close(r.out, np.broadcast_to(c, r.out.shape), 1e-13, "constant V")


def pin_masked_key_inert(lib):
    """A key masked out for every row has weight exactly 0; changing its K/V
    changes nothing."""
    p = _rand_problem(5, rel=False, Hq=2, Hkv=2)
    keep = np.ones((1, 1, 6, 6), dtype=np.uint8)
    keep[..., 4] = 0
    a = oracle.sdpa(p["q"], p["k"], p["v"], 0.6, mask_kind=MASK_BOOL, mask=keep, want_weights=True, lib=lib)
    assert np.all(a.weights[..., 4] == 0.0)
    k2, v2 = p["k"].copy(), p["v"].copy()
    k2[:, :, 4] = 100.0
    v2[:, :, 4] = -1e6
    b = oracle.sdpa(p["q"], k2, v2, 0.6, mask_kind=MASK_BOOL, mask=keep, lib=lib)
    _close(b.out, a.out, 0.0, "masked key changed")
    fm = np.where(keep == 1, 0.0, -np.inf)
    c = oracle.sdpa(p["q"], p["k"], p["v"], 0.6, mask_kind=MASK_FLOAT, mask=fm, lib=lib)
    _close(c.out, a.out, 1e-14, "bool == float {0,-inf}")


def pin_index_table_2x3(lib):
    """The rel-pos bias matches the hand-enumerated index table of a 2x3 grid,
    through torch's float64 SDPA given the bias as its additive mask."""
    p = _rand_problem(6, Hq=3, Hkv=3, d=3)
    bias = _bias_from_index_table(p["q"], p["rel_pos_h"], p["rel_pos_w"])
    r = oracle.sdpa(p["q"], p["k"], p["v"], 0.45, rel_pos_h=p["rel_pos_h"], rel_pos_w=p["rel_pos_w"],
                    q_hw=(2, 3), k_hw=(2, 3), lib=lib)
    t = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(p["q"]), torch.from_numpy(p["k"]), torch.from_numpy(p["v"]),
        attn_mask=torch.from_numpy(bias), scale=0.45)
    _close(r.out, t.numpy(), 1e-12, "2x3 index table")


def pin_index_table_q2x3_k3x2(lib):
    """Query and key grids of their own (2x3 against 3x2): the rel-pos bias
    matches the hand-enumerated index table, through torch's float64 SDPA
    given the bias as its additive mask."""
    r = _rng(16)
    q, k, v = (r.standard_normal((1, 2, 6, 3)) for _ in range(3))
    Rh = r.standard_normal((4, 3)) * 0.8
    Rw = r.standard_normal((4, 3)) * 0.8
    bias = _bias_from_index_table_q2x3_k3x2(q, Rh, Rw)
    res = oracle.sdpa(q, k, v, 0.45, rel_pos_h=Rh, rel_pos_w=Rw, q_hw=(2, 3), k_hw=(3, 2), lib=lib)
    t = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=torch.from_numpy(bias),
        scale=0.45)
    _close(res.out, t.numpy(), 1e-12, "query 2x3 / key 3x2 index table")


def pin_unequal_grids_factorise(lib):
    """With K = 0 and query / key grids of their own (3x4 queries, 5x2 keys)
    the scores are rel_h[i, kh] + rel_w[i, kw], so each row of weights, viewed
    as a Kh x Kw matrix, has rank 1 and equals the outer product of its two
    marginals (the index itself is pinned by the hand-enumerated table and the
    worked example)."""
    r = _rng(17)
    Qh, Qw, Kh, Kw, d = 3, 4, 5, 2, 3
    q = r.standard_normal((1, 2, Qh * Qw, d))
    k = np.zeros((1, 2, Kh * Kw, d))
    v = r.standard_normal((1, 2, Kh * Kw, d))
    Rh = r.standard_normal((Qh + Kh - 1, d))
    Rw = r.standard_normal((Qw + Kw - 1, d))
    res = oracle.sdpa(q, k, v, 0.3, rel_pos_h=Rh, rel_pos_w=Rw, q_hw=(Qh, Qw), k_hw=(Kh, Kw),
                      want_weights=True, lib=lib)
    W = res.weights.reshape(1, 2, Qh * Qw, Kh, Kw)
    sv = np.linalg.svd(W, compute_uv=False)
    assert np.all(sv[..., 1] < 1e-12 * sv[..., 0]), "weights not rank-1 over (kh, kw)"
    _close(np.einsum("...a,...b->...ab", W.sum(-1), W.sum(-2)), W, 1e-12, "outer product of marginals")


def pin_factorisation(lib):
    """With K = 0 the scores are rel_h[i,kh] + rel_w[i,kw], so each row of
    weights, viewed as a Kh x Kw matrix, is an outer product (rank 1) of two
    softmaxes."""
    r = _rng(7)
    hw = (4, 5)
    q = r.standard_normal((1, 2, 20, 3))
    k = np.zeros((1, 2, 20, 3))
    v = r.standard_normal((1, 2, 20, 3))
    Rh = r.standard_normal((7, 3))
    Rw = r.standard_normal((9, 3))
    res = oracle.sdpa(q, k, v, 0.3, rel_pos_h=Rh, rel_pos_w=Rw, q_hw=hw, k_hw=hw, want_weights=True, lib=lib)
    W = res.weights.reshape(1, 2, 20, 4, 5)
    sv = np.linalg.svd(W, compute_uv=False)
    assert np.all(sv[..., 1] < 1e-12 * sv[..., 0]), "weights not rank-1 over (kh, kw)"
    # and the height marginal of row i depends only on q_i and the query's grid row
    Ph = W.sum(-1)
    Pw = W.sum(-2)
    _close(np.einsum("...a,...b->...ab", Ph, Pw), W, 1e-12, "outer product of marginals")


def pin_key_permutation(lib):
    """Without a bias, permuting keys and values together leaves the output unchanged."""
    p = _rand_problem(8, rel=False, Tkv=9)
    perm = _rng(80).permutation(9)
    a = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, lib=lib)
    b = oracle.sdpa(p["q"], p["k"][:, :, perm], p["v"][:, :, perm], 0.5, lib=lib)
    _close(a.out, b.out, 1e-13, "key permutation")


def pin_gqa_repeat(lib):
    """GQA equals plain attention on K/V heads repeated consecutively (Axon:
    repeating key/value heads to match the query)."""
    p = _rand_problem(9, Hq=6, Hkv=2, rel=False)
    a = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, mask_kind=MASK_CAUSAL, lib=lib)
    kr = np.repeat(p["k"], 3, axis=1)
    vr = np.repeat(p["v"], 3, axis=1)
    b = oracle.sdpa(p["q"], kr, vr, 0.5, mask_kind=MASK_CAUSAL, lib=lib)
    _close(a.out, b.out, 0.0, "gqa == repeat")
    t = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(p["q"]), torch.from_numpy(p["k"]), torch.from_numpy(p["v"]),
        is_causal=True, scale=0.5, enable_gqa=True)
    _close(a.out, t.numpy(), 1e-12, "gqa vs torch")


def pin_window_special_cases(lib):
    """w = 1 gives out[i] = v[i]; w >= T equals causal; rows past w-1 see exactly w keys."""
    p = _rand_problem(10, rel=False, Tq=8, Tkv=8)
    a = oracle.sdpa(p["q"], p["k"], p["v"], 0.7, mask_kind=MASK_SLIDING, window=1, lib=lib)
    _close(a.out, np.repeat(p["v"], 2, axis=1), 1e-14, "w = 1")
    b = oracle.sdpa(p["q"], p["k"], p["v"], 0.7, mask_kind=MASK_SLIDING, window=8, lib=lib)
    c = oracle.sdpa(p["q"], p["k"], p["v"], 0.7, mask_kind=MASK_CAUSAL, lib=lib)
    _close(b.out, c.out, 0.0, "w >= T == causal")
    w = oracle.sdpa(p["q"], p["k"], p["v"], 0.7, mask_kind=MASK_SLIDING, window=3, want_weights=True, lib=lib)
    nz = (w.weights > 0).sum(-1)
    assert np.all(nz[..., 2:] == 3) and np.all(nz[..., :2] == np.array([1, 2])), nz


def pin_float_and_bool_neutral(lib):
    """An all-zero float mask and an all-true boolean mask equal no mask."""
    p = _rand_problem(11, rel=False)
    a = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, lib=lib)
    b = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, mask_kind=MASK_FLOAT, mask=np.zeros((6, 6)), lib=lib)
    c = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, mask_kind=MASK_BOOL, mask=np.ones((6, 6), np.uint8), lib=lib)
    _close(b.out, a.out, 0.0, "zero float mask")
    _close(c.out, a.out, 0.0, "all-true bool mask")


def pin_torch_library_masks(lib):
    """torch float64 SDPA with the mask materialised (the mlx issue's proposal)
    agrees for float masks broadcast over heads and per batch, bool masks,
    causal and sliding masks with an offset."""
    r = _rng(12)
    B, Hq, Hkv, Tq, Tkv, d = 2, 4, 2, 5, 7, 4
    q = r.standard_normal((B, Hq, Tq, d))
    k = r.standard_normal((B, Hkv, Tkv, d))
    v = r.standard_normal((B, Hkv, Tkv, d))
    fm = r.standard_normal((B, 1, Tq, Tkv))
    fm[r.random(fm.shape) < 0.2] = -np.inf
    fm[..., 0] = 0.5  # every row keeps key 0
    bm = (r.random((B, Hq, Tq, Tkv)) < 0.6).astype(np.uint8)
    bm[..., 3] = 1
    ii = np.arange(Tq)[:, None]
    jj = np.arange(Tkv)[None, :]
    causal2 = np.where(jj <= ii + 2, 0.0, -np.inf)
    slide = np.where((jj <= ii + 1) & (jj > ii + 1 - 3), 0.0, -np.inf)
    T = lambda x: torch.from_numpy(np.array(x, copy=True))
    cases = [
        (dict(mask_kind=MASK_FLOAT, mask=fm), fm),
        (dict(mask_kind=MASK_BOOL, mask=bm), np.where(bm == 1, 0.0, -np.inf)),
        (dict(mask_kind=MASK_CAUSAL, offset=2), causal2),
        (dict(mask_kind=MASK_SLIDING, window=3, offset=1), slide),
    ]
    for kw, dense in cases:
        a = oracle.sdpa(q, k, v, 0.37, lib=lib, **kw)
        t = torch.nn.functional.scaled_dot_product_attention(
            T(q), T(k), T(v), attn_mask=T(np.broadcast_to(dense, (B, Hq, Tq, Tkv))), scale=0.37, enable_gqa=True)
        _close(a.out, t.numpy(), 1e-12, f"torch mask {kw['mask_kind']}")


def pin_lse_closed_form(lib):
    """q = 0 gives lse = log(#visible keys) and out = mean of the visible values."""
    r = _rng(13)
    k = r.standard_normal((1, 1, 5, 2))
    v = r.standard_normal((1, 1, 5, 2))
    q = np.zeros((1, 1, 5, 2))
    a = oracle.sdpa(q, k, v, 1.0, mask_kind=MASK_CAUSAL, lib=lib)
    _close(a.lse, np.log(np.arange(1, 6, dtype=np.float64))[None, None], 1e-14, "lse")
    want = np.cumsum(v[0, 0], axis=0) / np.arange(1, 6)[:, None]
    _close(a.out[0, 0], want, 1e-14, "prefix means")


def pin_rows_subset(lib):
    """Computing a subset of rows gives exactly those rows of the full result."""
    p = _rand_problem(14)
    full = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, rel_pos_h=p["rel_pos_h"], rel_pos_w=p["rel_pos_w"],
                       q_hw=p["q_hw"], k_hw=p["k_hw"], lib=lib)
    rows = [5, 0, 3]
    sub = oracle.sdpa(p["q"], p["k"], p["v"], 0.5, rel_pos_h=p["rel_pos_h"], rel_pos_w=p["rel_pos_w"],
                      q_hw=p["q_hw"], k_hw=p["k_hw"], rows=rows, lib=lib)
    _close(sub.out, full.out[:, :, rows], 0.0, "row subset")


ALL_PINS = [pin_hand_cases, pin_weights_sum_to_one, pin_zero_tables_equal_plain,
            pin_row_constant_bias_shift, pin_constant_values, pin_masked_key_inert,
            pin_index_table_2x3, pin_index_table_q2x3_k3x2, pin_unequal_grids_factorise, pin_factorisation, pin_key_permutation, pin_gqa_repeat,
            pin_window_special_cases, pin_float_and_bool_neutral, pin_torch_library_masks,
            pin_lse_closed_form, pin_rows_subset]
