"""Shared test helpers: the numeric gates and GPU / oracle runners.

Gates (the fused SDPA's own tolerance statement: max |diff| <= 1e-4 for fp32
I/O; max |diff| <= 2e-2 and mean |diff| <= 4e-3 for bf16 I/O with fp32
accumulation), plus a relative-L2 gate (1e-5 fp32, 1e-2 bf16) because the
absolute bf16 gates alone would accept an output with the bias left out.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

import oracle
from attention_sdpa_fwd_b200 import workloads as W

GATES = {
    torch.float32: dict(max_abs=1e-4, mean_abs=1e-4, rel_l2=1e-5),
    torch.bfloat16: dict(max_abs=2e-2, mean_abs=4e-3, rel_l2=1e-2),
}


def stats(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(got - ref)
    n = float(np.linalg.norm(ref))
    return dict(max_abs=float(diff.max()) if diff.size else 0.0,
                mean_abs=float(diff.mean()) if diff.size else 0.0,
                rel_l2=float(np.linalg.norm(got - ref) / n) if n > 0 else float(np.linalg.norm(got - ref)))


def passes(s: dict, dtype) -> bool:
    g = GATES[dtype]
    return all(s[k] <= g[k] for k in g)


def assert_gates(got, ref, dtype, what="", strong=False):
    """The stated gates.  ``strong`` (bias-dominated companions only, never the
    stated workloads) replaces the flat bf16 max gate by 2e-2 + 2^-7*|ref| per
    element: there the output sits on single value rows of magnitude up to ~5,
    where bf16 output rounding (unit roundoff 2^-8) is up to 2^-8*|ref| and the
    bf16 rounding of P adds at most another 2^-8*|ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    s = stats(got, ref)
    if strong and dtype == torch.bfloat16:
        bound = 2e-2 + 2.0 ** -7 * np.abs(ref)
        worst = float(np.max(np.abs(got - ref) - bound)) if got.size else 0.0
        assert worst <= 0.0, f"{what}: |diff| exceeds 2e-2 + 2^-7|ref| by {worst:.3e} ({s})"
        g = GATES[dtype]
        assert s["mean_abs"] <= g["mean_abs"] and s["rel_l2"] <= g["rel_l2"], f"{what}: {s} vs gates {g}"
        return s
    assert passes(s, dtype), f"{what}: {s} vs gates {GATES[dtype]}"
    return s


def oracle_ref(wl: W.Workload, rows: Optional[Sequence[int]] = None, drop_bias: bool = False):
    sp = wl.spec
    kw = dict(mask_kind=sp.mask_kind, offset=sp.offset, window=sp.window, rows=rows)
    if drop_bias:
        kw["mask_kind"] = W.MASK_NONE
    elif sp.mask_kind in (W.MASK_FLOAT, W.MASK_BOOL):
        kw["mask"] = wl.mask
    if sp.rel and not drop_bias:
        kw.update(rel_pos_h=wl.rel_pos_h, rel_pos_w=wl.rel_pos_w, q_hw=sp.q_hw, k_hw=sp.k_hw)
    return oracle.sdpa(wl.q, wl.k, wl.v, sp.scale, **kw)


def to_device(wl: W.Workload, device="cuda"):
    t = lambda x: None if x is None else x.to(device).contiguous()
    return dict(q=t(wl.q), k=t(wl.k), v=t(wl.v), rel_pos_h=t(wl.rel_pos_h), rel_pos_w=t(wl.rel_pos_w),
                mask=t(wl.mask))


def gpu_run(wl: W.Workload, path: str = "auto", want_lse: bool = False, dev=None):
    """Run the CUDA path through the C ABI; returns (out, lse) as CPU tensors."""
    import attention_sdpa_fwd_b200 as S
    sp = wl.spec
    dev = dev or to_device(wl)
    lse = torch.empty(sp.B, sp.Hq, sp.Tq, device="cuda", dtype=torch.float32) if want_lse else None
    out = S.sdpa(dev["q"], dev["k"], dev["v"], sp.scale, mask_kind=sp.mask_kind, offset=sp.offset,
                 window=sp.window, mask=dev["mask"], rel_pos_h=dev["rel_pos_h"], rel_pos_w=dev["rel_pos_w"],
                 q_hw=sp.q_hw, k_hw=sp.k_hw, lse=lse, path=path)
    torch.cuda.synchronize()
    rc = S.sdpa_last_device_error(torch.cuda.current_stream().cuda_stream)
    assert rc == 0, f"device error word: {S.STATUS.get(rc, rc)}"
    return out.cpu(), (lse.cpu() if lse is not None else None)


def sample_rows(Tq: int, n: int = 128, seed: int = 0, must=()) -> list:
    """Deterministic row sample that always holds the edge and tile-boundary rows."""
    base = {0, 1, Tq - 2, Tq - 1, 127, 128, 255, 256}
    base.update(must)
    base = {r for r in base if 0 <= r < Tq}
    rng = np.random.default_rng(seed)
    extra = rng.choice(Tq, size=min(Tq, max(0, n - len(base))), replace=False)
    return sorted(base.union(int(x) for x in extra))
