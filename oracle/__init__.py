"""Oracle for the fused SDPA forward -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU definition of ``softmax(Q.K^T*scale + bias).V`` (Axon PR
"Add scaled_dot_product_attention", description and :mask option; mlx-examples
issue "segment_anything: fuse attention with mx.fast.scaled_dot_product_attention",
SAM image-encoder attention with ``add_decomposed_rel_pos``; candle PR "SDPA
with Relative Positional Embeddings", term_h / term_w).  The arithmetic lives
in ``sdpa_oracle.c``; this module builds it with gcc, widens the inputs to
float64 and calls it.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package: the library under
``attention_sdpa_fwd_b200`` never does and shares no code with it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sdpa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_sdpa.so")
_lib = None

MASK_NONE, MASK_CAUSAL, MASK_SLIDING, MASK_FLOAT, MASK_BOOL = 0, 1, 2, 3, 4


def compile_oracle(out_path: str = _LIB_PATH, plant: int = 0) -> str:
    """Compile ``sdpa_oracle.c`` into a shared library (gcc, OpenMP, IEEE math).

    ``plant`` != 0 builds a deliberately wrong copy (used only by the test that
    checks the pins reject planted mistakes)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", out_path, _SRC, "-lm"]
    if plant:
        cmd.insert(1, f"-DORACLE_PLANT={int(plant)}")
    subprocess.run(cmd, check=True)
    return out_path


def _bind(path: str):
    lib = ctypes.CDLL(path)
    f = lib.oracle_sdpa_rows
    dp = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_longlong, ctypes.c_double
    f.argtypes = [dp, dp, dp, i32, i32, i32, i32, i32, i32, f64,
                  i32, i64, i64, dp, dp, i64, i64, i64,
                  dp, dp, i32, i32, i32, i32,
                  dp, i64, dp, dp, dp]
    f.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def load(path: Optional[str] = None):
    """Return the bound oracle library, compiling it on first use."""
    global _lib
    if path is not None:
        return _bind(path)
    if _lib is None:
        if (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
            compile_oracle()
        _lib = _bind(_LIB_PATH)
    return _lib


def num_threads() -> int:
    return int(load().oracle_num_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> numpy without importing torch here
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


@dataclass
class OracleResult:
    out: np.ndarray            # [B, Hq, rows, d] float64
    lse: np.ndarray            # [B, Hq, rows]    float64
    weights: Optional[np.ndarray] = None  # [B, Hq, rows, Tkv] when requested


def sdpa(q, k, v, scale: float, *, mask_kind: int = MASK_NONE, offset: int = 0,
         window: int = 0, mask=None, rel_pos_h=None, rel_pos_w=None,
         q_hw: Optional[Sequence[int]] = None, k_hw: Optional[Sequence[int]] = None,
         rows: Optional[Sequence[int]] = None, want_weights: bool = False,
         lib=None) -> OracleResult:
    """fp64 reference of the fused SDPA forward.

    q [B,Hq,Tq,d]; k, v [B,Hkv,Tkv,d]; ``mask`` is a float (MASK_FLOAT) or
    boolean/uint8 (MASK_BOOL) array broadcastable to [B,Hq,Tq,Tkv] (size-1
    axes broadcast); rel_pos_h [q_hw[0]+k_hw[0]-1, d] and rel_pos_w
    [q_hw[1]+k_hw[1]-1, d] (2*K-1 rows each when the query and key grids are
    equal; with grids of their own, the offset qh - kh runs over
    -(Kh-1) .. Qh-1 and the shift Kh-1 maps it onto the table's rows).
    ``rows`` restricts the computation to those query rows (same rows for
    every (b, h)); the result then has len(rows) rows."""
    lib = lib or load()
    qd, kd, vd = _f64(q), _f64(k), _f64(v)
    B, Hq, Tq, d = qd.shape
    _, Hkv, Tkv, _ = kd.shape
    fm = bm = None
    msb = msh = msq = 0
    if mask_kind in (MASK_FLOAT, MASK_BOOL):
        if hasattr(mask, "detach"):
            mask = mask.detach().to("cpu").numpy() if mask_kind == MASK_BOOL else mask.detach().to("cpu").double().numpy()
        mk = np.asarray(mask)
        while mk.ndim < 4:
            mk = mk[None]
        if mk.shape[3] != Tkv or mk.shape[2] != Tq:
            raise ValueError("mask must end in [Tq, Tkv]")
        if mask_kind == MASK_FLOAT:
            fm = np.ascontiguousarray(mk, dtype=np.float64)
            base = fm
        else:
            bm = np.ascontiguousarray(mk != 0, dtype=np.uint8)
            base = bm
        msq = Tkv
        msh = 0 if base.shape[1] == 1 else Tq * Tkv
        msb = 0 if base.shape[0] == 1 else base.shape[1] * Tq * Tkv
    rh, rw = _f64(rel_pos_h), _f64(rel_pos_w)
    qh, qw = (q_hw if q_hw is not None else (0, 0))
    kh, kw = (k_hw if k_hw is not None else (0, 0))
    if rh is not None and rw is not None:
        if rh.shape != (qh + kh - 1, d) or rw.shape != (qw + kw - 1, d):
            raise ValueError("rel tables must be [q_hw[0]+k_hw[0]-1, d] and [q_hw[1]+k_hw[1]-1, d]")
    rows_arr = None
    n = Tq
    if rows is not None:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = len(rows_arr)
        if n and (rows_arr.min() < 0 or rows_arr.max() >= Tq):
            raise ValueError("row index out of range")
    out = np.zeros((B, Hq, n, d), dtype=np.float64)
    lse = np.zeros((B, Hq, n), dtype=np.float64)
    w = np.zeros((B, Hq, n, Tkv), dtype=np.float64) if want_weights else None
    rc = lib.oracle_sdpa_rows(_ptr(qd), _ptr(kd), _ptr(vd), B, Hq, Hkv, Tq, Tkv, d, float(scale),
                              int(mask_kind), int(offset), int(window), _ptr(fm), _ptr(bm),
                              msb, msh, msq, _ptr(rh), _ptr(rw), int(qh), int(qw), int(kh), int(kw),
                              _ptr(rows_arr), n, _ptr(out), _ptr(lse), _ptr(w))
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return OracleResult(out=out, lse=lse, weights=w)


def merge(outs: Sequence, lses: Sequence):
    """Combine attention results over disjoint key subsets into the result
    over their union, in fp64.

    Part i holds ``out_i = sum_j p_ij v_j / l_i`` and ``lse_i = m_i + log l_i``
    over its own keys (the natural-log sum-exp of its score rows, -inf when
    no key is visible).  Over the union the normaliser is
    ``L = log sum_i exp(lse_i)`` and every part's unnormalised sum is
    ``exp(lse_i) * out_i``, so ``out = sum_i exp(lse_i - L) * out_i``; a row
    with no visible key anywhere gives ``out = 0``, ``L = -inf``.  This is the
    split-key combination the Axon PR's attention reaches by summing the
    softmax numerators of all keys (PR description: softmax(Q.K^T*scale+mask).V
    over the whole key axis).  Inputs: sequences of arrays [..., d] and [...].
    Returns (out, lse) as float64 arrays."""
    o = np.stack([_f64(x) for x in outs])            # [n, ..., d]
    s = np.stack([_f64(x) for x in lses])            # [n, ...]
    top = np.max(s, axis=0)                          # [...]
    finite = np.isfinite(top)
    shifted = np.where(finite[None], s - np.where(finite, top, 0.0)[None], -np.inf)
    w = np.exp(shifted)                              # exp(lse_i - top), 0 for -inf parts
    tot = np.sum(w, axis=0)
    lse = np.where(finite, top + np.log(np.where(finite, tot, 1.0)), -np.inf)
    wn = np.where(finite[None], w / np.where(finite, tot, 1.0)[None], 0.0)
    out = np.sum(wn[..., None] * o, axis=0)
    return out, lse
