"""Seeded synthetic workloads for the fused SDPA forward.

This module only draws random inputs (a seeded CPU ``torch.Generator``, the
draws made in the fixed order q, k, v, rel_pos_h, rel_pos_w, mask, then each
tensor rounded once to its I/O dtype) and describes the shapes.  It holds none
of the attention arithmetic, so both the CUDA path and the fp64 oracle can be
fed from it.

The shapes follow the workloads the pages talk about: the SAM ViT-B image
encoder's global attention over a 64x64 patch grid and its 14x14 windowed
attention (mlx-examples issue "segment_anything: fuse attention ...", image
encoder Attention), the mask decoder's two-way cross attention with head_dim
16 (same issue, transformer.py Attention; candle PR, head_dim=16 support),
and a generic GQA model under the Axon :mask family (Axon PR description).
The pages name no dataset; every tensor is synthetic.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import torch

MASK_NONE, MASK_CAUSAL, MASK_SLIDING, MASK_FLOAT, MASK_BOOL = 0, 1, 2, 3, 4
MASK_NAMES = {MASK_NONE: "none", MASK_CAUSAL: "causal", MASK_SLIDING: "sliding",
              MASK_FLOAT: "float", MASK_BOOL: "bool"}


@dataclass(frozen=True)
class Spec:
    """Shape and distribution of one workload."""
    name: str
    dtype: torch.dtype
    B: int
    Hq: int
    Hkv: int
    Tq: int
    Tkv: int
    d: int
    scale: float
    seed: int
    qkv_std: float = 1.0
    # decomposed relative position (SAM): query / key patch grids and table std
    q_hw: Optional[Tuple[int, int]] = None
    k_hw: Optional[Tuple[int, int]] = None
    rel_std: float = 0.02
    # mask
    mask_kind: int = MASK_NONE
    offset: int = 0
    window: int = 0
    mask_std: float = 1.0
    mask_neg_inf_frac: float = 0.0
    mask_heads: int = 1          # 1 = [B,1,Tq,Tkv] broadcast over heads, else Hq
    note: str = ""

    @property
    def rel(self) -> bool:
        return self.q_hw is not None

    def table_rows(self) -> Tuple[int, int]:
        """Rows of the rel-pos tables: Qh + Kh - 1 and Qw + Kw - 1 (2*K - 1 for
        equal query and key grids)."""
        return self.q_hw[0] + self.k_hw[0] - 1, self.q_hw[1] + self.k_hw[1] - 1

    # -- algorithmic work (counts the pages' math, not tile padding) ---------
    def allowed_pairs_per_head(self) -> int:
        """Visible (query, key) pairs of one (b, h) under a causal/sliding mask;
        Tq*Tkv otherwise (a float/bool mask cannot be skipped at tile level)."""
        Tq, Tkv = self.Tq, self.Tkv
        if self.mask_kind == MASK_CAUSAL:
            return sum(max(0, min(Tkv, i + self.offset + 1)) for i in range(Tq))
        if self.mask_kind == MASK_SLIDING:
            tot = 0
            for i in range(Tq):
                hi = min(Tkv - 1, i + self.offset)
                lo = max(0, i + self.offset - self.window + 1)
                tot += max(0, hi - lo + 1)
            return tot
        return Tq * Tkv

    def flops(self) -> float:
        """4*d per visible pair (QK^T and PV), plus 2*d*(Kh+Kw) per query row for
        the rel-pos projections."""
        f = 4.0 * self.d * self.allowed_pairs_per_head() * self.B * self.Hq
        if self.rel:
            f += 2.0 * self.d * (self.k_hw[0] + self.k_hw[1]) * self.Tq * self.B * self.Hq
        return f

    def bytes(self) -> float:
        """Q, K, V, O once each, plus the mask and rel-pos tables once."""
        e = 4 if self.dtype == torch.float32 else 2
        n = (2 * self.B * self.Hq * self.Tq + 2 * self.B * self.Hkv * self.Tkv) * self.d * e
        if self.rel:
            n += sum(self.table_rows()) * self.d * e
        if self.mask_kind == MASK_FLOAT:
            n += self.B * self.mask_heads * self.Tq * self.Tkv * e
        if self.mask_kind == MASK_BOOL:
            n += self.B * self.mask_heads * self.Tq * self.Tkv
        return float(n)


@dataclass
class Workload:
    spec: Spec
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    rel_pos_h: Optional[torch.Tensor] = None
    rel_pos_w: Optional[torch.Tensor] = None
    mask: Optional[torch.Tensor] = None   # [B, 1|Hq, Tq, Tkv], I/O dtype (float) or uint8 (bool)
    extra: Dict[str, object] = field(default_factory=dict)


def _randn(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def make(spec: Spec, seed: Optional[int] = None) -> Workload:
    """Draw the inputs of ``spec`` on the CPU, deterministically from the seed."""
    g = torch.Generator(device="cpu")
    g.manual_seed(spec.seed if seed is None else seed)
    dt = spec.dtype
    q = _randn(g, (spec.B, spec.Hq, spec.Tq, spec.d), spec.qkv_std).to(dt)
    k = _randn(g, (spec.B, spec.Hkv, spec.Tkv, spec.d), spec.qkv_std).to(dt)
    v = _randn(g, (spec.B, spec.Hkv, spec.Tkv, spec.d), spec.qkv_std).to(dt)
    rh = rw = None
    if spec.rel:
        nh, nw = spec.table_rows()
        rh = _randn(g, (nh, spec.d), spec.rel_std).to(dt)
        rw = _randn(g, (nw, spec.d), spec.rel_std).to(dt)
    mask = None
    if spec.mask_kind == MASK_FLOAT:
        shape = (spec.B, spec.mask_heads, spec.Tq, spec.Tkv)
        m = _randn(g, shape, spec.mask_std)
        if spec.mask_neg_inf_frac > 0:
            drop = torch.rand(*shape, generator=g) < spec.mask_neg_inf_frac
            # never a fully masked row: such a row keeps its diagonal entry
            full = drop.all(dim=-1)
            if bool(full.any()):
                idx = full.nonzero()
                for b, h, i in idx.tolist():
                    drop[b, h, i, min(i, spec.Tkv - 1)] = False
            m = m.masked_fill(drop, float("-inf"))
        mask = m.to(dt)
    elif spec.mask_kind == MASK_BOOL:
        shape = (spec.B, spec.mask_heads, spec.Tq, spec.Tkv)
        keep = torch.rand(*shape, generator=g) >= max(spec.mask_neg_inf_frac, 0.0)
        full = ~keep.any(dim=-1)
        if bool(full.any()):
            for b, h, i in full.nonzero().tolist():
                keep[b, h, i, min(i, spec.Tkv - 1)] = True
        mask = keep.to(torch.uint8)
    return Workload(spec=spec, q=q, k=k, v=v, rel_pos_h=rh, rel_pos_w=rw, mask=mask)


# --------------------------------------------------------------------------
# The benchmark workloads (full sizes).
# --------------------------------------------------------------------------
BF16, F32 = torch.bfloat16, torch.float32

SPECS: Dict[str, Spec] = {
    # Tiny rel-pos SDPA in fp32: 8x8 grid, head_dim 16, two heads.
    "tiny_relpos_f32": Spec("tiny_relpos_f32", F32, 1, 2, 2, 64, 64, 16, 0.25, seed=0,
                            q_hw=(8, 8), k_hw=(8, 8), rel_std=0.02),
    # SAM ViT-B global attention: 64x64 patch grid, 12 heads, head_dim 64.
    "sam_global": Spec("sam_global", BF16, 1, 12, 12, 4096, 4096, 64, 0.125, seed=1,
                       qkv_std=1.0 / math.sqrt(2.0), q_hw=(64, 64), k_hw=(64, 64), rel_std=0.02),
    # SAM ViT-B windowed attention: 25 windows of 14x14 x batch 4 = 100 batches.
    "sam_windowed": Spec("sam_windowed", BF16, 100, 12, 12, 196, 196, 64, 0.125, seed=2,
                         q_hw=(14, 14), k_hw=(14, 14), rel_std=0.02),
    # SAM mask decoder, head_dim 16, 8 heads, batch 4: both cross directions and self.
    "decoder_token_to_image": Spec("decoder_token_to_image", BF16, 4, 8, 8, 8, 4096, 16, 0.25, seed=3),
    "decoder_image_to_token": Spec("decoder_image_to_token", BF16, 4, 8, 8, 4096, 8, 16, 0.25, seed=3),
    "decoder_self": Spec("decoder_self", BF16, 4, 8, 8, 8, 8, 16, 0.25, seed=3),
    # Generic GQA, 32 query heads over 8 kv heads, head_dim 128, T = 8192.
    "gqa_causal": Spec("gqa_causal", BF16, 2, 32, 8, 8192, 8192, 128, 1.0 / math.sqrt(128.0), seed=4,
                       mask_kind=MASK_CAUSAL),
    "gqa_sliding": Spec("gqa_sliding", BF16, 2, 32, 8, 8192, 8192, 128, 1.0 / math.sqrt(128.0), seed=4,
                        mask_kind=MASK_SLIDING, window=1024, offset=0),
    "gqa_float_mask": Spec("gqa_float_mask", BF16, 2, 32, 8, 8192, 8192, 128, 1.0 / math.sqrt(128.0),
                           seed=4, mask_kind=MASK_FLOAT, mask_std=1.0, mask_neg_inf_frac=0.10,
                           mask_heads=1),
}

# Shapes outside the benchmark, for the ncu evidence of kernels no benchmark
# workload reaches: head_dim 16 with long key axes, on the tensor-core small-d
# kernel (1024 query rows against 2048 keys) and on the global-workspace
# split-KV kernel (8 rows against 16384 keys).
EXTRA_SPECS: Dict[str, Spec] = {
    "d16_long_self": Spec("d16_long_self", BF16, 4, 8, 8, 1024, 2048, 16, 0.25, seed=3),
    "d16_very_long_keys": Spec("d16_very_long_keys", BF16, 4, 8, 8, 8, 16384, 16, 0.25, seed=3),
}


def spec_named(name: str) -> Spec:
    """A benchmark workload, or one of the extra profiling shapes."""
    return SPECS[name] if name in SPECS else EXTRA_SPECS[name]


# Bias-dominated companions: with these the bias decides the scores, so a
# missing or misindexed bias fails every gate.
STRONG_SPECS: Dict[str, Spec] = {
    "tiny_relpos_f32_strong": replace(SPECS["tiny_relpos_f32"], name="tiny_relpos_f32_strong", rel_std=1.0),
    "sam_global_strong": replace(SPECS["sam_global"], name="sam_global_strong", rel_std=1.0),
    "gqa_float_mask_strong": replace(SPECS["gqa_float_mask"], name="gqa_float_mask_strong", mask_std=2.0),
}


def scaled(spec: Spec, **kw) -> Spec:
    """A copy of ``spec`` with some fields replaced (used for the reduced parity sizes)."""
    return replace(spec, **kw)
