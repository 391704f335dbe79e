"""GPU parity: every kernel family of libsdpa against the fp64 oracle, element
by element, on seeded inputs that span several 128-row tiles and ragged tails,
for every mask kind, rel-pos, GQA/MQA, head_dim 16/64/128, fp32 and bf16."""
from __future__ import annotations

import math
import zlib

import numpy as np
import pytest
import torch

from attention_sdpa_fwd_b200 import workloads as W
from helpers import GATES, assert_gates, gpu_run, oracle_ref, stats, passes

pytestmark = pytest.mark.gpu

F32, BF16 = torch.float32, torch.bfloat16


def S_(name, dtype, B, Hq, Hkv, Tq, Tkv, d, **kw):
    kw.setdefault("scale", 1.0 / math.sqrt(d))
    kw.setdefault("seed", zlib.crc32(name.encode()) % 1000)
    return W.Spec(name, dtype, B, Hq, Hkv, Tq, Tkv, d, **kw)


CASES = [
    S_("relpos_f32_d16_8x8", F32, 1, 2, 2, 64, 64, 16, scale=0.25, q_hw=(8, 8), k_hw=(8, 8), rel_std=0.5, seed=1),
    S_("relpos_f32_d64_10x20", F32, 1, 2, 2, 200, 200, 64, q_hw=(10, 20), k_hw=(10, 20), rel_std=0.3, seed=2),
    S_("relpos_bf16_d64_10x20", BF16, 2, 3, 3, 200, 200, 64, q_hw=(10, 20), k_hw=(10, 20), rel_std=0.3, seed=3),
    S_("relpos_bf16_d64_13x23", BF16, 1, 2, 2, 299, 299, 64, q_hw=(13, 23), k_hw=(13, 23), rel_std=0.3, seed=4),
    S_("relpos_bf16_d128_16x16", BF16, 1, 2, 2, 256, 256, 128, q_hw=(16, 16), k_hw=(16, 16), rel_std=0.3, seed=5),
    S_("relpos_bf16_d64_14x14_b5", BF16, 5, 2, 2, 196, 196, 64, q_hw=(14, 14), k_hw=(14, 14), rel_std=0.5, seed=6),
    S_("relpos_bf16_d16_9x7", BF16, 2, 2, 2, 63, 63, 16, q_hw=(9, 7), k_hw=(9, 7), rel_std=0.5, seed=7),
    S_("none_bf16_d64_ragged", BF16, 2, 4, 2, 300, 333, 64, seed=8),
    S_("none_bf16_d128_ragged", BF16, 1, 4, 1, 257, 383, 128, seed=9),
    S_("none_bf16_d16_ragged", BF16, 2, 4, 4, 150, 77, 16, seed=10),
    S_("none_f32_d128", F32, 1, 2, 1, 130, 140, 128, seed=11),
    S_("none_bf16_d64_tq1", BF16, 1, 2, 2, 1, 500, 64, seed=12),
    S_("none_bf16_d64_tkv1", BF16, 1, 2, 2, 300, 1, 64, seed=13),
    S_("causal_bf16_d128", BF16, 1, 4, 2, 300, 300, 128, mask_kind=W.MASK_CAUSAL, seed=14),
    S_("causal_bf16_d64_offset", BF16, 1, 2, 2, 200, 333, 64, mask_kind=W.MASK_CAUSAL, offset=133, seed=15),
    S_("causal_bf16_d64_negoffset", BF16, 1, 2, 2, 260, 260, 64, mask_kind=W.MASK_CAUSAL, offset=-5, seed=16),
    S_("causal_f32_d64", F32, 1, 2, 1, 129, 129, 64, mask_kind=W.MASK_CAUSAL, seed=17),
    S_("sliding_bf16_d128", BF16, 1, 4, 2, 400, 400, 128, mask_kind=W.MASK_SLIDING, window=37, seed=18),
    S_("sliding_bf16_d64_offset", BF16, 1, 2, 1, 300, 350, 64, mask_kind=W.MASK_SLIDING, window=150,
       offset=50, seed=19),
    S_("sliding_bf16_d16", BF16, 1, 2, 2, 200, 200, 16, mask_kind=W.MASK_SLIDING, window=1, seed=20),
    S_("float_bf16_d128_bcast", BF16, 2, 4, 2, 260, 300, 128, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.1, mask_heads=1, seed=21),
    S_("float_bf16_d64_perhead", BF16, 1, 3, 3, 200, 256, 64, mask_kind=W.MASK_FLOAT, mask_std=2.0,
       mask_neg_inf_frac=0.3, mask_heads=3, seed=22),
    S_("float_f32_d16", F32, 1, 2, 2, 100, 90, 16, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=1, seed=23),
    S_("bool_bf16_d64", BF16, 2, 2, 1, 300, 260, 64, mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.5,
       mask_heads=2, seed=24),
    S_("bool_bf16_d128_bcast", BF16, 1, 4, 4, 130, 128, 128, mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.9,
       mask_heads=1, seed=25),
    S_("mqa_bf16_d128", BF16, 2, 8, 1, 200, 256, 128, seed=26),
    # head_dim 16: mask-decoder shapes, reduced, with every mask kind and GQA
    S_("d16_cross_short_q", BF16, 2, 4, 2, 9, 1500, 16, seed=40),
    S_("d16_cross_short_kv", BF16, 2, 4, 4, 700, 7, 16, seed=41),
    S_("d16_causal_gqa", BF16, 1, 4, 2, 300, 300, 16, mask_kind=W.MASK_CAUSAL, offset=3, seed=42),
    S_("d16_float_mask", BF16, 2, 2, 2, 40, 1100, 16, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.3, mask_heads=2, seed=43),
    S_("d16_bool_mask", BF16, 1, 2, 1, 130, 333, 16, mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.6,
       mask_heads=1, seed=44),
    S_("d16_sliding_long_kv", BF16, 1, 2, 2, 16, 3000, 16, mask_kind=W.MASK_SLIDING, window=700, offset=2000,
       seed=45),
    # head_dim 16, short query axis and enough heads for the small-d kernel to
    # pack several heads per CTA (16 heads of 7 rows; 4 heads of 30 rows; 2
    # heads of 16 rows with the second CTA's second group past the last head)
    S_("d16_packed16_causal_gqa", BF16, 150, 16, 8, 7, 19, 16, mask_kind=W.MASK_CAUSAL, offset=11, seed=46),
    S_("d16_packed4_float_mask", BF16, 80, 8, 8, 30, 70, 16, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=8, seed=47),
    S_("d16_packed2_sliding_odd_heads", BF16, 160, 3, 3, 16, 50, 16, mask_kind=W.MASK_SLIDING, window=9,
       offset=20, seed=48),
    # enough (batch, head) pairs for the split-KV clusters of 4 larger parts
    # (more than one wave of 8-part clusters): plain, and a float mask per head
    S_("d16_cluster4_cross", BF16, 10, 4, 2, 9, 3000, 16, seed=59),
    S_("d16_cluster4_float_mask", BF16, 13, 3, 3, 20, 1234, 16, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=3, seed=60),
    # the same packing on the tensor-core small-d kernel (64 keys or more):
    # 8 heads of 13 rows per CTA, GQA, causal with an offset
    S_("d16_packed8_mma_causal_gqa", BF16, 150, 8, 4, 13, 100, 16, mask_kind=W.MASK_CAUSAL, offset=60, seed=58),
    # rel-pos shapes the tensor-core path specialises (key-grid width 14/16/32/64)
    S_("relpos_bf16_d64_12x16", BF16, 2, 3, 3, 192, 192, 64, q_hw=(12, 16), k_hw=(12, 16), rel_std=0.5, seed=27),
    S_("relpos_bf16_d64_8x32", BF16, 1, 4, 2, 256, 256, 64, q_hw=(8, 32), k_hw=(8, 32), rel_std=0.5, seed=28),
    S_("relpos_bf16_d64_20x14", BF16, 3, 2, 2, 280, 280, 64, q_hw=(20, 14), k_hw=(20, 14), rel_std=0.5, seed=29),
    S_("relpos_bf16_d64_9x64", BF16, 1, 2, 2, 576, 576, 64, q_hw=(9, 64), k_hw=(9, 64), rel_std=0.5, seed=30),
    S_("relpos_bf16_d64_14x14_strong", BF16, 7, 3, 3, 196, 196, 64, q_hw=(14, 14), k_hw=(14, 14), rel_std=1.0,
       seed=31),
    # rel-pos combined with a causal / sliding mask
    S_("relpos_causal_bf16_d64_12x16", BF16, 1, 2, 2, 192, 192, 64, q_hw=(12, 16), k_hw=(12, 16), rel_std=0.5,
       mask_kind=W.MASK_CAUSAL, seed=32),
    S_("relpos_sliding_bf16_d64_20x14", BF16, 1, 2, 2, 280, 280, 64, q_hw=(20, 14), k_hw=(20, 14), rel_std=0.5,
       mask_kind=W.MASK_SLIDING, window=60, offset=3, seed=33),
    S_("float_bf16_d64_aligned", BF16, 2, 2, 1, 300, 296, 64, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=2, seed=34),
    S_("bool_bf16_d128_aligned", BF16, 1, 2, 2, 260, 272, 128, mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.5,
       mask_heads=1, seed=35),
    # head_dim 128 with a mask tensor runs 64-key tiles with two score buffers:
    # a single key tile, and an odd number of tiles with a ragged last one
    S_("float_bf16_d128_one_tile", BF16, 1, 2, 1, 70, 50, 128, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=1, seed=36),
    S_("float_bf16_d128_odd_tiles", BF16, 2, 3, 3, 200, 300, 128, mask_kind=W.MASK_FLOAT, mask_std=2.0,
       mask_neg_inf_frac=0.1, mask_heads=3, seed=37),
    # key counts that are multiples of 8 (16-byte mask rows): the mask tiles
    # reach shared memory by TMA -- broadcast over heads with a ragged last
    # key tile and query block, one mask per head, a single partial tile
    S_("float_bf16_d128_tma_bcast", BF16, 2, 4, 2, 260, 296, 128, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=1, seed=38),
    S_("float_bf16_d128_tma_perhead", BF16, 1, 3, 1, 130, 200, 128, mask_kind=W.MASK_FLOAT, mask_std=2.0,
       mask_neg_inf_frac=0.3, mask_heads=3, seed=39),
    S_("float_bf16_d128_tma_one_tile", BF16, 1, 2, 2, 40, 40, 128, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=2, seed=49),
    # boolean masks with 16-byte rows (key counts that are multiples of 16):
    # the same TMA tiles, in the 64-byte swizzle; one mask per head with a
    # ragged last tile, and a mostly hidden one with fully masked rows
    S_("bool_bf16_d128_tma_perhead", BF16, 1, 2, 1, 150, 208, 128, mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.6,
       mask_heads=2, seed=56),
    S_("bool_bf16_d128_tma_sparse", BF16, 2, 2, 2, 70, 48, 128, mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.9,
       mask_heads=1, seed=57),
    # more query blocks than SMs: the persistent form walks several per CTA
    # (consecutive units of one CTA differ in window, head and query block)
    S_("persist_relpos_14x14_many", BF16, 40, 4, 4, 196, 196, 64, q_hw=(14, 14), k_hw=(14, 14), rel_std=0.5,
       seed=50),
    S_("persist_relpos_16x16_many", BF16, 20, 8, 8, 256, 256, 64, q_hw=(16, 16), k_hw=(16, 16), rel_std=0.5,
       seed=51),
    S_("persist_relpos_6x14_many", BF16, 50, 4, 2, 84, 84, 64, q_hw=(6, 14), k_hw=(6, 14), rel_std=1.0, seed=52),
    S_("persist_none_ragged_many", BF16, 8, 12, 3, 260, 300, 64, seed=53),
    S_("persist_none_four_tiles_many", BF16, 10, 16, 16, 100, 500, 64, seed=54),
    # three or four units per CTA: both Q buffers are refilled after their
    # first unit (the hand-over that waits for the unit two back)
    S_("persist_relpos_14x14_deep", BF16, 80, 6, 6, 196, 196, 64, q_hw=(14, 14), k_hw=(14, 14), rel_std=0.5,
       seed=55),
    # rel-pos combined with an additive float or a boolean mask tensor
    S_("relpos_float_bf16_d64_12x16", BF16, 2, 2, 1, 192, 192, 64, q_hw=(12, 16), k_hw=(12, 16), rel_std=0.5,
       mask_kind=W.MASK_FLOAT, mask_std=1.0, mask_neg_inf_frac=0.2, mask_heads=2, seed=70),
    S_("relpos_bool_bf16_d64_20x14", BF16, 1, 3, 3, 280, 280, 64, q_hw=(20, 14), k_hw=(20, 14), rel_std=0.5,
       mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.4, mask_heads=1, seed=71),
    S_("relpos_float_bf16_d64_5x64", BF16, 1, 2, 2, 320, 320, 64, q_hw=(5, 64), k_hw=(5, 64), rel_std=0.5,
       mask_kind=W.MASK_FLOAT, mask_std=2.0, mask_neg_inf_frac=0.1, mask_heads=1, seed=72),
    S_("relpos_bool_bf16_d64_8x32_strong", BF16, 1, 2, 2, 256, 256, 64, q_hw=(8, 32), k_hw=(8, 32), rel_std=1.0,
       mask_kind=W.MASK_BOOL, mask_neg_inf_frac=0.5, mask_heads=2, seed=73),
    S_("relpos_float_f32_d16_6x6", F32, 1, 2, 2, 36, 36, 16, q_hw=(6, 6), k_hw=(6, 6), rel_std=0.5,
       mask_kind=W.MASK_FLOAT, mask_std=1.0, mask_neg_inf_frac=0.2, mask_heads=2, seed=74),
    # rel-pos with query and key grids of their own (tables of Qh+Kh-1 and Qw+Kw-1 rows)
    S_("relpos_qk_bf16_d64_q8x16_k12x16", BF16, 2, 2, 2, 128, 192, 64, q_hw=(8, 16), k_hw=(12, 16), rel_std=0.5,
       seed=80),
    S_("relpos_qk_bf16_d64_q10x14_k14x14", BF16, 3, 2, 2, 140, 196, 64, q_hw=(10, 14), k_hw=(14, 14),
       rel_std=0.5, seed=81),
    S_("relpos_qk_bf16_d64_q16x32_k8x32", BF16, 1, 3, 3, 512, 256, 64, q_hw=(16, 32), k_hw=(8, 32), rel_std=0.5,
       seed=82),
    S_("relpos_qk_bf16_d64_q64x64_k16x16", BF16, 1, 2, 2, 4096, 256, 64, q_hw=(64, 64), k_hw=(16, 16),
       rel_std=0.3, seed=83),
    S_("relpos_qk_bf16_d64_q3x64_k5x64_causal", BF16, 1, 2, 2, 192, 320, 64, q_hw=(3, 64), k_hw=(5, 64),
       rel_std=0.5, mask_kind=W.MASK_CAUSAL, offset=100, seed=84),
    S_("relpos_qk_bf16_d16_q5x7_k3x9", BF16, 2, 2, 1, 35, 27, 16, q_hw=(5, 7), k_hw=(3, 9), rel_std=0.5, seed=85),
    S_("relpos_qk_f32_d64_q4x6_k6x4", F32, 1, 2, 2, 24, 24, 64, q_hw=(4, 6), k_hw=(6, 4), rel_std=0.5, seed=86),
    S_("relpos_qk_bf16_d64_q14x14_k7x14_strong", BF16, 40, 2, 2, 196, 98, 64, q_hw=(14, 14), k_hw=(7, 14),
       rel_std=1.0, seed=87),
]
CASE_IDS = [c.name for c in CASES]

PATHS = ["exact", "tcgen05", "small_d", "split_kv", "tc_persistent"]


def applicable(path: str, sp: W.Spec) -> bool:
    import attention_sdpa_fwd_b200 as S
    if path == "exact":
        return True
    if sp.dtype != BF16:
        return False
    if path == "tcgen05":
        if sp.d not in (64, 128):
            return False
        if sp.rel:
            kh, kw = sp.k_hw
            bn = 112 if kw == 14 else 128
            return (sp.d == 64 and kw in (14, 16, 32, 64) and kh <= 64
                    and (max(sp.table_rows()) + 15) // 16 * 16 <= bn)
        return True
    if path in ("small_d", "split_kv"):
        return sp.d == 16 and not sp.rel
    if path == "tc_persistent":
        if sp.d != 64 or sp.mask_kind != W.MASK_NONE:
            return False
        return (not sp.rel) or (sp.k_hw[1] in (14, 16) and sp.k_hw[0] <= 16 and max(sp.table_rows()) <= 32)
    return False


def _implemented(path):
    # a path not built yet reports SDPA_ERR_UNSUPPORTED for everything
    return path in _BUILT


_BUILT = {"exact", "tcgen05", "small_d", "split_kv", "tc_persistent"}


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("sp", CASES, ids=CASE_IDS)
def test_parity(sp, path):
    if not applicable(path, sp) or not _implemented(path):
        pytest.skip(f"{path} does not take this problem")
    wl = W.make(sp)
    out, lse = gpu_run(wl, path=path, want_lse=True)
    ref = oracle_ref(wl)
    assert_gates(out.double().numpy(), ref.out, sp.dtype, f"{sp.name}/{path}", strong=sp.name.endswith("_strong"))
    fin = np.isfinite(ref.lse)
    got = lse.double().numpy()
    assert np.array_equal(np.isfinite(got), fin), "lse -inf pattern"
    assert np.max(np.abs(got[fin] - ref.lse[fin])) < 2e-3, "lse"


@pytest.mark.parametrize("path", ["exact", "tcgen05", "small_d", "split_kv"])
def test_edge_cases(path):
    _edge_cases(path)


def _edge_cases(path):
    import attention_sdpa_fwd_b200 as S
    dev = "cuda"
    d = 16 if path in ("small_d", "split_kv") else 64
    if path == "exact":
        # Tkv = 0: every row sees nothing -> zeros, lse = -inf
        q = torch.randn(1, 2, 5, d, device=dev, dtype=BF16)
        e = torch.empty(1, 2, 0, d, device=dev, dtype=BF16)
        lse = torch.zeros(1, 2, 5, device=dev)
        out = torch.full_like(q, 7.0)
        S.sdpa(q, e, e, 0.1, out=out, lse=lse, path=path)
        torch.cuda.synchronize()
        assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    # causal with a large negative offset: no row sees a key -> zeros, lse = -inf
    q = torch.randn(1, 2, 300, d, device=dev, dtype=BF16)
    lse = torch.zeros(1, 2, 300, device=dev)
    out = torch.full_like(q, 7.0)
    S.sdpa(q, q, q, 0.1, mask_kind=S.MASK_CAUSAL, offset=-400, out=out, lse=lse, path=path)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    # B = 0: nothing to do
    z = torch.empty(0, 2, 5, d, device=dev, dtype=BF16)
    S.sdpa(z, z, z, 0.1, path=path)
    # Tq = Tkv = 1: output is v
    q1 = torch.randn(2, 2, 1, d, device=dev, dtype=BF16)
    k1 = torch.randn(2, 2, 1, d, device=dev, dtype=BF16)
    v1 = torch.randn(2, 2, 1, d, device=dev, dtype=BF16)
    o1 = S.sdpa(q1, k1, v1, path=path)
    torch.cuda.synchronize()
    assert torch.equal(o1, v1)
    # fully masked rows (bool) -> zeros
    q2 = torch.randn(1, 1, 130, d, device=dev, dtype=BF16)
    k2 = torch.randn(1, 1, 144, d, device=dev, dtype=BF16)
    keep = torch.ones(1, 1, 130, 144, device=dev, dtype=torch.uint8)
    keep[0, 0, 3] = 0
    keep[0, 0, 129] = 0
    o2 = S.sdpa(q2, k2, k2, mask_kind=S.MASK_BOOL, mask=keep, path=path)
    torch.cuda.synchronize()
    assert torch.all(o2[0, 0, 3] == 0) and torch.all(o2[0, 0, 129] == 0)
    assert torch.all(o2[0, 0, 4].abs().sum() > 0)


def test_persistent_edges():
    """Persistent form: a single key, a single query, B = 0, and more SMs than units."""
    import attention_sdpa_fwd_b200 as S
    dev = "cuda"
    q1 = torch.randn(3, 2, 1, 64, device=dev, dtype=BF16)
    k1 = torch.randn(3, 2, 1, 64, device=dev, dtype=BF16)
    v1 = torch.randn(3, 2, 1, 64, device=dev, dtype=BF16)
    o1 = S.sdpa(q1, k1, v1, path="tc_persistent")
    torch.cuda.synchronize()
    assert torch.equal(o1, v1)
    z = torch.empty(0, 2, 5, 64, device=dev, dtype=BF16)
    S.sdpa(z, z, z, 0.1, path="tc_persistent")
    torch.cuda.synchronize()


def test_host_entry_point_matches_device_entry_point():
    """sdpa_fwd_host (host buffers, copies inside the call) gives the same bytes."""
    import attention_sdpa_fwd_b200 as S
    sp = CASES[2]
    wl = W.make(sp)
    dev_out, _ = gpu_run(wl)
    qh, kh, vh = (x.contiguous().pin_memory() for x in (wl.q, wl.k, wl.v))
    rh, rw = wl.rel_pos_h.contiguous(), wl.rel_pos_w.contiguous()
    out = torch.empty_like(qh).pin_memory()
    rc = S.sdpa_fwd_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), out.data_ptr(), S.SDPA_BF16,
                         sp.B, sp.Hq, sp.Hkv, sp.Tq, sp.Tkv, sp.d, sp.scale, 0, None,
                         rh.data_ptr(), rw.data_ptr(), sp.q_hw, sp.k_hw, 0,
                         torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    assert torch.equal(out, dev_out)


# More 256-row query blocks than one wave of SMs: the tensor-core path runs
# whole blocks first and splits the remainder's key ranges (merged in-kernel);
# causal problems take their query blocks last-first.
SCHEDULE_CASES = [
    S_("sched_none_bf16_d64_h40", BF16, 1, 40, 40, 1000, 1000, 64, seed=50),
    S_("sched_gqa_bf16_d128_h24", BF16, 3, 24, 8, 600, 777, 128, seed=51),
    S_("sched_causal_bf16_d64_h40", BF16, 1, 40, 20, 1000, 1000, 64, mask_kind=W.MASK_CAUSAL, seed=52),
    S_("sched_relpos_bf16_d64_32x32_h44", BF16, 1, 44, 44, 1024, 1024, 64, q_hw=(32, 32), k_hw=(32, 32),
       rel_std=0.5, seed=53),
]


@pytest.mark.parametrize("sp", SCHEDULE_CASES, ids=[c.name for c in SCHEDULE_CASES])
def test_mixed_schedule(sp):
    from helpers import sample_rows
    wl = W.make(sp)
    out, lse = gpu_run(wl, path="tcgen05", want_lse=True)
    rows = sample_rows(sp.Tq, 160, seed=sp.seed)
    ref = oracle_ref(wl, rows=rows)
    assert_gates(out[:, :, rows].double().numpy(), ref.out, sp.dtype, sp.name)
    got = lse[:, :, rows].double().numpy()
    assert np.max(np.abs(got - ref.lse)) < 2e-3, "lse"


HOST_CASES = [
    # whole-batch slabs (B at least the slab count), per-head float mask with -inf entries
    S_("host_batches_float_mask", BF16, 7, 4, 2, 200, 150, 64, mask_kind=W.MASK_FLOAT, mask_std=1.0,
       mask_neg_inf_frac=0.2, mask_heads=4, seed=60),
    # head slabs covering whole GQA groups (group of 4)
    S_("host_gqa_head_slabs", BF16, 1, 8, 2, 300, 260, 128, mask_kind=W.MASK_CAUSAL, seed=61),
    # rel-pos, several slabs per batch
    S_("host_relpos_slabs", BF16, 2, 6, 6, 192, 192, 64, q_hw=(12, 16), k_hw=(12, 16), rel_std=0.5, seed=62),
]


@pytest.mark.parametrize("sp", HOST_CASES, ids=[c.name for c in HOST_CASES])
def test_host_entry_point_slabs(sp):
    """sdpa_fwd_host pipelines the problem over (batch, head) slabs; the bytes
    must equal the device entry point's, and the values the oracle's."""
    import ctypes
    import attention_sdpa_fwd_b200 as S
    wl = W.make(sp)
    dev_out, _ = gpu_run(wl)
    pin = lambda x: None if x is None else x.contiguous().pin_memory()
    qh, kh, vh, mh = pin(wl.q), pin(wl.k), pin(wl.v), pin(wl.mask)
    rh = wl.rel_pos_h.contiguous() if wl.rel_pos_h is not None else None
    rw = wl.rel_pos_w.contiguous() if wl.rel_pos_w is not None else None
    out = torch.empty_like(qh).pin_memory()
    m = None
    if sp.mask_kind != W.MASK_NONE:
        m = S.sdpa_mask_t(offset=sp.offset, window=sp.window, data=None, stride_b=0, stride_h=0, stride_q=0)
        if mh is not None:
            m.data = mh.data_ptr()
            m.stride_b = 0 if mh.shape[0] == 1 else mh.stride(0)
            m.stride_h = 0 if mh.shape[1] == 1 else mh.stride(1)
            m.stride_q = mh.stride(2)
    rc = S.sdpa_fwd_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), out.data_ptr(), S.SDPA_BF16,
                         sp.B, sp.Hq, sp.Hkv, sp.Tq, sp.Tkv, sp.d, sp.scale, sp.mask_kind,
                         ctypes.byref(m) if m is not None else None,
                         rh.data_ptr() if rh is not None else None, rw.data_ptr() if rw is not None else None,
                         sp.q_hw, sp.k_hw, 0, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    assert torch.equal(out, dev_out)
    ref = oracle_ref(wl)
    assert_gates(out.double().numpy(), ref.out, sp.dtype, sp.name)
