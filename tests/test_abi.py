"""The C-ABI library loads, exports every symbol include/sdpa.h declares, and
rejects bad arguments on the host before touching a GPU (no compute calls)."""
import ctypes
import os
import re

import pytest

import attention_sdpa_fwd_b200 as S
from attention_sdpa_fwd_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w[\w\s\*]*?\b(sdpa_\w+)\s*\(", txt, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    build.build()
    return S.lib()


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "sdpa_fwd" in names and "sdpa_fwd_ex" in names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(names) <= set(S.EXPORTS) | set(names)
    assert set(S.EXPORTS) <= set(names), "binding lists a symbol the header does not declare"


def test_version_and_strerror(L):
    assert S.sdpa_version() >= 100
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert S.sdpa_strerror(code) not in ("", "unknown status")
    assert S.sdpa_strerror(12345) == "unknown status"


# Distinct fake device addresses (never dereferenced: validation fails first).
Q, K, V, O = 0x100000, 0x200000, 0x300000, 0x400000
BF16 = S.SDPA_BF16


def sel(*a, **kw):
    args = dict(q=Q, k=K, v=V, out=O, dtype=BF16, B=1, Hq=4, Hkv=2, Tq=8, Tkv=8, d=64,
                mask_kind=0, mask=None, rh=None, rw=None, q_hw=None, k_hw=None)
    args.update(kw)
    m = args["mask"]
    return S.sdpa_select_path(args["q"], args["k"], args["v"], args["out"], args["dtype"], args["B"],
                              args["Hq"], args["Hkv"], args["Tq"], args["Tkv"], args["d"], args["mask_kind"],
                              ctypes.byref(m) if m is not None else None, args["rh"], args["rw"],
                              args["q_hw"], args["k_hw"])


def test_valid_problem_selects_a_path(L):
    assert sel() >= 0


def test_auto_takes_persistent_form_for_many_short_problems(L):
    """SAM windowed attention (100 windows x 12 heads of 14x14 tokens), with or
    without the rel-pos bias, takes the persistent tensor-core form; SAM global
    attention (one 64x64 grid, 12 heads: 16 query blocks per head), masked
    problems and long key axes keep the one-CTA-per-block form."""
    rh, rw = 0x500000, 0x600000
    far = dict(q=0x10000000, k=0x20000000, v=0x30000000, out=0x40000000)  # spans of up to 256 MB apart
    sel_far = lambda **kw: sel(**far, **kw)
    win = dict(B=100, Hq=12, Hkv=12, Tq=196, Tkv=196, rh=rh, rw=rw, q_hw=(ctypes.c_int * 2)(14, 14),
               k_hw=(ctypes.c_int * 2)(14, 14))
    assert sel_far(**win) == S.PATH_TC_PERSISTENT
    glob = dict(B=1, Hq=12, Hkv=12, Tq=4096, Tkv=4096, rh=rh, rw=rw, q_hw=(ctypes.c_int * 2)(64, 64),
                k_hw=(ctypes.c_int * 2)(64, 64))
    assert sel_far(**glob) == S.PATH_TCGEN05
    assert sel_far(B=100, Hq=12, Hkv=12, Tq=196, Tkv=196, mask_kind=S.MASK_CAUSAL) == S.PATH_TCGEN05
    assert sel_far(B=100, Hq=12, Hkv=12, Tq=196, Tkv=196) == S.PATH_TC_PERSISTENT
    assert sel_far(B=100, Hq=12, Hkv=12, Tq=196, Tkv=700) == S.PATH_TCGEN05   # > 4 key tiles per block


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), -1),                 # Hq % Hkv != 0
    (dict(Hkv=0), -1),
    (dict(B=-1), -1),
    (dict(Tq=-5), -1),
    (dict(d=32), -2),                        # head_dim outside {16, 64, 128}
    (dict(d=96), -2),
    (dict(dtype=7), -1),
    (dict(q=0), -1),                         # NULL q with work to do
    (dict(k=0), -1),
    (dict(out=0), -1),
    (dict(out=Q + 64), -1),                  # out overlaps q
    (dict(q=Q + 1), -3),                     # bf16 pointer not 2-byte aligned
    (dict(mask_kind=9), -1),
    (dict(mask_kind=S.MASK_SLIDING), -1),    # sliding needs a descriptor
    (dict(mask_kind=S.MASK_SLIDING, mask=S.sdpa_mask_t(window=0)), -1),
    (dict(mask_kind=S.MASK_FLOAT), -1),      # float mask needs a descriptor
    (dict(mask_kind=S.MASK_FLOAT, mask=S.sdpa_mask_t(data=None)), -1),
    (dict(mask_kind=S.MASK_FLOAT, mask=S.sdpa_mask_t(data=0x500001, stride_q=8)), -3),
    (dict(mask_kind=S.MASK_BOOL, mask=S.sdpa_mask_t(data=0x500000, stride_q=-8)), -1),
    (dict(rh=0x600000), -1),                 # only one table
    (dict(rh=0x600000, rw=0x700000), -1),    # tables without grids
    (dict(rh=0x600000, rw=0x700000, q_hw=(2, 3), k_hw=(2, 4)), -1),   # grid != Tq
    (dict(rh=0x600000, rw=0x700000, q_hw=(0, 8), k_hw=(0, 8)), -1),
    (dict(rh=0x600001, rw=0x700000, q_hw=(2, 4), k_hw=(2, 4)), -3),
])
def test_invalid_arguments_rejected(L, kw, code):
    assert sel(**kw) == code


def test_unequal_query_and_key_grids_are_valid(L):
    """Rel-pos with query and key grids of their own (tables of Qh+Kh-1 and
    Qw+Kw-1 rows) is a valid problem; the tensor-core path takes it when the
    key-grid width is one it specialises and both tables fit its 128 rows."""
    rh, rw = 0x600000, 0x700000
    far = dict(q=0x10000000, k=0x20000000, v=0x30000000, out=0x40000000)
    assert sel(**far, rh=rh, rw=rw, Tq=8, Tkv=8, q_hw=(2, 4), k_hw=(4, 2)) == S.PATH_EXACT
    assert sel(**far, rh=rh, rw=rw, Tq=64, Tkv=256, q_hw=(8, 8), k_hw=(16, 16)) == S.PATH_TCGEN05
    assert sel(**far, rh=rh, rw=rw, Tq=4096, Tkv=1024, q_hw=(64, 64), k_hw=(32, 32)) == S.PATH_TCGEN05
    # 100 + 64 - 1 table rows do not fit the 128-row projection
    assert sel(**far, rh=rh, rw=rw, Tq=6400, Tkv=4096, q_hw=(100, 64), k_hw=(64, 64)) == S.PATH_EXACT


def test_empty_problems_are_valid(L):
    assert sel(B=0, q=0, out=0) >= 0
    assert sel(Tq=0, q=0, out=0) >= 0
    assert sel(Tkv=0, k=0, v=0) >= 0


def test_forward_rejects_before_launch(L):
    # invalid problems return their status from sdpa_fwd / sdpa_fwd_ex without touching a device
    rc = S.sdpa_fwd(Q, K, V, O, BF16, 1, 3, 2, 8, 8, 64, 0.125, 0, None, None, None, None, None, None)
    assert rc == -1
    rc = S.sdpa_fwd_ex(Q, K, V, O, BF16, 1, 4, 2, 8, 8, 64, float("nan"), 0, None, None, None, None, None,
                       None, 0, None)
    assert rc == -1
    rc = S.sdpa_fwd_ex(Q, K, V, O, BF16, 1, 4, 2, 8, 8, 64, 0.1, 0, None, None, None, None, None, None, 17, None)
    assert rc == -1
    rc = S.sdpa_fwd_host(Q, K, V, O, BF16, 1, 4, 2, 8, 8, 32, 0.1, 0, None, None, None, None, None, 0, None)
    assert rc == -2


def fwd_ex(path, **kw):
    args = dict(q=Q, k=K, v=V, out=O, dtype=BF16, B=1, Hq=4, Hkv=2, Tq=8, Tkv=8, d=64,
                mask_kind=0, mask=None, rh=None, rw=None, q_hw=None, k_hw=None)
    args.update(kw)
    m = args["mask"]
    return S.sdpa_fwd_ex(args["q"], args["k"], args["v"], args["out"], args["dtype"], args["B"], args["Hq"],
                         args["Hkv"], args["Tq"], args["Tkv"], args["d"], 0.125, args["mask_kind"],
                         ctypes.byref(m) if m is not None else None, args["rh"], args["rw"], args["q_hw"],
                         args["k_hw"], None, path, None)


REL14 = dict(rh=0x600000, rw=0x700000, Tq=196, Tkv=196, q_hw=(14, 14), k_hw=(14, 14))


@pytest.mark.parametrize("path,kw", [
    (S.PATH_TC_PERSISTENT, dict(d=128)),                                   # head_dim 64 only
    (S.PATH_TC_PERSISTENT, dict(d=16)),
    (S.PATH_TC_PERSISTENT, dict(dtype=S.SDPA_F32)),                         # bf16 only
    (S.PATH_TC_PERSISTENT, dict(mask_kind=S.MASK_CAUSAL, mask=S.sdpa_mask_t())),
    (S.PATH_TC_PERSISTENT, dict(REL14, q_hw=(7, 28), k_hw=(7, 28))),          # key-grid width 28
    (S.PATH_TC_PERSISTENT, dict(REL14, Tq=238, Tkv=238, q_hw=(17, 14), k_hw=(17, 14))),  # height 17 > 16
    (S.PATH_TCGEN05, dict(d=16)),
    (S.PATH_TCGEN05, dict(REL14, q_hw=(7, 28), k_hw=(7, 28))),
    (S.PATH_SMALL_D, dict(d=64)),
    (S.PATH_SPLIT_KV, dict(REL14, d=16)),
])
def test_forced_path_rejected_before_launch(L, path, kw):
    """A forced kernel family that cannot take the problem returns
    SDPA_ERR_UNSUPPORTED before any device work (no GPU needed)."""
    assert fwd_ex(path, **kw) == -2


def test_binding_has_no_cpu_path():
    import torch
    q = torch.zeros(1, 1, 4, 16)
    with pytest.raises(ValueError):
        S.sdpa(q, q, q)


def test_strided_entry_validates_strides(L):
    """sdpa_fwd_strided rejects non-positive strides and an output whose
    address span overlaps an input's, before any launch."""
    B, H, T, d = 1, 2, 8, 64
    q, k, v, out = 4096, 4096 * 64, 4096 * 128, 4096 * 256  # fake, 16-byte aligned, disjoint
    base = dict(dtype=S.SDPA_BF16, B=B, Hq=H, Hkv=H, Tq=T, Tkv=T, d=d, scale=0.1, mask_kind=0, mask_ptr=None,
                rel_pos_h=None, rel_pos_w=None, q_hw=None, k_hw=None, lse=None, path=0, stream=None)

    def call(qs=None, ks=None, vs=None, os_=None, out_ptr=out):
        return S.sdpa_fwd_strided(q, qs, k, ks, v, vs, out_ptr, os_, **base)

    for bad in ((0, 64, 128), (1024, -64, 128), (1024, 64, 0)):
        assert call(qs=bad) == -1
        assert call(ks=bad) == -1
        assert call(os_=bad) == -1
    # bshd out whose span reaches into q
    assert call(os_=(T * H * d, d, H * d), out_ptr=q + 64) == -1
    # unsupported head_dim is reported as such whatever the strides
    b2 = dict(base, d=48)
    assert S.sdpa_fwd_strided(q, None, k, None, v, None, out, None, **b2) == -2


def test_merge_validates_on_host(L):
    o, l = [4096, 8192], [65536, 131072]  # fake, aligned, disjoint device addresses
    ok = dict(dtype=S.SDPA_BF16, B=1, Hq=2, Tq=8, d=64, stream=None)
    assert S.sdpa_merge(o, l, 0, 1 << 20, 1 << 21, **ok) == -1          # no parts
    assert S.sdpa_merge(o * 9, l * 9, 17, 1 << 20, 1 << 21, **ok) == -1  # too many parts
    assert S.sdpa_merge(o, l, 2, 1 << 20, 1 << 21, **dict(ok, d=48)) == -2
    assert S.sdpa_merge(o, l, 2, (1 << 20) + 8, 1 << 21, **ok) == -3     # out not 16-byte aligned
    assert S.sdpa_merge(o, l, 2, 8192 + 64, 1 << 21, **ok) == -1         # out overlaps part 1
    assert S.sdpa_merge(o, l, 2, 1 << 20, None, **dict(ok, Tq=0)) == 0   # nothing to do


@pytest.mark.parametrize("where", ["q", "k", "v", "out", "mask"])
def test_lse_overlapping_an_input_is_rejected(L, where):
    """lse is written while other CTAs still read q, k, v and the mask tensor:
    an lse buffer that overlaps any of them (or out) is an argument error,
    reported before any launch."""
    mask_data = 0x500000
    m = S.sdpa_mask_t(data=mask_data, stride_b=0, stride_h=0, stride_q=8)
    at = dict(q=Q, k=K, v=V, out=O, mask=mask_data)[where]
    lse = ctypes.c_void_p(at + 4)
    rc = S.sdpa_fwd_ex(Q, K, V, O, BF16, 1, 4, 2, 8, 8, 64, 0.125, S.MASK_FLOAT, ctypes.byref(m),
                       None, None, None, None, lse, 0, None)
    assert rc == -1
