"""Python binding of libsdpa, the fused SDPA forward for B200 (sm_100a).

Argument marshalling only: every step of the attention runs in the CUDA
kernels of ``libsdpa.so`` behind the C ABI declared in ``include/sdpa.h``.
PyTorch supplies device memory and the current stream.  There is no CPU
fallback: importing works without a GPU (so the ABI can be inspected), but
every call needs CUDA tensors and the built library, and raises otherwise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
RELEASE_LIB_PATH = os.path.join(_PKG, "libsdpa.so")
# the build with device-side index checks (see sdpa_debug_checks)
DEBUG_LIB_PATH = os.path.join(_PKG, "libsdpa_debug.so")
# SDPA_DEBUG=1 in the environment selects the debug build for this process
LIB_PATH = DEBUG_LIB_PATH if os.environ.get("SDPA_DEBUG", "0") not in ("", "0") else RELEASE_LIB_PATH

SDPA_F32, SDPA_BF16 = 0, 1
MASK_NONE, MASK_CAUSAL, MASK_SLIDING, MASK_FLOAT, MASK_BOOL = 0, 1, 2, 3, 4
PATH_AUTO, PATH_EXACT, PATH_TCGEN05, PATH_SMALL_D, PATH_SPLIT_KV, PATH_TC_PERSISTENT = 0, 1, 2, 3, 4, 5
PATHS = {"auto": PATH_AUTO, "exact": PATH_EXACT, "tcgen05": PATH_TCGEN05,
         "small_d": PATH_SMALL_D, "split_kv": PATH_SPLIT_KV, "tc_persistent": PATH_TC_PERSISTENT}
STATUS = {0: "SDPA_OK", -1: "SDPA_ERR_INVALID_ARG", -2: "SDPA_ERR_UNSUPPORTED",
          -3: "SDPA_ERR_MISALIGNED", -4: "SDPA_ERR_CUDA", -5: "SDPA_ERR_TIMEOUT",
          -6: "SDPA_ERR_CAPACITY", -7: "SDPA_ERR_DEVICE_INDEX"}

# Every symbol include/sdpa.h declares.
EXPORTS = ("sdpa_fwd", "sdpa_fwd_ex", "sdpa_fwd_strided", "sdpa_merge", "sdpa_select_path", "sdpa_fwd_host",
           "sdpa_fwd_split_kv_static", "sdpa_last_device_error", "sdpa_debug_checks", "sdpa_selftest_wait_timeout",
           "sdpa_selftest_index_check", "sdpa_strerror", "sdpa_version")


class SdpaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}" if what else STATUS.get(status, str(status)))


class sdpa_mask_t(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_int64), ("window", ctypes.c_int64), ("data", ctypes.c_void_p),
                ("stride_b", ctypes.c_int64), ("stride_h", ctypes.c_int64), ("stride_q", ctypes.c_int64)]


class sdpa_strides_t(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("t", ctypes.c_int64)]


_lib = None
_vp, _i32, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_COMMON = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32]


def lib():
    """The loaded ``libsdpa.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            flag = " --debug" if LIB_PATH == DEBUG_LIB_PATH else ""
            raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                              f"`python -m attention_sdpa_fwd_b200.build{flag}`")
        L = ctypes.CDLL(LIB_PATH)
        L.sdpa_fwd.argtypes = _COMMON + [_f32, _i32, _vp, _vp, _vp, _vp, _vp, _vp]
        L.sdpa_fwd_ex.argtypes = _COMMON + [_f32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp]
        L.sdpa_fwd_host.argtypes = _COMMON + [_f32, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp]
        L.sdpa_merge.argtypes = [_vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp]
        L.sdpa_fwd_strided.argtypes = [_vp] * 8 + [_i32] * 7 + [_f32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp]
        L.sdpa_select_path.argtypes = _COMMON + [_i32, _vp, _vp, _vp, _vp, _vp]
        L.sdpa_fwd_split_kv_static.argtypes = _COMMON + [_f32, _i32, _vp, _vp, _vp]
        L.sdpa_last_device_error.argtypes = [_vp]
        L.sdpa_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, _vp]
        L.sdpa_selftest_index_check.argtypes = [ctypes.c_longlong, ctypes.c_longlong, _vp]
        L.sdpa_debug_checks.argtypes = []
        L.sdpa_strerror.argtypes = [_i32]
        L.sdpa_strerror.restype = ctypes.c_char_p
        for name in ("sdpa_fwd", "sdpa_fwd_ex", "sdpa_fwd_strided", "sdpa_merge", "sdpa_fwd_host", "sdpa_select_path",
                     "sdpa_fwd_split_kv_static", "sdpa_last_device_error", "sdpa_selftest_wait_timeout",
                     "sdpa_selftest_index_check", "sdpa_debug_checks", "sdpa_version"):
            getattr(L, name).restype = _i32
        _lib = L
    return _lib


# ---------------------------------------------------------------------------
# Raw C-ABI calls (same names as the C functions; pointers are ints)
# ---------------------------------------------------------------------------
def _hw(x):
    return None if x is None else (ctypes.c_int * 2)(int(x[0]), int(x[1]))


def sdpa_fwd(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
             rel_pos_h, rel_pos_w, q_hw, k_hw, stream) -> int:
    return lib().sdpa_fwd(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                          rel_pos_h, rel_pos_w, _hw(q_hw), _hw(k_hw), stream)


def sdpa_fwd_ex(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                rel_pos_h, rel_pos_w, q_hw, k_hw, lse, path, stream) -> int:
    return lib().sdpa_fwd_ex(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                             rel_pos_h, rel_pos_w, _hw(q_hw), _hw(k_hw), lse, path, stream)


def sdpa_fwd_strided(q, q_strides, k, k_strides, v, v_strides, out, out_strides, dtype, B, Hq, Hkv, Tq, Tkv,
                     d, scale, mask_kind, mask_ptr, rel_pos_h, rel_pos_w, q_hw, k_hw, lse, path, stream) -> int:
    st = lambda x: None if x is None else ctypes.byref(sdpa_strides_t(*(int(y) for y in x)))
    return lib().sdpa_fwd_strided(q, st(q_strides), k, st(k_strides), v, st(v_strides), out, st(out_strides),
                                  dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr, rel_pos_h, rel_pos_w,
                                  _hw(q_hw), _hw(k_hw), lse, path, stream)


def sdpa_merge(outs, lses, nparts, out, lse, dtype, B, Hq, Tq, d, stream) -> int:
    """outs / lses: sequences of device pointers (ints)."""
    po = (ctypes.c_void_p * len(outs))(*outs)
    pl = (ctypes.c_void_p * len(lses))(*lses)
    return lib().sdpa_merge(po, pl, nparts, out, lse, dtype, B, Hq, Tq, d, stream)


def sdpa_fwd_host(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                  rel_pos_h, rel_pos_w, q_hw, k_hw, path, stream) -> int:
    return lib().sdpa_fwd_host(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                               rel_pos_h, rel_pos_w, _hw(q_hw), _hw(k_hw), path, stream)


def sdpa_select_path(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, mask_kind, mask_ptr,
                     rel_pos_h, rel_pos_w, q_hw, k_hw) -> int:
    return lib().sdpa_select_path(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, mask_kind, mask_ptr,
                                  rel_pos_h, rel_pos_w, _hw(q_hw), _hw(k_hw))


def sdpa_fwd_split_kv_static(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind, mask_ptr,
                             lse, stream) -> int:
    return lib().sdpa_fwd_split_kv_static(q, k, v, out, dtype, B, Hq, Hkv, Tq, Tkv, d, scale, mask_kind,
                                          mask_ptr, lse, stream)


def sdpa_last_device_error(stream) -> int:
    return lib().sdpa_last_device_error(stream)


def sdpa_selftest_wait_timeout(limit_ns, stream) -> int:
    return lib().sdpa_selftest_wait_timeout(limit_ns, stream)


def sdpa_strerror(status: int) -> str:
    return lib().sdpa_strerror(status).decode()


def sdpa_selftest_index_check(index, extent, stream) -> int:
    return lib().sdpa_selftest_index_check(index, extent, stream)


def sdpa_debug_checks() -> int:
    return lib().sdpa_debug_checks()


def sdpa_version() -> int:
    return lib().sdpa_version()


# ---------------------------------------------------------------------------
# Tensor-level convenience wrapper (marshalling only)
# ---------------------------------------------------------------------------
def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return SDPA_F32
    if t.dtype == torch.bfloat16:
        return SDPA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def make_mask(kind: int, *, offset: int = 0, window: int = 0, tensor=None) -> Optional[sdpa_mask_t]:
    """Build the host mask descriptor.  ``tensor`` (ADD_FLOAT / BOOL) must be a
    CUDA tensor of 4 dims [B|1, Hq|1, Tq, Tkv] with a contiguous key axis;
    size-1 batch / head axes broadcast (stride 0)."""
    if kind == MASK_NONE:
        return None
    m = sdpa_mask_t(offset=int(offset), window=int(window), data=None, stride_b=0, stride_h=0, stride_q=0)
    if kind in (MASK_FLOAT, MASK_BOOL):
        t = tensor
        if t is None or t.dim() != 4 or t.stride(3) != 1:
            raise ValueError("mask tensor must be 4-D with a contiguous last axis")
        m.data = t.data_ptr()
        m.stride_b = 0 if t.shape[0] == 1 else t.stride(0)
        m.stride_h = 0 if t.shape[1] == 1 else t.stride(1)
        m.stride_q = t.stride(2)
    return m


def sdpa(q, k, v, scale: Optional[float] = None, *, mask_kind: int = MASK_NONE, offset: int = 0,
         window: int = 0, mask=None, rel_pos_h=None, rel_pos_w=None,
         q_hw: Optional[Sequence[int]] = None, k_hw: Optional[Sequence[int]] = None,
         out=None, lse=None, path: str = "auto", stream=None):
    """softmax(q.k^T*scale + bias).v on CUDA tensors indexed [B, H, T, d].

    q [B,Hq,Tq,d], k/v [B,Hkv,Tkv,d], float32 or bfloat16, with a contiguous
    last axis and any batch / head / token strides: a "bshd" tensor [B,T,H,d]
    passed as x.transpose(1, 2) is used in place (sdpa_fwd_strided), dense
    bhsd tensors go through sdpa_fwd_ex.  ``out`` (allocated bhsd when None)
    may be strided the same way.  ``scale`` defaults to 1/sqrt(d) (Axon PR,
    :scale option).  Returns ``out``."""
    import torch
    for t in (q, k, v):
        if not t.is_cuda:
            raise ValueError("sdpa runs on CUDA tensors only (no CPU fallback)")
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError("q, k, v must be 4-D [B, H, T, d] with a contiguous last axis")
    B, Hq, Tq, d = q.shape
    Hkv, Tkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, Tq, d), device=q.device, dtype=q.dtype)
    elif out.dim() != 4 or out.stride(3) != 1:
        raise ValueError("out must be 4-D with a contiguous last axis")
    m = make_mask(mask_kind, offset=offset, window=window, tensor=mask)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    mp = ctypes.byref(m) if m is not None else None
    with torch.cuda.device(q.device):
        if all(t.is_contiguous() for t in (q, k, v, out)):
            rc = sdpa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), B, Hq, Hkv, Tq, Tkv, d,
                             float(scale), mask_kind, mp, _ptr(rel_pos_h), _ptr(rel_pos_w), q_hw, k_hw,
                             _ptr(lse), PATHS[path], st.cuda_stream)
            what = "sdpa_fwd_ex"
        else:
            s3 = lambda t: (t.stride(0), t.stride(1), t.stride(2))
            rc = sdpa_fwd_strided(_ptr(q), s3(q), _ptr(k), s3(k), _ptr(v), s3(v), _ptr(out), s3(out),
                                  _dtype_code(q), B, Hq, Hkv, Tq, Tkv, d, float(scale), mask_kind, mp,
                                  _ptr(rel_pos_h), _ptr(rel_pos_w), q_hw, k_hw, _ptr(lse), PATHS[path],
                                  st.cuda_stream)
            what = "sdpa_fwd_strided"
    if rc != 0:
        raise SdpaError(rc, what)
    return out


def merge(outs, lses, out=None, lse=None, stream=None):
    """Combine attention results over disjoint key subsets (sdpa_merge).

    outs: sequence of [B, Hq, Tq, d] CUDA tensors (dense, same dtype); lses:
    matching [B, Hq, Tq] float32 tensors as written by ``sdpa(..., lse=)``.
    Returns (out, lse); ``out`` may be ``outs[0]`` (in place)."""
    import torch
    o0 = outs[0]
    for t in list(outs) + list(lses):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("merge takes dense CUDA tensors only")
    B, Hq, Tq, d = o0.shape
    if out is None:
        out = torch.empty_like(o0)
    if lse is None:
        lse = torch.empty((B, Hq, Tq), device=o0.device, dtype=torch.float32)
    st = stream if stream is not None else torch.cuda.current_stream(o0.device)
    with torch.cuda.device(o0.device):
        rc = sdpa_merge([t.data_ptr() for t in outs], [t.data_ptr() for t in lses], len(outs), out.data_ptr(),
                        lse.data_ptr(), _dtype_code(o0), B, Hq, Tq, d, st.cuda_stream)
    if rc != 0:
        raise SdpaError(rc, "sdpa_merge")
    return out, lse
