"""The allocation-free split-KV entry point.

Some callers cannot let the library allocate device memory during a call
(for instance code running inside a memory pool it does not own);
sdpa_fwd_split_kv_static serves them from a fixed-size scratch array inside
the library.  This file runs last so that, should it fail, a run that stops
at the first failure has run every other test already.  It passes alone in a
fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from helpers import GATES, assert_gates, stats

pytestmark = pytest.mark.gpu


def _inputs(B, H, Tq, Tkv, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16).cuda()
    return mk(B, H, Tq, 16), mk(B, H, Tkv, 16), mk(B, H, Tkv, 16)


def _static_call(S, q, k, v, out, lse, scale, mask_kind=0, mask=None):
    B, H, Tq, d = q.shape
    Tkv = k.shape[2]
    m = S.make_mask(mask_kind, tensor=mask) if mask_kind else None
    return S.sdpa_fwd_split_kv_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), S.SDPA_BF16,
                                      B, H, H, Tq, Tkv, d, scale, mask_kind,
                                      ctypes.byref(m) if m is not None else None,
                                      lse.data_ptr() if lse is not None else None,
                                      torch.cuda.current_stream().cuda_stream)


def test_static_scratch_entry_matches_split_kv_and_oracle_twice():
    """Two calls in a row (the second reuses the scratch the first one left
    behind): each agrees with the regular split-KV entry point and with the
    fp64 oracle, within the bf16 gates; lse within 2e-3 of the oracle's."""
    import attention_sdpa_fwd_b200 as S
    q, k, v = _inputs(4, 8, 8, 4096, seed=11)
    ref_lse = torch.empty(4, 8, 8, device="cuda")
    ref = S.sdpa(q, k, v, 0.25, lse=ref_lse, path="split_kv")
    torch.cuda.synchronize()
    orc = oracle.sdpa(q.cpu(), k.cpu(), v.cpu(), 0.25)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.empty_like(ref_lse)
        assert _static_call(S, q, k, v, out, lse, 0.25) == 0
        torch.cuda.synchronize()
        assert S.sdpa_last_device_error(torch.cuda.current_stream().cuda_stream) == 0
        got = out.double().cpu().numpy()
        s = stats(got, ref.double().cpu().numpy())
        assert all(s[key] <= GATES[torch.bfloat16][key] for key in GATES[torch.bfloat16]), (call, s)
        assert torch.allclose(lse, ref_lse, atol=1e-3, rtol=0), call
        assert_gates(got, orc.out, torch.bfloat16, f"static entry vs oracle, call {call}")
        assert np.max(np.abs(lse.double().cpu().numpy() - orc.lse)) < 2e-3, call


def test_static_scratch_entry_with_mask_and_a_new_shape():
    import attention_sdpa_fwd_b200 as S
    q, k, v = _inputs(2, 3, 5, 1500, seed=12)
    keep = (torch.rand(2, 3, 5, 1504, generator=torch.Generator().manual_seed(3)) < 0.7).to(torch.uint8).cuda()
    keep = keep[..., :1500]
    ref = S.sdpa(q, k, v, 0.25, mask_kind=S.MASK_BOOL, mask=keep, path="split_kv")
    out = torch.empty_like(q)
    assert _static_call(S, q, k, v, out, None, 0.25, S.MASK_BOOL, keep) == 0
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    s = stats(got, ref.double().cpu().numpy())
    assert all(s[key] <= GATES[torch.bfloat16][key] for key in GATES[torch.bfloat16]), s
    orc = oracle.sdpa(q.cpu(), k.cpu(), v.cpu(), 0.25, mask_kind=S.MASK_BOOL, mask=keep.cpu())
    assert_gates(got, orc.out, torch.bfloat16, "static entry with a bool mask vs oracle")


def test_static_scratch_entry_rejects_oversized_problems():
    import attention_sdpa_fwd_b200 as S
    # 4 MiB of scratch cannot hold the partial results of 2048 (batch, head) pairs x 64 query rows
    q, k, v = _inputs(64, 32, 64, 1024, seed=13)
    out = torch.empty_like(q)
    assert _static_call(S, q, k, v, out, None, 0.25) == -6  # SDPA_ERR_CAPACITY
    # head_dim 64 is not a split-KV shape
    q64 = torch.zeros(1, 1, 4, 64, device="cuda", dtype=torch.bfloat16)
    assert _static_call(S, q64, q64, q64, torch.empty_like(q64), None, 0.1) == -2
