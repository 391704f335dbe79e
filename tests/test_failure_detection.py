"""Failure detection without a fault: every tensor-core kernel bounds its
mbarrier waits by %globaltimer and reports an expired wait through the device
error word (sdpa_last_device_error -> SDPA_ERR_TIMEOUT).  The self-test entry
point makes one such wait run out on an mbarrier nothing arrives on; the
context must stay usable and the next forward call must be correct."""
import pytest
import torch

import attention_sdpa_fwd_b200 as S
from attention_sdpa_fwd_b200 import build

TIMEOUT = -5


def test_selftest_rejects_bad_limits_before_launch():
    build.build()
    assert S.sdpa_selftest_wait_timeout(0, None) == -1
    assert S.sdpa_selftest_wait_timeout(3_000_000_000, None) == -1


@pytest.mark.gpu
def test_expired_wait_reports_timeout_and_context_survives():
    from attention_sdpa_fwd_b200 import workloads as W
    from helpers import assert_gates, gpu_run, oracle_ref
    stream = torch.cuda.current_stream().cuda_stream
    assert S.sdpa_last_device_error(stream) == 0          # nothing pending
    assert S.sdpa_selftest_wait_timeout(1_000_000, stream) == 0  # 1 ms
    assert S.sdpa_last_device_error(stream) == TIMEOUT
    assert S.sdpa_last_device_error(stream) == 0          # the word was cleared
    # a forward call on the tensor-core path right after is still correct
    sp = W.Spec("after_timeout", torch.bfloat16, 1, 2, 2, 240, 240, 64, 0.125, seed=93,
                q_hw=(15, 16), k_hw=(15, 16), rel_std=0.5)
    wl = W.make(sp)
    out, _ = gpu_run(wl, path="tcgen05")
    assert_gates(out.double().numpy(), oracle_ref(wl).out, sp.dtype, "forward after an expired wait")
    # and twice in a row on a split-KV problem, whose scratch was marked for clearing
    sp2 = W.Spec("after_timeout_split", torch.bfloat16, 2, 2, 2, 8, 3000, 16, 0.25, seed=94)
    assert S.sdpa_selftest_wait_timeout(500_000, stream) == 0
    assert S.sdpa_last_device_error(stream) == TIMEOUT
    wl2 = W.make(sp2)
    out2, _ = gpu_run(wl2, path="split_kv")
    assert_gates(out2.double().numpy(), oracle_ref(wl2).out, sp2.dtype, "split-KV after an expired wait")
