"""The debug build (libsdpa_debug.so, compiled with SDPA_DEBUG): device-side
index checks that write the error word instead of trapping.

CPU: the debug library exports every declared symbol and reports itself as
the debug build; the release library reports 0.  GPU: the index-check
self-test sets SDPA_ERR_DEVICE_INDEX in the debug build only (no memory is
touched at the checked index), and the parity suites run green through the
debug library -- every check stays silent on every case while the results
still meet the oracle gates."""
import ctypes
import os
import subprocess
import sys

import pytest

import attention_sdpa_fwd_b200 as S
from attention_sdpa_fwd_b200 import build
from test_abi import declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def debug_lib():
    build.build(debug=True)
    L = ctypes.CDLL(build.DEBUG_LIB)
    L.sdpa_debug_checks.restype = ctypes.c_int
    return L


def test_debug_library_exports_and_flag(debug_lib):
    for n in declared_functions():
        assert hasattr(debug_lib, n), f"{n} missing from the debug build"
    assert debug_lib.sdpa_debug_checks() == 1


def test_release_library_flag():
    build.build()
    L = ctypes.CDLL(build.LIB)
    L.sdpa_debug_checks.restype = ctypes.c_int
    assert L.sdpa_debug_checks() == 0


def test_debug_status_code_named():
    assert S.STATUS[-7] == "SDPA_ERR_DEVICE_INDEX"


def _child(code: str, timeout: int = 900) -> subprocess.CompletedProcess:
    env = dict(os.environ, SDPA_DEBUG="1", PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


@pytest.mark.gpu
def test_index_selftest_debug_and_release(debug_lib):
    import torch
    # release build (this process): the check is compiled out, nothing is set
    build.build()
    st = torch.cuda.current_stream().cuda_stream
    assert S.sdpa_debug_checks() == 0
    assert S.sdpa_selftest_index_check(5, 3, st) == 0
    assert S.sdpa_last_device_error(st) == 0
    assert S.sdpa_selftest_index_check(0, -1, st) == -1  # negative extent: refused on the host
    # debug build (child process, same binding selected by SDPA_DEBUG=1)
    code = (
        "import torch, attention_sdpa_fwd_b200 as S\n"
        "assert S.LIB_PATH == S.DEBUG_LIB_PATH and S.sdpa_debug_checks() == 1\n"
        "st = torch.cuda.current_stream().cuda_stream\n"
        "assert S.sdpa_selftest_index_check(2, 3, st) == 0\n"
        "assert S.sdpa_last_device_error(st) == 0\n"
        "for i, n in ((3, 3), (5, 3), (-1, 3), (0, 0)):\n"
        "    assert S.sdpa_selftest_index_check(i, n, st) == 0\n"
        "    rc = S.sdpa_last_device_error(st)\n"
        "    assert rc == -7, (i, n, rc)\n"
        "    assert S.sdpa_last_device_error(st) == 0  # the word was cleared\n"
        "x = torch.randn(1, 2, 64, 64, device='cuda', dtype=torch.bfloat16)\n"
        "o = S.sdpa(x, x, x, 0.125)\n"
        "torch.cuda.synchronize()\n"
        "assert S.sdpa_last_device_error(st) == 0\n"
        "print('ok')\n")
    r = _child(code, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-4000:]


@pytest.mark.gpu
def test_parity_through_debug_build(debug_lib):
    """test_parity and the random sweep with SDPA_DEBUG=1: every gpu_run call
    there reads the error word, so one failed index check fails the case."""
    code = (
        "import sys, pytest, attention_sdpa_fwd_b200 as S\n"
        "assert S.LIB_PATH == S.DEBUG_LIB_PATH and S.sdpa_debug_checks() == 1\n"
        "sys.exit(pytest.main(['-q', '-x', '-m', 'gpu', '-p', 'no:cacheprovider',\n"
        "                      'tests/test_parity.py', 'tests/test_random_sweep.py', 'tests/test_strided.py']))\n")
    r = _child(code, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
