"""The bounded wait of the decode pipeline gives up instead of hanging.

A test kernel (tests/csrc/wait_timeout.cu) waits, through the library's own
mbar_wait_bounded, on an mbarrier that nothing ever completes.  The wait must
stop after its cycle limit (about a second), set PA_FLAG_TIMEOUT in the
caller's flag and return false; the kernel then ends and the context stays
usable.  Nothing is faulted, trapped or hung.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from tests.conftest import ROOT

SRC = os.path.join(ROOT, "tests", "csrc", "wait_timeout.cu")


def _compile(out_path):
    from paged_kv_cache_349_b200 import build as B
    subprocess.check_call([B._nvcc(), *B.ARCH, "-O3", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler",
                           "-fPIC", "-shared", "-cudart", "static", "-I", B.INCLUDE, "-o", str(out_path), SRC])


def test_timeout_kernel_builds(tmp_path):
    """The test kernel compiles for sm_100a against the library's device header (no GPU needed)."""
    out = tmp_path / "libwait_timeout.so"
    _compile(out)
    assert out.stat().st_size > 0


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives(tmp_path):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_cache_349_b200 as pa
    import workloads as W
    out = tmp_path / "libwait_timeout.so"
    _compile(out)
    lib = ctypes.CDLL(str(out))
    lib.run_wait_timeout.restype = ctypes.c_int
    lib.run_wait_timeout.argtypes = [ctypes.c_void_p] * 3 + [ctypes.POINTER(ctypes.c_longlong)]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    cycles = torch.zeros(1, dtype=torch.int64, device="cuda")
    limit = ctypes.c_longlong()
    assert lib.run_wait_timeout(ctypes.c_void_p(flag.data_ptr()), ctypes.c_void_p(result.data_ptr()),
                                ctypes.c_void_p(cycles.data_ptr()), ctypes.byref(limit)) == 0
    torch.cuda.synchronize()
    assert int(result.item()) == 0                      # the wait reported failure
    assert int(flag.item()) == pa.PA_FLAG_TIMEOUT       # and said why
    assert limit.value <= int(cycles.item()) < 2 * limit.value + 10_000_000  # after the limit, not much later

    # The context is still usable: a small decode runs and is correct.
    case = W.make_case(1)
    from tests.gpu_helpers import DeviceCase, run_step, assert_close
    import oracle
    dc = DeviceCase(case)
    got = run_step(dc)
    assert int(dc.flag.item()) == 0
    want, _, _ = oracle.decode_step(case)
    assert_close(got, want, "decode after a timed-out wait")
