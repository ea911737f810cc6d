"""Failure detection on the GPU without a fault: the bounded mbarrier wait
that every kernel of the library uses (csrc/ptx.cuh, mbar_wait) gives up on
its time limit, or at once when another thread of the CTA raises the abort
flag, returns false, and the error word keeps the first recorded code; the
CUDA context stays usable afterwards.  A small harness compiled here with
nvcc runs the waits on a barrier that nothing ever completes."""
import ctypes
import os
import subprocess

import pytest
import torch

from full_gqa_attention_swa_b200 import api

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(REPO, "full_gqa_attention_swa_b200", "csrc")

pytestmark = pytest.mark.gpu


class _Result(ctypes.Structure):
    _fields_ = [("ok_timeout", ctypes.c_int), ("ok_abort", ctypes.c_int), ("ok_arrived", ctypes.c_int),
                ("first_code", ctypes.c_int), ("ns_timeout", ctypes.c_ulonglong), ("ns_abort", ctypes.c_ulonglong),
                ("ns_arrived", ctypes.c_ulonglong)]


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("wait") / "wait_check.so")
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared", "-Xcompiler",
           "-fPIC", "-I", CSRC, "-o", so, os.path.join(REPO, "tests", "gpu_kernels", "wait_timeout_check.cu")]
    subprocess.run(cmd, check=True)
    lib = ctypes.CDLL(so)
    lib.wait_exits_run.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_ulonglong]
    lib.wait_exits_run.restype = ctypes.c_int
    lib.wait_error_word.restype = ctypes.c_int
    return lib


def test_bounded_wait_exits(cuda_device, harness):
    limit = 50_000_000     # 50 ms time limit on the first wait
    delay = 5_000_000      # the abort / arrival come 5 ms after their cue
    r = _Result()
    assert harness.wait_exits_run(ctypes.byref(r), limit, delay) == 0
    # time limit: false, after at least the limit and well before any watchdog
    assert r.ok_timeout == 0
    assert limit <= r.ns_timeout < limit + 20_000_000
    # abort flag: false after about the delay, far below its 1 s limit
    assert r.ok_abort == 0
    assert delay <= r.ns_abort < 10 * delay
    # arrival: true
    assert r.ok_arrived == 1
    assert r.ns_arrived < 20 * limit
    # the first recorded code stays in the error word
    assert r.first_code == 9901
    assert harness.wait_error_word() == 9901
    # the context is still usable, and the library's own word is untouched
    x = torch.arange(1 << 20, device=cuda_device, dtype=torch.float32)
    assert float(x.sum().item()) == float((1 << 20) * ((1 << 20) - 1) / 2)
    assert api.device_error(reset=False) == 0
