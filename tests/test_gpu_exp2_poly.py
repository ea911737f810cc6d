"""Accuracy of the polynomial exp2 the prefill softmax evaluates on the FMA
pipe for part of its exponentials (csrc/ptx.cuh, exp2_poly2).

GPU: a small harness compiled here with nvcc evaluates it on a device array;
the values are compared with exact powers of two (float64).  The bound is the
minimax relative error of the fitted cubic (1.014e-4 in float32 evaluation).
CPU: the coefficients in the header are the ones the fit script produces.
"""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest
import torch

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(REPO, "full_gqa_attention_swa_b200", "csrc")
REL_BOUND = 1.1e-4


def test_header_coefficients_match_fit():
    out = subprocess.run([sys.executable, os.path.join(REPO, "tests", "exp2_poly_fit.py")], capture_output=True, text=True,
                         check=True).stdout
    fitted = [float(v) for v in re.findall(r"c\d = ([-0-9.e+]+)f", out)]
    assert len(fitted) == 3
    header = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = header[header.index("exp2_poly2(uint64_t y)"):]
    body = body[:body.index("\n}\n")]
    for c in fitted:
        assert ("%.9ef" % c) in body, c
    err = float(re.search(r"float32 evaluation: ([0-9.e+-]+)", out).group(1))
    assert err < REL_BOUND


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("exp2") / "exp2_check.so")
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared", "-Xcompiler",
           "-fPIC", "-I", CSRC, "-o", so, os.path.join(REPO, "tests", "gpu_kernels", "exp2_poly_check.cu")]
    subprocess.run(cmd, check=True)
    lib = ctypes.CDLL(so)
    lib.exp2_poly_eval.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.exp2_poly_eval.restype = ctypes.c_int
    return lib


def _eval(lib, dev, x):
    x = np.asarray(x, np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0))
    xd = torch.from_numpy(x).to(dev)
    yd = torch.empty_like(xd)
    assert lib.exp2_poly_eval(xd.data_ptr(), yd.data_ptr(), x.size // 2) == 0
    return x, yd.cpu().numpy()


@pytest.mark.gpu
def test_exp2_poly_relative_error(harness, cuda_device):
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-126.0, 10.0, 1 << 20, dtype=np.float32),
        rng.uniform(-126.0, 8.0, 1 << 20).astype(np.float32),
        np.arange(-126, 10, dtype=np.float32) + np.float32(0.5),  # rounding ties
        np.array([0.0, -0.0, 0.5, -0.5, 1e-30, -1e-30, 8.0], np.float32),
    ])
    x, y = _eval(harness, cuda_device, x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - exact) / exact
    assert rel.max() <= REL_BOUND, (rel.max(), x[rel.argmax()])
    assert y[x == 0].tolist() == [1.0] * int((x == 0).sum())


@pytest.mark.gpu
def test_exp2_poly_underflow_is_exact_zero(harness, cuda_device):
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -127.5, -127.0], np.float32)
    _, y = _eval(harness, cuda_device, x)
    assert (y.view(np.uint32) == 0).all(), y


@pytest.mark.gpu
def test_exp2_poly_subnormal_band(harness, cuda_device):
    # between -127 and -126 the exponent field would go to zero: the result is
    # some non-negative value below the smallest normal 2^-126 (the softmax
    # only needs it negligible next to a row sum of at least 1)
    x = np.linspace(-126.999, -126.001, 4096, dtype=np.float32)
    x, y = _eval(harness, cuda_device, x)
    assert (y >= 0).all() and (y < 2.0 ** -126).all()
