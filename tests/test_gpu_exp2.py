"""The attention kernel's FMA-pipe exp2 (our own cubic, see
rolling_kv_cache_rope_b200/csrc/fit_exp2_poly.py) against CUDA's exp2f and
float64: relative error below 1e-4 over the range the softmax uses, about
2^-126 (never negative, NaN or inf) below it."""

import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from tests._gpu import need_gpu

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def check_lib(tmp_path_factory):
    need_gpu()
    out = tmp_path_factory.mktemp("exp2") / "libexp2check.so"
    nvcc = os.environ.get("NVCC", "nvcc")
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared", "-Xcompiler",
                           "-fPIC", "-I", os.path.join(ROOT, "rolling_kv_cache_rope_b200", "csrc"),
                           os.path.join(ROOT, "tests", "kernels", "exp2_check.cu"), "-o", str(out)])
    lib = ctypes.CDLL(str(out))
    lib.exp2_check.restype = ctypes.c_int
    lib.exp2_check.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return lib


def run(lib, x):
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    a, r = torch.empty_like(xd), torch.empty_like(xd)
    assert lib.exp2_check(xd.data_ptr(), a.data_ptr(), r.data_ptr(), xd.numel()) == 0
    return a.cpu().numpy().astype(np.float64), r.cpu().numpy().astype(np.float64)


def test_relative_error_in_softmax_range(check_lib):
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-120.0, 20.0, 1 << 20), rng.uniform(-30.0, 8.0, 1 << 20),
                        np.arange(-120, 21, dtype=np.float64) + 0.5, np.arange(-120, 21, dtype=np.float64)])
    x = x[: (x.size // 2) * 2].astype(np.float32)
    approx, ref = run(check_lib, x)
    exact = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(approx / exact - 1.0)) < 1e-4
    assert np.max(np.abs(approx / ref - 1.0)) < 1e-4


def test_underflow_side_is_tiny_and_nonnegative(check_lib):
    x = np.concatenate([np.linspace(-140.0, -120.0, 4096), np.array([-np.float32(3e38), -1e30, -126.0, -126.5])])
    x = x[: (x.size // 2) * 2].astype(np.float32)
    approx, _ = run(check_lib, x)
    assert np.all(np.isfinite(approx)) and np.all(approx >= 0.0)
    assert np.all(approx[x < -126.0] <= 2.0 ** -125)
