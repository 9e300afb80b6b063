"""The FMA-pipe 2^x that the e4m3 forward pass uses for an eighth of its exponentials.

CPU: the constants in ptx.cuh are the float32 Remez fit that fit_exp2_poly.py makes,
and the range reduction + polynomial, restated in float32 numpy, meets the fit's
relative error bound. GPU: the device function itself, on a dense sweep of arguments,
against 2^x in double precision.
"""

import ctypes
import os
import re
import shutil
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "tiled_attention_19_b200", "csrc")
BOUND = 3.0e-6  # float32 Horner error of the degree-4 fit (2.7e-6) plus the final product


def _kernel_constants():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = src[src.index("void ex2_fma2("):]
    body = body[: body.index("\n}\n")]
    return np.array([float(re.search(r"kC%d = ([0-9.eE+-]+)f" % k, body).group(1)) for k in range(5)],
                    dtype=np.float32)


def _fit():
    sys.path.insert(0, CSRC)
    try:
        import fit_exp2_poly
    finally:
        sys.path.remove(CSRC)
    return fit_exp2_poly.fit(4)


def _sweep():
    x = np.concatenate([
        np.linspace(-140.0, 10.0, 300001),
        np.arange(-127, 11, dtype=np.float64) + 0.5,  # halfway cases of round-to-nearest
        np.arange(-127, 11, dtype=np.float64),
        [-np.inf, -1e30, -128.0, 0.0, -0.0],
    ]).astype(np.float32)
    return x


def _check(x, y):
    x64 = x.astype(np.float64)
    want = np.exp2(x64)
    normal = x64 >= -125.0
    rel = np.abs(y[normal].astype(np.float64) / want[normal] - 1.0)
    assert rel.max() <= BOUND, (rel.max(), x[normal][np.argmax(rel)])
    # below the normal range the result is flushed: 0 at or below -127, never above 2^-125
    tiny = ~normal
    assert np.all(y[tiny] >= 0.0) and np.all(y[tiny] <= 2.0 ** -125)
    assert np.all(y[x64 <= -127.5] == 0.0)
    assert y[np.isneginf(x64)][0] == 0.0


def test_constants_are_the_remez_fit():
    c32, err, err32 = _fit()
    np.testing.assert_array_equal(_kernel_constants(), c32)
    assert err < 2.7e-6 and err32 < 2.8e-6


def test_fit_equioscillates():
    # a minimax fit of degree 4 touches its error bound with alternating sign at 6 points
    c32, err, _ = _fit()
    g = np.linspace(-0.5, 0.5, 20001)
    e = np.polynomial.polynomial.polyval(g, c32.astype(np.float64)) / 2.0 ** g - 1.0
    peaks = np.abs(e) > 0.9 * np.abs(e).max()
    signs = np.sign(e[peaks])
    changes = np.count_nonzero(np.diff(signs))
    assert changes >= 5


def test_float32_restatement_meets_bound():
    c = _kernel_constants()
    x = _sweep()
    xc = np.maximum(x, np.float32(-127.0))
    r = np.float32(12582912.0)
    t = (xc + r).astype(np.float32)
    f = (xc - (t - r)).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    p = np.full_like(f, c[4])
    for k in (3, 2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = t.view(np.uint32).astype(np.uint64)
    s = (((bits << np.uint64(23)) + np.uint64(0x3F800000)) & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    with np.errstate(under="ignore"):
        y = (p * s).astype(np.float32)
    _check(x, y)


@pytest.mark.gpu
def test_device_ex2_fma2(tmp_path):
    so = str(tmp_path / "ex2_check.so")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    cmd = [nvcc, "-std=c++17", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
           "-Xcompiler", "-fPIC", "-I", CSRC, "-o", so, os.path.join(ROOT, "tests", "kernels", "ex2_check.cu")]
    subprocess.run(cmd, check=True, capture_output=True)
    lib = ctypes.CDLL(so)
    lib.ex2_fma2_eval.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.ex2_fma2_eval.restype = ctypes.c_int
    x = _sweep()
    y = np.zeros_like(x)
    assert lib.ex2_fma2_eval(x.ctypes.data, y.ctypes.data, x.size) == 0
    _check(x, y)
