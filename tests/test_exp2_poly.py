"""The FMA-pipe 2^x used for part of the prefill softmax (csrc/pod_exp2.cuh),
compiled for the host from the same header, against float64 exp2 (no GPU)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "hybrid_prefill_decode_pod_b200", "csrc")
WRAP = r'''
#include "pod_exp2.cuh"
extern "C" void eval_exp2(const float* x, float* y, long n) {
  for (long i = 0; i < n; ++i) y[i] = pod::exp2_poly(x[i]);
}
'''


@pytest.fixture(scope="module")
def exp2_lib(tmp_path_factory):
    d = tmp_path_factory.mktemp("exp2")
    src = d / "w.cpp"
    src.write_text(WRAP)
    so = d / "w.so"
    subprocess.check_call(["g++", "-O2", "-ffp-contract=off", "-shared", "-fPIC", "-I", CSRC,
                           "-o", str(so), str(src)])
    lib = ctypes.CDLL(str(so))
    lib.eval_exp2.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long]
    return lib


def _eval(lib, x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    lib.eval_exp2(x.ctypes.data, y.ctypes.data, x.size)
    return y


def test_relative_error_bound(exp2_lib):
    g = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001, dtype=np.float32),
                        g.uniform(-30.0, 8.0, 200000).astype(np.float32),
                        np.arange(-125, 9, dtype=np.float32)])
    y = _eval(exp2_lib, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    # fitted polynomial error 7.5e-5 plus a few fp32 roundings
    assert rel.max() < 8.0e-5, rel.max()


def test_clamped_below_and_monotone_on_grid(exp2_lib):
    y = _eval(exp2_lib, np.array([-1e30, -400.0, -125.0], np.float32))
    assert np.all(y > 0) and np.all(np.isfinite(y))
    assert np.allclose(y, 2.0 ** -125, rtol=1e-4)
    x = np.linspace(-20, 8, 100001, dtype=np.float32)
    y = _eval(exp2_lib, x)
    # not strictly monotone at segment joins, but never off by more than the error bound
    assert np.all(np.diff(y) > -2e-4 * y[1:])


def test_coefficients_match_generator():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    c, worst = m.fit()
    text = open(os.path.join(CSRC, "pod_exp2.cuh")).read()
    for i, v in enumerate(c):
        assert ("kExp2C%d = %.9ef" % (i, v)) in text
    assert worst < 7.6e-5
