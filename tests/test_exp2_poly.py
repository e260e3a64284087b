"""The FMA-pipe 2^x used by the attention kernels' softmax passes: its
constants are the minimax fit that fit_exp2_poly.py derives, and their fp32
evaluation (range reduction, Horner, exponent add) stays within the stated
relative error over the softmax's input range."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "segmented_fine_tuning_b200", "csrc")


def _header_constants():
    text = open(os.path.join(CSRC, "hga_ptx.cuh")).read()
    found = dict(re.findall(r"kExp2C(\d) = (0x[0-9a-fA-F.p+-]+)f", text))
    return [np.float32(float.fromhex(found[str(k)])) for k in range(4)]


def _fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.fit()


def _fma32(a, b, c):
    # a*b is exact in fp64 for fp32 inputs; one rounding to fp32 after the add
    return (a.astype(np.float64) * b + c).astype(np.float32)


def _exp2_poly(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = _fma32(np.full_like(f, c[3]), f, c[2])
    p = _fma32(p, f, c[1])
    p = _fma32(p, f, c[0])
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(
        0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_constants_are_the_fit():
    c_fit, err = _fit()
    c_hdr = _header_constants()
    assert err < 7.6e-5
    for a, b in zip(c_hdr, c_fit):
        assert abs(float(a) - b) <= 2e-7 * abs(b)


def test_fp32_evaluation_error_bound():
    c = _header_constants()
    x = np.linspace(-125.0, 12.0, 1_370_001, dtype=np.float32)
    y = _exp2_poly(x, c)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.0e-4
    # integers come out within the polynomial's error at f = 0
    xi = np.arange(-125, 13, dtype=np.float32)
    assert np.all(np.abs(_exp2_poly(xi, c) / np.exp2(xi.astype(np.float64)) - 1) < 8e-5)


def test_clamped_tail_is_tiny_and_positive():
    c = _header_constants()
    x = np.array([-np.inf, -1e30, -1000.0, -126.5, -126.0], dtype=np.float32)
    y = _exp2_poly(x, c)
    assert np.all(y > 0) and np.all(y < 2e-38)
