"""The FMA-pipe exponential's coefficients are reproducible from their fit.

The one-tile query x summary kernel evaluates part of its softmax
exponentials as x = n + f, 2^n by the exponent field and 2^f by a cubic.  The
cubic's float32 coefficients in csrc/common.cuh must be the ones the Remez
exchange in fit_exp2.py produces, and that fit's relative error must be the
bound the library states (7.5e-5).  The device evaluation is checked against
a float64 reference in tests/test_gpu_parity.py.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_cubic_coefficients_come_from_the_fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(ROOT, "geometry_aware_local_b200",
                                                                           "fit_exp2.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    coeffs, err = mod.check()
    src = open(os.path.join(ROOT, "geometry_aware_local_b200", "csrc", "common.cuh")).read()
    m = re.search(r"kC0 = ([0-9.e+-]+)f, kC1 = ([0-9.e+-]+)f, kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f", src)
    assert m, "exp2_fma coefficients not found"
    in_source = np.array([float(v) for v in m.groups()], dtype=np.float32)
    assert np.array_equal(in_source, coeffs), (in_source, coeffs)
    assert err <= 7.5e-5
    # the equioscillation of a minimax fit: the error reaches its bound at both ends of [-1/2, 1/2]
    f = np.array([-0.5, 0.5], dtype=np.float64)
    p = np.polyval(coeffs.astype(np.float64)[::-1], f)
    assert np.all(np.abs(p / np.exp2(f) - 1) > 0.9 * err)
