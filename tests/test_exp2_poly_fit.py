"""The polynomial behind the softmax's FMA-pipe exponential (no GPU).

The constants compiled into csrc/exp2_poly.cuh must be what the Remez fit
in exp2_poly_fit.py produces, and that fit must be the minimax one: by the
Chebyshev alternation theorem a degree-3 polynomial is the best relative
approximation of 2^f on [-1/2, 1/2] exactly when its relative error takes
its maximum magnitude at 5 points with alternating signs."""
import os
import re

import numpy as np

from pretraining_step_b200 import exp2_poly_fit

HDR = os.path.join(os.path.dirname(exp2_poly_fit.__file__), "csrc", "exp2_poly.cuh")


def _header_coefficients():
    src = open(HDR).read()
    return [float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f;" % k, src).group(1)) for k in range(4)]


def test_header_holds_the_fitted_coefficients():
    c, _ = exp2_poly_fit.fit(3)
    assert np.array_equal(np.float32(c), np.float32(_header_coefficients()))


def test_fit_equioscillates():
    c, emax = exp2_poly_fit.fit(3)
    g = np.linspace(-0.5, 0.5, 400001)
    err = exp2_poly_fit.rel_error(c, g)
    # Extremum of each run of constant sign.
    ext, start, sign = [], 0, np.sign(err)
    for j in range(1, g.size):
        if sign[j] != sign[j - 1]:
            ext.append(start + int(np.argmax(np.abs(err[start:j]))))
            start = j
    ext.append(start + int(np.argmax(np.abs(err[start:]))))
    e = err[ext]
    assert len(e) == 5
    assert np.all(np.sign(e[1:]) == -np.sign(e[:-1]))
    assert np.max(np.abs(e)) - np.min(np.abs(e)) < 1e-3 * emax
    # Both interval ends are reference points (2^f is smooth and monotone).
    assert ext[0] == 0 and ext[-1] == g.size - 1


def test_error_of_the_compiled_coefficients():
    """fp32-rounded coefficients evaluated in fp64: within 7.5e-5 relative,
    a twenty-sixth of bf16's half unit; a degree-2 fit would not be
    (1.7e-3, close to that half unit)."""
    g = np.linspace(-0.5, 0.5, 200001)
    assert np.max(np.abs(exp2_poly_fit.rel_error(np.float64(_header_coefficients()), g))) < 7.5e-5
    _, e2 = exp2_poly_fit.fit(2)
    assert e2 > 1e-3
