"""HyperDual number type on the device against closed-form derivatives.

f1 and f2 are the worked examples of the page "How to Implement Automatic
Differentiation Using the $autodiff Block for Custom Kernels" (section Code
Examples; tests/golden/autodiff_examples.json): the page states d/dx[x sin x]
= sin x + x cos x.  Second derivatives and f3, f4 are derived by hand.
"""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def closed_forms(a, b):
    r = np.hypot(a, b)
    f1 = [a * np.sin(a), np.sin(a) + a * np.cos(a), 0.0, 2 * np.cos(a) - a * np.sin(a), 0.0, 0.0]
    f2 = [a * np.sin(b) + b * np.cos(a), np.sin(b) - b * np.sin(a), a * np.cos(b) + np.cos(a),
          -b * np.cos(a), np.cos(b) - np.sin(a), -a * np.sin(b)]
    f3 = [r, a / r, b / r, b * b / r ** 3, -a * b / r ** 3, a * a / r ** 3]
    f4 = [a / b, 1 / b, -a / b ** 2, 0.0, -1 / b ** 2, 2 * a / b ** 3]
    return np.array([f1, f2, f3, f4])


@pytest.mark.gpu
def test_hyperdual_closed_forms():
    import hessian_assembly_b200 as mad
    pts = np.array(json.load(open(os.path.join(HERE, "golden", "autodiff_examples.json")))["points"])
    out = mad.mad_selftest_dual(pts)
    for k, (a, b) in enumerate(pts):
        ref = closed_forms(a, b)
        if a == 0.0 and b != 0.0:
            pass  # f3 defined (r = |b|)
        np.testing.assert_allclose(out[k], ref, rtol=1e-13, atol=1e-13)
    # the page's stated gradient of x sin x
    a = pts[:, 0]
    np.testing.assert_allclose(out[:, 0, 1], np.sin(a) + a * np.cos(a), rtol=1e-14, atol=1e-15)
