"""Pins for the oracle's area-preservation face term (3-DOF face, 9-variable
stencil; no GPU): hand values on the unit right triangle, central finite
differences of the energy (gradient) and of the gradient (Hessian), symmetry,
translation and rotation invariance, and the assembled version on a cloth
grid.  A planted mistake (the bilinear part of d2A dropped) must fail them."""
import numpy as np
import pytest

import mesh_inputs as mi
import oracle


def tri(seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((3, 3))


def test_area_hand_values(orc):
    # x0 = 0, x1 = e_x, x2 = e_y: A = 1/2, dA/dx1 = e_x / 2, dA/dx2 = e_y / 2
    E, g, H = orc.area_local([0, 0, 0], [1, 0, 0], [0, 1, 0], 0.4, 2.0)
    assert E == pytest.approx(0.5 * 2.0 * 0.1 ** 2 / 0.4, rel=1e-14)
    np.testing.assert_allclose(g, 0.5 * np.array([-0.5, -0.5, 0, 0.5, 0, 0, 0, 0.5, 0]),
                               atol=1e-15)
    # at the rest area the Hessian is k/A0 dA dA^T
    E0, g0, H0 = orc.area_local([0, 0, 0], [1, 0, 0], [0, 1, 0], 0.5, 2.0)
    dA = 0.5 * np.array([-1, -1, 0, 1, 0, 0, 0, 1, 0.0])
    assert E0 == 0.0
    np.testing.assert_allclose(H0, 2.0 / 0.5 * np.outer(dA, dA), atol=1e-14)


def _local(o, X, A0=0.3, k=3.0):
    return o.area_local(X[0], X[1], X[2], A0, k)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_area_fd_gradient_and_hessian(orc, seed):
    X = tri(seed)
    E, g, H = _local(orc, X)
    h = 1e-6
    gfd = np.zeros(9)
    Hfd = np.zeros((9, 9))
    for q in range(9):
        Xp = X.copy().reshape(-1)
        Xm = X.copy().reshape(-1)
        Xp[q] += h
        Xm[q] -= h
        Ep, gp, _ = _local(orc, Xp.reshape(3, 3))
        Em, gm, _ = _local(orc, Xm.reshape(3, 3))
        gfd[q] = (Ep - Em) / (2 * h)
        Hfd[q] = (gp - gm) / (2 * h)
    np.testing.assert_allclose(g, gfd, atol=1e-7 * max(1, np.abs(g).max()))
    np.testing.assert_allclose(H, Hfd, atol=1e-6 * max(1, np.abs(H).max()))
    np.testing.assert_allclose(H, H.T, atol=1e-12 * np.abs(H).max())


def test_area_translation_and_rotation(orc):
    X = tri(4)
    E, g, H = _local(orc, X)
    g3 = g.reshape(3, 3)
    np.testing.assert_allclose(g3.sum(0), 0, atol=1e-13)
    for a in range(3):
        t = np.zeros((3, 3))
        t[:, a] = 1
        np.testing.assert_allclose(H @ t.reshape(-1), 0, atol=1e-12 * np.abs(H).max())
    # rotation generator W: d/dtheta of g(R x) = W g  ->  H (W x) = W g
    for axis in range(3):
        W = np.zeros((3, 3))
        b, c = [q for q in range(3) if q != axis]
        W[b, c], W[c, b] = -1, 1
        np.testing.assert_allclose(H @ (X @ W.T).reshape(-1), (g3 @ W.T).reshape(-1),
                                   atol=1e-11 * np.abs(H).max())
    # energy is rotation invariant
    th = 0.7
    R = np.array([[np.cos(th), -np.sin(th), 0], [np.sin(th), np.cos(th), 0], [0, 0, 1]])
    assert _local(orc, X @ R.T)[0] == pytest.approx(E, rel=1e-12)


def test_area_assembled_on_cloth_fd(orc):
    n = 4
    st = mi.cloth_static(n, np.float64)
    x = mi.cloth_x(n, 21, 0, np.float64) + 0.05 * np.random.default_rng(5).standard_normal((n * n, 3))
    F = st["F"]
    A0 = 0.5 * np.linalg.norm(np.cross(st["X"][F[:, 1]] - st["X"][F[:, 0]],
                                        st["X"][F[:, 2]] - st["X"][F[:, 0]]), axis=1)
    rp, ci = orc.pattern(st["V"], F)

    def ev(xx):
        return orc.eval(st["V"], 3, xx, 16, rp, ci, F=F, area=A0, ka=5.0)

    g, H, E = ev(x)
    h = 1e-6
    V = st["V"]
    D = np.zeros((3 * V, 3 * V))
    for i in range(V):
        for q in range(rp[i], rp[i + 1]):
            D[3 * i:3 * i + 3, 3 * ci[q]:3 * ci[q] + 3] = H[q]
    xf = x.reshape(-1)
    for c in (0, 7, 20, 3 * V - 1):
        xp = xf.copy()
        xm = xf.copy()
        xp[c] += h
        xm[c] -= h
        gp, _, Ep = ev(xp.reshape(-1, 3))
        gm, _, Em = ev(xm.reshape(-1, 3))
        assert g.reshape(-1)[c] == pytest.approx((Ep - Em) / (2 * h), abs=1e-6)
        np.testing.assert_allclose(D[:, c], (gp - gm).reshape(-1) / (2 * h), atol=1e-5)
    np.testing.assert_allclose(D, D.T, atol=1e-12 * np.abs(D).max())


def _area_pins_pass(o):
    try:
        test_area_hand_values(o)
        test_area_fd_gradient_and_hessian(o, 1)
        test_area_translation_and_rotation(o)
    except AssertionError:
        return False
    return True


def test_area_pins_pass_on_oracle(orc):
    assert _area_pins_pass(orc)


def test_area_pins_catch_planted_mistake():
    assert not _area_pins_pass(oracle.load_mutant(7))
