"""Pins for the oracle's ARAP face term (2D parameterization, no GPU).

The energy is checked against its textbook definition through numpy's SVD
(E = A sum_i (sigma_i - 1)^2 for det J > 0, i.e. A |J - U V^T|_F^2), and
against the closed forms at rotations and scaled rotations.  The gradient
and Hessian are checked by central finite differences, symmetry, and
translation / rotation invariance.  The assembled version is checked by
finite differences on a small grid.  A planted mistake (the sign of the
mixed term of the Hessian of s) must fail the pins."""
import numpy as np
import pytest

import mesh_inputs as mi
import oracle


def face(seed):
    """A random triangle in UV with a random non-degenerate Dm^-1 and det J > 0."""
    rng = np.random.default_rng(seed)
    while True:
        U = rng.standard_normal((3, 2))
        Dm = rng.standard_normal((2, 2))
        if abs(np.linalg.det(Dm)) < 0.2:
            continue
        M = np.linalg.inv(Dm)
        J = np.stack([U[1] - U[0], U[2] - U[0]], axis=1) @ M
        if np.linalg.det(J) > 0.1:
            return U, M, J


def rot(t):
    return np.array([[np.cos(t), -np.sin(t)], [np.sin(t), np.cos(t)]])


def test_arap_energy_matches_svd(orc):
    for seed in range(6):
        U, M, J = face(seed)
        A = 0.37
        E, _, _ = orc.arap_local(U[0], U[1], U[2], M.reshape(-1), A)
        sv = np.linalg.svd(J, compute_uv=False)
        assert E == pytest.approx(A * np.sum((sv - 1.0) ** 2), rel=1e-12)
        W, _, Vt = np.linalg.svd(J)
        R = W @ Vt
        assert np.linalg.det(R) > 0
        assert E == pytest.approx(A * np.sum((J - R) ** 2), rel=1e-12)


def test_arap_rotations_and_scaled_rotations(orc):
    # rest triangle (0,0), (1,0), (0,1): Dm = I; U = rest mapped by s R
    X = np.array([[0.0, 0.0], [1.0, 0.0], [0.0, 1.0]])
    M = np.eye(2).reshape(-1)
    for t in (0.0, 0.4, 2.5, -1.2):
        for sc in (1.0, 0.5, 1.7):
            U = X @ (sc * rot(t)).T + np.array([0.3, -0.2])
            E, g, _ = orc.arap_local(U[0], U[1], U[2], M, 0.8)
            assert E == pytest.approx(2 * 0.8 * (sc - 1.0) ** 2, abs=1e-14)
            if sc == 1.0:
                np.testing.assert_allclose(g, 0.0, atol=1e-14)


def _local(o, U, M, A=0.6):
    return o.arap_local(U[0], U[1], U[2], M.reshape(-1), A)


@pytest.mark.parametrize("seed", [11, 12, 13])
def test_arap_fd_gradient_and_hessian(orc, seed):
    U, M, _ = face(seed)
    E, g, H = _local(orc, U, M)
    h = 1e-6
    gfd = np.zeros(6)
    Hfd = np.zeros((6, 6))
    for q in range(6):
        Up = U.reshape(-1).copy()
        Um = U.reshape(-1).copy()
        Up[q] += h
        Um[q] -= h
        Ep, gp, _ = _local(orc, Up.reshape(3, 2), M)
        Em, gm, _ = _local(orc, Um.reshape(3, 2), M)
        gfd[q] = (Ep - Em) / (2 * h)
        Hfd[q] = (gp - gm) / (2 * h)
    np.testing.assert_allclose(g, gfd, atol=1e-7 * max(1, np.abs(g).max()))
    np.testing.assert_allclose(H, Hfd, atol=1e-6 * max(1, np.abs(H).max()))
    np.testing.assert_allclose(H, H.T, atol=1e-13 * np.abs(H).max())


def test_arap_translation_and_rotation(orc):
    U, M, _ = face(21)
    E, g, H = _local(orc, U, M)
    g2 = g.reshape(3, 2)
    np.testing.assert_allclose(g2.sum(0), 0, atol=1e-13 * max(1, np.abs(g).max()))
    for a in range(2):
        t = np.zeros((3, 2))
        t[:, a] = 1
        np.testing.assert_allclose(H @ t.reshape(-1), 0, atol=1e-12 * np.abs(H).max())
    # rotating the UV leaves E unchanged: H (W u) = W g with W the generator
    W = np.array([[0.0, -1.0], [1.0, 0.0]])
    np.testing.assert_allclose(H @ (U @ W.T).reshape(-1), (g2 @ W.T).reshape(-1),
                               atol=1e-11 * max(1, np.abs(H).max()))
    assert _local(orc, U @ rot(0.9).T, M)[0] == pytest.approx(E, rel=1e-12)


def test_arap_assembled_on_grid_fd(orc):
    ps = mi.param_static(4, 31, np.float64)
    V, F = ps["V"], ps["F"]
    rp, ci = orc.pattern(V, F)

    def ev(uv):
        return orc.eval(V, 2, uv, 32, rp, ci, F=F, Minv=ps["Minv"], area=ps["area"])

    x = ps["UV"].astype(np.float64)
    g, H, E = ev(x)
    # the assembled energy is the sum of the per-face SVD energies
    Es = 0.0
    for f in range(len(F)):
        Ds = np.stack([x[F[f, 1]] - x[F[f, 0]], x[F[f, 2]] - x[F[f, 0]]], axis=1)
        sv = np.linalg.svd(Ds @ ps["Minv"][f], compute_uv=False)
        Es += ps["area"][f] * np.sum((sv - 1) ** 2)
    assert E == pytest.approx(Es, rel=1e-12)
    D = np.zeros((2 * V, 2 * V))
    for i in range(V):
        for q in range(rp[i], rp[i + 1]):
            D[2 * i:2 * i + 2, 2 * ci[q]:2 * ci[q] + 2] = H[q]
    h = 1e-6
    xf = x.reshape(-1)
    for c in (0, 5, 13, 2 * V - 1):
        xp = xf.copy()
        xm = xf.copy()
        xp[c] += h
        xm[c] -= h
        gp, _, Ep = ev(xp.reshape(-1, 2))
        gm, _, Em = ev(xm.reshape(-1, 2))
        assert g.reshape(-1)[c] == pytest.approx((Ep - Em) / (2 * h), abs=1e-6)
        np.testing.assert_allclose(D[:, c], (gp - gm).reshape(-1) / (2 * h), atol=1e-5)
    np.testing.assert_allclose(D, D.T, atol=1e-12 * np.abs(D).max())


def _arap_pins_pass(o):
    try:
        test_arap_energy_matches_svd(o)
        test_arap_rotations_and_scaled_rotations(o)
        test_arap_fd_gradient_and_hessian(o, 11)
        test_arap_translation_and_rotation(o)
    except AssertionError:
        return False
    return True


def test_arap_pins_pass_on_oracle(orc):
    assert _arap_pins_pass(orc)


def test_arap_pins_catch_planted_mistake():
    assert not _arap_pins_pass(oracle.load_mutant(8))
