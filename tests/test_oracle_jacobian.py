"""Pins for the oracle's vector-valued objective: residuals and the sparse
Jacobian J = sum_j P_j^T J_j S_j (no GPU).

Each mesh term's residual vector is defined so that F = 1/2 |r|^2 is the
term's scalar energy.  That ties the Jacobian to the scalar oracle, which is
pinned on its own: 1/2 |r|^2 = E and J^T r = g at any x.  Independent of it:
central finite differences of r, hand values, J^T J = H for springs at their
rest length (where the spring Hessian is exactly its Gauss-Newton part), and
the row/column structure.  Planted mistakes 5 and 6 in the C source must fail
these pins.
"""
import numpy as np
import pytest

import mesh_inputs as mi
import oracle


def dense_j(rows, ncols, rp, ci, vals):
    D = np.zeros((rows, ncols))
    for i in range(rows):
        for q in range(rp[i], rp[i + 1]):
            D[i, ci[q]] += vals[q]
    return D


def cloth_jac(o, n, seed, mask=3, L0=None):
    st = mi.cloth_static(n, np.float64)
    x = mi.cloth_x(n, seed, 0, np.float64)
    L0 = st["L0"] if L0 is None else L0
    r, rp, ci, vals = o.jacobian(st["V"], 3, x, mask, edges=st["edges"], L0=L0, k=st["k"],
                                 xt=st["xt"], w=st["w"])
    return st, x, r, rp, ci, vals


def param_jac(o, n, seed):
    ps = mi.param_static(n, seed, np.float64)
    r, rp, ci, vals = o.jacobian(ps["V"], 2, ps["UV"], 4, F=ps["F"], Minv=ps["Minv"],
                                 area=ps["area"])
    return ps, r, rp, ci, vals


def test_spring_residual_hand_example(orc):
    # xi = (1,0,0), xj = 0, L0 = 1/2, k = 4: r = 2 (1 - 1/2) = 1, dr/dxi = 2 n
    r, J = orc.spring_res(3, [1, 0, 0], [0, 0, 0], 0.5, 4.0)
    assert r[0] == pytest.approx(1.0, abs=1e-15)
    np.testing.assert_allclose(J[0], [2, 0, 0, -2, 0, 0], atol=1e-15)


def test_symdir_residual_at_identity(orc):
    # rest Dm = I (M = I, A = 1/2), u = rest: J = I, J^-1 = I, sqrt(2A) = 1
    r, J = orc.symdir_res([0, 0], [1, 0], [0, 1], np.eye(2), 0.5)
    np.testing.assert_allclose(r, [1, 0, 0, 1, 1, 0, 0, 1], atol=1e-15)
    # d(vec J)/du: w0 = (-1,-1), w1 = (1,0), w2 = (0,1); row 2al+ga, column 2k+be
    W = np.array([[-1, -1], [1, 0], [0, 1]], float)
    for al in range(2):
        for ga in range(2):
            for k in range(3):
                for be in range(2):
                    want = W[k, ga] if al == be else 0.0
                    assert J[2 * al + ga, 2 * k + be] == pytest.approx(want, abs=1e-15)
    # at J = I, d(J^-1) = -dJ: the inverse rows are the negated J rows
    np.testing.assert_allclose(J[4:], -J[:4], atol=1e-15)


@pytest.mark.parametrize("mask", [1, 2, 3])
def test_cloth_half_norm_and_gradient(orc, mask):
    st, x, r, rp, ci, vals = cloth_jac(orc, 6, 11, mask)
    prp, pci = orc.pattern(st["V"], st["F"])
    g, H, E = orc.eval(st["V"], 3, x, mask, prp, pci, edges=st["edges"], L0=st["L0"],
                       k=st["k"], xt=st["xt"], w=st["w"])
    assert 0.5 * r @ r == pytest.approx(E, rel=1e-12)
    D = dense_j(len(r), st["V"] * 3, rp, ci, vals)
    np.testing.assert_allclose(D.T @ r, g.reshape(-1), atol=1e-9 * np.abs(g).max())


def test_symdir_half_norm_and_gradient(orc):
    ps, r, rp, ci, vals = param_jac(orc, 6, 12)
    prp, pci = orc.pattern(ps["V"], ps["F"])
    g, H, E = orc.eval(ps["V"], 2, ps["UV"], 4, prp, pci, F=ps["F"], Minv=ps["Minv"],
                       area=ps["area"])
    assert 0.5 * r @ r == pytest.approx(E, rel=1e-12)
    D = dense_j(len(r), ps["V"] * 2, rp, ci, vals)
    np.testing.assert_allclose(D.T @ r, g.reshape(-1), atol=1e-9 * np.abs(g).max())


def _fd_jacobian(res, x, h):
    x = x.reshape(-1).copy()
    cols = []
    for c in range(x.size):
        xp = x.copy()
        xm = x.copy()
        xp[c] += h
        xm[c] -= h
        cols.append((res(xp) - res(xm)) / (2 * h))
    return np.stack(cols, 1)


def test_cloth_jacobian_fd(orc):
    st = mi.cloth_static(4, np.float64)
    x = mi.cloth_x(4, 13, 0, np.float64)

    def res(xf):
        return orc.jacobian(st["V"], 3, xf, 3, edges=st["edges"], L0=st["L0"], k=st["k"],
                            xt=st["xt"], w=st["w"])[0]

    r, rp, ci, vals = orc.jacobian(st["V"], 3, x, 3, edges=st["edges"], L0=st["L0"],
                                   k=st["k"], xt=st["xt"], w=st["w"])
    D = dense_j(len(r), st["V"] * 3, rp, ci, vals)
    Dfd = _fd_jacobian(res, x, 1e-6)
    np.testing.assert_allclose(D, Dfd, atol=1e-6 * np.abs(D).max())


def test_symdir_jacobian_fd(orc):
    ps = mi.param_static(4, 14, np.float64)

    def res(u):
        return orc.jacobian(ps["V"], 2, u, 4, F=ps["F"], Minv=ps["Minv"], area=ps["area"])[0]

    r, rp, ci, vals = orc.jacobian(ps["V"], 2, ps["UV"], 4, F=ps["F"], Minv=ps["Minv"],
                                   area=ps["area"])
    D = dense_j(len(r), ps["V"] * 2, rp, ci, vals)
    Dfd = _fd_jacobian(res, ps["UV"].astype(np.float64), 1e-7)
    np.testing.assert_allclose(D, Dfd, atol=1e-5 * np.abs(D).max())


def test_springs_at_rest_length_gauss_newton_is_the_hessian(orc):
    # with L0 = |xi - xj| the spring Hessian is k n n^T, i.e. exactly J^T J
    st = mi.cloth_static(5, np.float64)
    x = mi.cloth_x(5, 15, 0, np.float64)
    e = st["edges"]
    L0 = np.linalg.norm(x[e[:, 0]] - x[e[:, 1]], axis=1)
    r, rp, ci, vals = orc.jacobian(st["V"], 3, x, 1, edges=e, L0=L0, k=st["k"])
    np.testing.assert_allclose(r, 0, atol=1e-12)
    prp, pci = orc.pattern(st["V"], st["F"])
    g, H, E = orc.eval(st["V"], 3, x, 1, prp, pci, edges=e, L0=L0, k=st["k"])
    D = dense_j(len(r), st["V"] * 3, rp, ci, vals)
    Hd = np.zeros((st["V"] * 3,) * 2)
    for i in range(st["V"]):
        for q in range(prp[i], prp[i + 1]):
            j = pci[q]
            Hd[3 * i:3 * i + 3, 3 * j:3 * j + 3] = H[q]
    np.testing.assert_allclose(D.T @ D, Hd, atol=1e-9 * np.abs(Hd).max())


def test_row_structure(orc):
    # rows: springs (edge order, 2 dof sorted columns), then inertia (one
    # nonzero on the row's own column), then nothing else
    st, x, r, rp, ci, vals = cloth_jac(orc, 5, 16, 3)
    E, V = len(st["edges"]), st["V"]
    assert len(r) == E + 3 * V and rp[-1] == E * 6 + 3 * V
    for e in range(E):
        a, b = st["edges"][e]
        np.testing.assert_array_equal(ci[rp[e]:rp[e + 1]],
                                      [3 * a, 3 * a + 1, 3 * a + 2, 3 * b, 3 * b + 1, 3 * b + 2])
    np.testing.assert_array_equal(ci[rp[E]:], np.arange(3 * V))
    np.testing.assert_allclose(vals[rp[E]:], np.sqrt(st["w"]), rtol=1e-15)
    # faces: 8 rows of 6 ascending columns over the face's sorted vertices
    ps, r2, rp2, ci2, v2 = param_jac(orc, 4, 17)
    for f, tri in enumerate(ps["F"]):
        vs = sorted(tri)
        want = [2 * vs[0], 2 * vs[0] + 1, 2 * vs[1], 2 * vs[1] + 1, 2 * vs[2], 2 * vs[2] + 1]
        for p in range(8):
            row = 8 * f + p
            np.testing.assert_array_equal(ci2[rp2[row]:rp2[row + 1]], want)


def _jac_pins_pass(o):
    try:
        test_symdir_residual_at_identity(o)
        test_symdir_half_norm_and_gradient(o)
        test_symdir_jacobian_fd(o)
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("mutant", [5, 6])
def test_jacobian_pins_catch_planted_mistakes(mutant):
    assert not _jac_pins_pass(oracle.load_mutant(mutant))


def test_jacobian_pins_pass_on_oracle(orc):
    assert _jac_pins_pass(orc)
