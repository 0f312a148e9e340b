"""Pins for the fp64 CPU oracle (no GPU).

The oracle is pinned to facts that do not come from itself: hand-derived
values of the energies at chosen points, central finite differences of its
own energy (which checks every derivative against the energy definition),
symmetry, translation and rotation invariance, linearity of the assembly sum,
and a CSR pattern built by brute force from a dense adjacency matrix.  A
mutation test at the end plants a plausible mistake in each part of the C
source and checks that some pin fails.
"""
import numpy as np
import pytest

import mesh_inputs as mi
import oracle

# ---------------------------------------------------------------- helpers


def dense(V, dof, rp, ci, H):
    D = np.zeros((V * dof, V * dof))
    for i in range(V):
        for q in range(rp[i], rp[i + 1]):
            j = ci[q]
            D[i * dof:(i + 1) * dof, j * dof:(j + 1) * dof] = H[q]
    return D


def cloth_case(orc, n, seed=7, step=0, with_pairs=0):
    st = mi.cloth_static(n, np.float64)
    x = mi.cloth_x(n, seed, step, np.float64)
    pairs = mi.random_pairs(n, with_pairs, seed, step) if with_pairs else None
    rest = mi.pair_rest(x, pairs, np.float64) if with_pairs else None
    rp, ci = orc.pattern(st["V"], st["F"], pairs)
    return st, x, pairs, rest, rp, ci


def cloth_eval(orc, st, x, rp, ci, mask, pairs=None, rest=None):
    return orc.eval(st["V"], 3, x, mask, rp, ci, edges=st["edges"], L0=st["L0"],
                    k=st["k"], xt=st["xt"], w=st["w"], pairs=pairs, prest=rest,
                    kp=mi.PAIR_K)


def single_tri(J, area_scale=1.0):
    """One triangle with rest Dm = I (M = I, area 1/2) whose UV Jacobian is J."""
    J = np.asarray(J, np.float64)
    u0 = np.zeros(2)
    return u0, J[:, 0].copy(), J[:, 1].copy(), np.eye(2), 0.5 * area_scale


# ------------------------------------------------------ local closed forms


def test_spring_hand_example(orc):
    # xi = 0, xj = (2,0,0), L0 = 1, k = 1: d = (-2,0,0), l = 2, n = (-1,0,0),
    # E = 1/2 (2-1)^2, g_i = k (l-L0) n = (-1,0,0) = -g_j,
    # K = n n^T + (1 - 1/2)(I - n n^T) = diag(1, 1/2, 1/2).
    E, g, H = orc.spring_local([0, 0, 0], [2, 0, 0], 1.0, 1.0)
    assert E == pytest.approx(0.5, abs=1e-15)
    np.testing.assert_allclose(g, [-1, 0, 0, 1, 0, 0], atol=1e-15)
    K = np.diag([1.0, 0.5, 0.5])
    np.testing.assert_allclose(H, np.block([[K, -K], [-K, K]]), atol=1e-15)


def test_spring_at_rest_length(orc):
    # at l = L0 the gradient vanishes and K = k n n^T
    d = np.array([0.3, -0.4, 1.2])
    L0 = np.linalg.norm(d)
    E, g, H = orc.spring_local(d, [0, 0, 0], L0, 5.0)
    assert E == pytest.approx(0.0, abs=1e-14)
    np.testing.assert_allclose(g, 0, atol=1e-13)
    nn = np.outer(d, d) / L0 ** 2
    np.testing.assert_allclose(H[:3, :3], 5.0 * nn, atol=1e-12)


def test_spring_2d(orc):
    # 2D spring, xi = (0,3), xj = (0,0), L0 = 1, k = 2: n = (0,1), s = 2,
    # E = 4, g_i = (0, 4), K = 2 [n n^T + (2/3)(I - n n^T)] = diag(4/3, 2)
    E, g, H = orc.spring_local([0, 3], [0, 0], 1.0, 2.0)
    assert E == pytest.approx(4.0)
    np.testing.assert_allclose(g, [0, 4, 0, -4], atol=1e-14)
    np.testing.assert_allclose(H[:2, :2], np.diag([4 / 3, 2.0]), atol=1e-14)


def test_inertia_closed_form(orc):
    E, g, H = orc.inertia_local([1.0, 2.0, 3.0], [1.0, 0.0, 4.0], 3.0)
    assert E == pytest.approx(0.5 * 3.0 * 5.0)
    np.testing.assert_allclose(g, [0.0, 6.0, -3.0])
    np.testing.assert_allclose(H, 3.0 * np.eye(3))


@pytest.mark.parametrize("J,expect", [
    (np.eye(2), 4.0),                          # |I|^2 + |I|^2
    (np.diag([2.0, 1.0]), 5.0 + 1.25),         # 4+1 and 1/4+1
    (3.0 * np.eye(2), 18.0 + 2.0 / 9.0),       # 2c^2 + 2/c^2
    (np.array([[1.0, 0.5], [0.0, 1.0]]), 2.25 + 2.25),  # shear: J^-1 = [[1,-.5],[0,1]]
])
def test_symdir_closed_form_values(orc, J, expect):
    u0, u1, u2, M, A = single_tri(J)
    E, g, H = orc.symdir_local(u0, u1, u2, M, A)
    assert E == pytest.approx(A * expect, rel=1e-14)


def test_symdir_rest_pose_and_rotation(orc):
    # at J = I the energy is minimal (g = 0); a rotated J has the same energy
    u0, u1, u2, M, A = single_tri(np.eye(2))
    E, g, H = orc.symdir_local(u0, u1, u2, M, A)
    np.testing.assert_allclose(g, 0, atol=1e-14)
    th = 0.7
    R = np.array([[np.cos(th), -np.sin(th)], [np.sin(th), np.cos(th)]])
    S = np.diag([2.0, 0.5])
    E1 = orc.symdir_local(*single_tri(S))[0]
    E2 = orc.symdir_local(*single_tri(R @ S))[0]
    assert E2 == pytest.approx(E1, rel=1e-13)


def test_symdir_general_rest_shape(orc):
    # a non-identity rest triangle: Dm = [[2, 1], [0, 1]] -> J = Ds Dm^-1; the
    # UV triangle equal to the rest triangle gives J = I, E = 4A, g = 0
    X = np.array([[0.0, 0.0], [2.0, 0.0], [1.0, 1.0]])
    Dm = np.stack([X[1] - X[0], X[2] - X[0]], 1)
    M = np.linalg.inv(Dm)
    A = 0.5 * abs(np.linalg.det(Dm))
    E, g, _ = orc.symdir_local(X[0], X[1], X[2], M, A)
    assert E == pytest.approx(4 * A, rel=1e-14)
    np.testing.assert_allclose(g, 0, atol=1e-14)
    # uniform scale by c: E = A (2 c^2 + 2 / c^2)
    E2, _, _ = orc.symdir_local(1.5 * X[0], 1.5 * X[1], 1.5 * X[2], M, A)
    assert E2 == pytest.approx(A * (2 * 1.5 ** 2 + 2 / 1.5 ** 2), rel=1e-13)


# ------------------------------------------- finite differences (fp64)


def _fd_check(energy_and_grad, x, h, rtol):
    E0, g0 = energy_and_grad(x)
    fd = np.zeros_like(x)
    flat = x.reshape(-1)
    for k in range(flat.size):
        xp = flat.copy(); xp[k] += h
        xm = flat.copy(); xm[k] -= h
        fd.reshape(-1)[k] = (energy_and_grad(xp.reshape(x.shape))[0] -
                             energy_and_grad(xm.reshape(x.shape))[0]) / (2 * h)
    scale = np.abs(g0).max()
    assert np.abs(fd - g0).max() <= rtol * scale, (np.abs(fd - g0).max(), scale)


def _fd_hessian_check(grad_and_dense_h, x, h, rtol):
    g0, D = grad_and_dense_h(x)
    flat = x.reshape(-1)
    fdH = np.zeros_like(D)
    for k in range(flat.size):
        xp = flat.copy(); xp[k] += h
        xm = flat.copy(); xm[k] -= h
        fdH[:, k] = (grad_and_dense_h(xp.reshape(x.shape))[0].reshape(-1) -
                     grad_and_dense_h(xm.reshape(x.shape))[0].reshape(-1)) / (2 * h)
    scale = np.abs(D).max()
    assert np.abs(fdH - D).max() <= rtol * scale, (np.abs(fdH - D).max(), scale)


@pytest.mark.parametrize("mask", [1, 2, 3, 1 | 8, 3 | 8])
def test_cloth_fd(orc, mask):
    n = 4
    st, x, pairs, rest, rp, ci = cloth_case(orc, n, with_pairs=3 if mask & 8 else 0)
    V = st["V"]
    h = 1e-6 * mi.grid_spacing(n)

    def eg(xx):
        g, H, E = cloth_eval(orc, st, xx, rp, ci, mask, pairs, rest)
        return E, g

    def gh(xx):
        g, H, E = cloth_eval(orc, st, xx, rp, ci, mask, pairs, rest)
        return g, dense(V, 3, rp, ci, H)

    _fd_check(eg, x.astype(np.float64), h, 1e-6)
    _fd_hessian_check(gh, x.astype(np.float64), h, 1e-6)


def test_symdir_fd(orc):
    n = 4
    ps = mi.param_static(n, 5, np.float64)
    V = ps["V"]
    rp, ci = orc.pattern(V, ps["F"])
    h = 1e-6 * mi.grid_spacing(n)

    def ev(xx):
        return orc.eval(V, 2, xx, 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])

    _fd_check(lambda xx: (ev(xx)[2], ev(xx)[0]), ps["UV"].astype(np.float64), h, 1e-6)
    _fd_hessian_check(lambda xx: (ev(xx)[0], dense(V, 2, rp, ci, ev(xx)[1])),
                      ps["UV"].astype(np.float64), h, 1e-6)


# ------------------------------------------------------ invariants


def test_cloth_symmetry_translation_rotation(orc):
    n = 6
    st, x, pairs, rest, rp, ci = cloth_case(orc, n, with_pairs=5)
    V = st["V"]
    g, H, E = cloth_eval(orc, st, x, rp, ci, 1 | 8, pairs, rest)  # no inertia
    D = dense(V, 3, rp, ci, H)
    scale = np.abs(D).max()
    np.testing.assert_allclose(D, D.T, atol=1e-12 * scale)
    # translation: sum_i g_i = 0, H t = 0
    np.testing.assert_allclose(g.sum(0), 0, atol=1e-12 * np.abs(g).max())
    for t in np.eye(3):
        Ht = D @ np.tile(t, V)
        assert np.abs(Ht).max() <= 1e-12 * scale
    # rotation: sum_i x_i x g_i = 0, and H (W x) = W g for every skew W
    x64 = x.astype(np.float64)
    np.testing.assert_allclose(np.cross(x64, g).sum(0), 0, atol=1e-12 * np.abs(g).max())
    for a in np.eye(3):
        W = np.cross(np.eye(3), a)  # W v = v x a (a skew matrix)
        lhs = (D @ (x64 @ W.T).reshape(-1)).reshape(V, 3)
        rhs = g @ W.T
        assert np.abs(lhs - rhs).max() <= 1e-10 * scale


def test_symdir_symmetry_translation_rotation(orc):
    n = 5
    ps = mi.param_static(n, 9, np.float64)
    V = ps["V"]
    rp, ci = orc.pattern(V, ps["F"])
    g, H, E = orc.eval(V, 2, ps["UV"], 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])
    D = dense(V, 2, rp, ci, H)
    scale = np.abs(D).max()
    np.testing.assert_allclose(D, D.T, atol=1e-12 * scale)
    np.testing.assert_allclose(g.sum(0), 0, atol=1e-12 * np.abs(g).max())
    for t in np.eye(2):
        assert np.abs(D @ np.tile(t, V)).max() <= 1e-12 * scale
    u = ps["UV"].astype(np.float64)
    assert abs((u[:, 0] * g[:, 1] - u[:, 1] * g[:, 0]).sum()) <= 1e-12 * np.abs(g).max() * V
    W = np.array([[0.0, -1.0], [1.0, 0.0]])
    lhs = (D @ (u @ W.T).reshape(-1)).reshape(V, 2)
    assert np.abs(lhs - g @ W.T).max() <= 1e-10 * scale


def test_symdir_rest_mesh_rotation_null(orc):
    # UV = rest grid: g = 0 and the infinitesimal rotation is in ker H
    n = 4
    ps = mi.param_static(n, 1, np.float64)
    V = ps["V"]
    rp, ci = orc.pattern(V, ps["F"])
    X = ps["X"]
    g, H, E = orc.eval(V, 2, X, 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])
    assert E == pytest.approx(4.0 * ps["area"].astype(np.float64).sum(), rel=1e-12)
    np.testing.assert_allclose(g, 0, atol=1e-10)
    D = dense(V, 2, rp, ci, H)
    rot = np.stack([-X[:, 1], X[:, 0]], 1).reshape(-1)
    assert np.abs(D @ rot).max() <= 1e-10 * np.abs(D).max()


def test_single_spring_block_placement(orc):
    # one triangle, one active spring on edge (0, 1): exact blocks by hand
    F = np.array([[0, 1, 2]], np.int32)
    rp, ci = orc.pattern(3, F)
    x = np.array([[0, 0, 0], [2, 0, 0], [5, 5, 5]], np.float64)
    g, H, E = orc.eval(3, 3, x, 1, rp, ci, edges=np.array([[0, 1]], np.int32),
                       L0=np.array([1.0]), k=1.0)
    K = np.diag([1.0, 0.5, 0.5])
    D = dense(3, 3, rp, ci, H)
    np.testing.assert_allclose(D[0:3, 0:3], K, atol=1e-15)
    np.testing.assert_allclose(D[0:3, 3:6], -K, atol=1e-15)
    np.testing.assert_allclose(D[3:6, 0:3], -K, atol=1e-15)
    np.testing.assert_allclose(D[3:6, 3:6], K, atol=1e-15)
    np.testing.assert_allclose(D[6:, :], 0, atol=0)
    np.testing.assert_allclose(g, [[-1, 0, 0], [1, 0, 0], [0, 0, 0]], atol=1e-15)
    assert E == pytest.approx(0.5)


def test_inertia_only_is_diagonal(orc):
    st, x, _, _, rp, ci = cloth_case(orc, 3)
    g, H, E = cloth_eval(orc, st, x, rp, ci, 2)
    D = dense(st["V"], 3, rp, ci, H)
    np.testing.assert_allclose(D, st["w"] * np.eye(D.shape[0]), atol=1e-15)
    np.testing.assert_allclose(g, st["w"] * (x.astype(np.float64) - st["xt"]), rtol=1e-14)


def test_pair_duplicates_and_edge_coincidence_merge(orc):
    n = 4
    st, x, _, _, rp0, ci0 = cloth_case(orc, n)
    V = st["V"]
    p = np.array([[0, 15]], np.int32)           # far apart: a new block
    e = np.array([[0, 1]], np.int32)            # an existing mesh edge
    rest = np.array([0.1])
    base = cloth_eval(orc, st, x, rp0, ci0, 3)
    # a pair on an existing edge adds no block
    rpe, cie = orc.pattern(V, st["F"], e)
    np.testing.assert_array_equal(rpe, rp0)
    np.testing.assert_array_equal(cie, ci0)
    # duplicated pair: one block pair, twice the single contribution (linearity)
    rp1, ci1 = orc.pattern(V, st["F"], p)
    rp2, ci2 = orc.pattern(V, st["F"], np.concatenate([p, p]))
    np.testing.assert_array_equal(rp1, rp2)
    np.testing.assert_array_equal(ci1, ci2)
    assert rp1[V] == rp0[V] + 2
    one = cloth_eval(orc, st, x, rp1, ci1, 3 | 8, p, rest)
    two = cloth_eval(orc, st, x, rp1, ci1, 3 | 8, np.concatenate([p, p]), np.concatenate([rest, rest]))
    D0 = dense(V, 3, rp0, ci0, base[1])
    D1 = dense(V, 3, rp1, ci1, one[1])
    D2 = dense(V, 3, rp1, ci1, two[1])
    np.testing.assert_allclose(D2 - D0, 2 * (D1 - D0), atol=1e-9 * np.abs(D1).max())
    np.testing.assert_allclose(two[0] - base[0], 2 * (one[0] - base[0]), atol=1e-12)
    # the pair's off-diagonal block equals -K of the hand formula
    Ep, gp, Hp = orc.spring_local(x[0], x[15], 0.1, mi.PAIR_K)
    np.testing.assert_allclose(D1[0:3, 45:48], Hp[:3, 3:], rtol=1e-12)
    # pair coinciding with an edge lands on that edge's existing block
    oe = cloth_eval(orc, st, x, rp0, ci0, 3 | 8, e, rest)
    Ee, ge, He = orc.spring_local(x[0], x[1], 0.1, mi.PAIR_K)
    De = dense(V, 3, rp0, ci0, oe[1])
    np.testing.assert_allclose(De[0:3, 3:6] - D0[0:3, 3:6], He[:3, 3:], rtol=1e-10, atol=1e-9)


# ------------------------------------------------------------- pattern


def brute_pattern(V, F, pairs=None):
    A = np.eye(V, dtype=bool)
    for f in F:
        for a in f:
            for b in f:
                A[a, b] = True
    if pairs is not None:
        for i, j in pairs:
            A[i, j] = A[j, i] = True
    rows, cols = np.nonzero(A)
    rp = np.zeros(V + 1, np.int64)
    np.add.at(rp, rows + 1, 1)
    return np.cumsum(rp), cols


@pytest.mark.parametrize("n", [1, 2, 3, 10])
def test_pattern_bruteforce_grid(orc, n):
    X, F = mi.grid_mesh(n)
    V = n * n
    rp, ci = orc.pattern(V, F)
    brp, bci = brute_pattern(V, F)
    np.testing.assert_array_equal(rp, brp)
    np.testing.assert_array_equal(ci, bci)
    E = 2 * n * (n - 1) + (n - 1) ** 2
    assert rp[V] == V + 2 * E
    if n == 10:
        assert rp[V] == 622


def test_pattern_bruteforce_random_mesh_with_pairs(orc):
    rng = np.random.default_rng(3)
    V = 40
    F = np.array([rng.choice(V, 3, replace=False) for _ in range(50)], np.int32)
    P = np.array([rng.choice(V, 2, replace=False) for _ in range(30)], np.int32)
    rp, ci = orc.pattern(V, F, P)
    brp, bci = brute_pattern(V, F, P)
    np.testing.assert_array_equal(rp, brp)
    np.testing.assert_array_equal(ci, bci)


@pytest.mark.parametrize("n", [2, 3, 10, 31])
def test_edges_match_grid_structure(orc, n):
    X, F = mi.grid_mesh(n)
    ij = orc.edges(n * n, F)
    np.testing.assert_array_equal(ij, mi.grid_edges(n))
    assert ij.shape[0] == 2 * n * (n - 1) + (n - 1) ** 2


def test_pattern_rejects_bad_faces(orc):
    with pytest.raises(ValueError):
        orc.pattern(3, np.array([[0, 1, 3]], np.int32))
    with pytest.raises(ValueError):
        orc.pattern(3, np.array([[0, 1, 1]], np.int32))


# ------------------------------------------------------------------- HVP


def test_hvp_matches_fd_of_gradient(orc):
    n = 5
    ps = mi.param_static(n, 4, np.float64)
    V = ps["V"]
    rp, ci = orc.pattern(V, ps["F"])
    v = mi.probe_vector(V, 2, 11, np.float64)
    u = ps["UV"].astype(np.float64)
    g, H, E = orc.eval(V, 2, u, 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])
    y = orc.bsr_mv(V, 2, rp, ci, H, v)
    eps = 1e-6 * mi.grid_spacing(n)
    gp = orc.eval(V, 2, u + eps * v, 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])[0]
    gm = orc.eval(V, 2, u - eps * v, 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])[0]
    fd = (gp - gm) / (2 * eps)
    assert np.abs(fd - y).max() <= 1e-6 * np.abs(y).max()


def test_bsr_mv_matches_dense(orc):
    st, x, pairs, rest, rp, ci = cloth_case(orc, 4, with_pairs=2)
    g, H, E = cloth_eval(orc, st, x, rp, ci, 3 | 8, pairs, rest)
    v = mi.probe_vector(st["V"], 3, 2, np.float64)
    y = orc.bsr_mv(st["V"], 3, rp, ci, H, v)
    np.testing.assert_allclose(y.reshape(-1), dense(st["V"], 3, rp, ci, H) @ v.reshape(-1),
                               rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- generators


def test_generator_counts_and_pairs():
    X, F = mi.grid_mesh(10)
    assert F.shape == (162, 3)
    assert mi.grid_edges(10).shape[0] == 261
    P = mi.random_pairs(30, 200, 5, 0)
    key = np.minimum(P[:, 0], P[:, 1]) * 900 + np.maximum(P[:, 0], P[:, 1])
    assert np.unique(key).size == 200
    assert not mi.grid_adjacent(30, P[:, 0], P[:, 1]).any()
    assert (P[:, 0] != P[:, 1]).all()
    ps = mi.param_static(10, 1)
    u = ps["UV"].astype(np.float64)
    e1 = u[ps["F"][:, 1]] - u[ps["F"][:, 0]]
    e2 = u[ps["F"][:, 2]] - u[ps["F"][:, 0]]
    assert ((e1[:, 0] * e2[:, 1] - e1[:, 1] * e2[:, 0]) > 0).all()


# --------------------------------------------------------- mutation test


def _pins_pass(o):
    """A compact subset of the pins above, run against an oracle build."""
    try:
        E, g, H = o.spring_local([0, 0, 0], [2, 0, 0], 1.0, 1.0)
        K = np.diag([1.0, 0.5, 0.5])
        if not np.allclose(g, [-1, 0, 0, 1, 0, 0]) or not np.allclose(H[:3, :3], K):
            return False
        for J in (np.diag([2.0, 1.0]), np.array([[1.2, 0.3], [-0.1, 0.9]])):
            u0, u1, u2, M, A = single_tri(J)
            _, gl, Hl = o.symdir_local(u0, u1, u2, M, A)
            if not np.allclose(Hl, Hl.T, atol=1e-12):
                return False
        st, x, pairs, rest, rp, ci = cloth_case(o, 3, with_pairs=2)
        V = st["V"]
        g, H, E = cloth_eval(o, st, x, rp, ci, 1 | 8, pairs, rest)
        if np.abs(g.sum(0)).max() > 1e-9 * np.abs(g).max():
            return False
        D = dense(V, 3, rp, ci, H)
        if np.abs(D @ np.tile([1.0, 0, 0], V)).max() > 1e-9 * np.abs(D).max():
            return False
        ps = mi.param_static(3, 2, np.float64)
        rpf, cif = o.pattern(9, ps["F"])
        gs, Hs, Es = o.eval(9, 2, ps["UV"], 4, rpf, cif, F=ps["F"], Minv=ps["Minv"], area=ps["area"])
        Ds = dense(9, 2, rpf, cif, Hs)
        if not np.allclose(Ds, Ds.T, atol=1e-10 * np.abs(Ds).max()):
            return False
        if np.abs(Ds @ np.tile([1.0, 0], 9)).max() > 1e-9 * np.abs(Ds).max():
            return False
        # H (W u) = W g for the infinitesimal rotation W
        u = ps["UV"].astype(np.float64)
        W = np.array([[0.0, -1.0], [1.0, 0.0]])
        if np.abs((Ds @ (u @ W.T).reshape(-1)).reshape(9, 2) - gs @ W.T).max() > \
                1e-8 * np.abs(Ds).max():
            return False
        return True
    except ValueError:
        return False


def test_pins_pass_on_oracle(orc):
    assert _pins_pass(orc)


@pytest.mark.parametrize("mutant", [1, 2, 3, 4])
def test_pins_catch_planted_mistakes(mutant):
    m = oracle.load_mutant(mutant)
    assert not _pins_pass(m), f"planted mistake {mutant} went unnoticed"
