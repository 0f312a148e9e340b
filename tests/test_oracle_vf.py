"""Pins for the oracle's vertex-face term (4-vertex stencil, 12 variables;
no GPU): E = 1/2 k (d - r)^2 with d the signed distance from p to the plane
of (a, b, c).  Closed forms over a flat triangle (the gradient on the corners
is minus the barycentric weights of p), central finite differences,
symmetry, translation and rotation invariance, and the orientation flip.  A
planted mistake (the bilinear part of the normal dropped) must fail them."""
import numpy as np
import pytest

import oracle


def config(seed):
    rng = np.random.default_rng(seed)
    while True:
        X = rng.standard_normal((4, 3))
        n = np.cross(X[2] - X[1], X[3] - X[1])
        if np.linalg.norm(n) > 0.3:
            return X


def test_vf_flat_triangle_closed_form(orc):
    a, b, c = np.zeros(3), np.array([1.0, 0, 0]), np.array([0, 1.0, 0])
    for (px, py, h) in ((0.2, 0.3, 0.5), (0.6, 0.1, -0.25), (-0.3, 1.4, 2.0)):
        p = np.array([px, py, h])
        r, k = 0.1, 2.0
        E, g, H = orc.vf_local(p, a, b, c, r, k)
        assert E == pytest.approx(0.5 * k * (h - r) ** 2, rel=1e-14)
        bary = np.array([1 - px - py, px, py])  # weights of a, b, c at p's foot point
        gd = np.zeros(12)
        gd[2] = 1.0
        gd[5::3] = -bary
        np.testing.assert_allclose(g, k * (h - r) * gd, atol=1e-14)


def _local(o, X, r=0.2, k=3.0):
    return o.vf_local(X[0], X[1], X[2], X[3], r, k)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_vf_fd_gradient_and_hessian(orc, seed):
    X = config(seed)
    E, g, H = _local(orc, X)
    h = 1e-6
    gfd = np.zeros(12)
    Hfd = np.zeros((12, 12))
    for q in range(12):
        Xp = X.reshape(-1).copy()
        Xm = X.reshape(-1).copy()
        Xp[q] += h
        Xm[q] -= h
        Ep, gp, _ = _local(orc, Xp.reshape(4, 3))
        Em, gm, _ = _local(orc, Xm.reshape(4, 3))
        gfd[q] = (Ep - Em) / (2 * h)
        Hfd[q] = (gp - gm) / (2 * h)
    np.testing.assert_allclose(g, gfd, atol=1e-7 * max(1, np.abs(g).max()))
    np.testing.assert_allclose(H, Hfd, atol=1e-6 * max(1, np.abs(H).max()))
    np.testing.assert_allclose(H, H.T, atol=1e-12 * np.abs(H).max())


def test_vf_translation_rotation_and_flip(orc):
    X = config(4)
    E, g, H = _local(orc, X)
    g4 = g.reshape(4, 3)
    np.testing.assert_allclose(g4.sum(0), 0, atol=1e-12 * max(1, np.abs(g).max()))
    for ax in range(3):
        t = np.zeros((4, 3))
        t[:, ax] = 1
        np.testing.assert_allclose(H @ t.reshape(-1), 0, atol=1e-11 * np.abs(H).max())
        W = np.zeros((3, 3))
        b, c = [q for q in range(3) if q != ax]
        W[b, c], W[c, b] = -1, 1
        np.testing.assert_allclose(H @ (X @ W.T).reshape(-1), (g4 @ W.T).reshape(-1),
                                   atol=1e-10 * max(1, np.abs(H).max()))
    th = 0.8
    R = np.array([[1, 0, 0], [0, np.cos(th), -np.sin(th)], [0, np.sin(th), np.cos(th)]])
    assert _local(orc, X @ R.T)[0] == pytest.approx(E, rel=1e-12)
    # swapping b and c flips the normal and with it the sign of d
    Ef, _, _ = orc.vf_local(X[0], X[1], X[3], X[2], -0.2, 3.0)
    assert Ef == pytest.approx(E, rel=1e-12)


def _vf_pins_pass(o):
    try:
        test_vf_flat_triangle_closed_form(o)
        test_vf_fd_gradient_and_hessian(o, 1)
        test_vf_translation_rotation_and_flip(o)
    except AssertionError:
        return False
    return True


def test_vf_pins_pass_on_oracle(orc):
    assert _vf_pins_pass(orc)


def test_vf_pins_catch_planted_mistake():
    assert not _vf_pins_pass(oracle.load_mutant(9))


def vf_pairs(vf, F):
    """The three vertex pairs that a vertex-face term adds to the pattern."""
    return np.array([(p, F[f][c]) for p, f in vf for c in range(3)], np.int32)


def test_vf_assembled_on_cloth_fd(orc):
    import mesh_inputs as mi
    n = 5
    st = mi.cloth_static(n, np.float64)
    V, F = st["V"], st["F"]
    rng = np.random.default_rng(9)
    x = mi.cloth_x(n, 22, 0, np.float64) + 0.05 * rng.standard_normal((V, 3))
    vf = []
    while len(vf) < 6:
        p, f = int(rng.integers(0, V)), int(rng.integers(0, len(F)))
        if p not in F[f]:
            vf.append((p, f))
    vf = np.array(vf, np.int32)
    rest = 0.01 * rng.standard_normal(len(vf))
    rp, ci = orc.pattern(V, F, vf_pairs(vf, F))
    kc = 40.0

    def ev(xx):
        return orc.eval(V, 3, xx, 2 | 64, rp, ci, xt=st["xt"], w=st["w"], F=F, vf=vf,
                        vf_rest=rest, kc=kc)

    g, H, E = ev(x)
    Eloc = sum(orc.vf_local(x[p], *x[F[f]], r, kc)[0] for (p, f), r in zip(vf, rest))
    Ein = 0.5 * st["w"] * np.sum((x - st["xt"]) ** 2)
    assert E == pytest.approx(Eloc + Ein, rel=1e-12)
    D = np.zeros((3 * V, 3 * V))
    for i in range(V):
        for q in range(rp[i], rp[i + 1]):
            D[3 * i:3 * i + 3, 3 * ci[q]:3 * ci[q] + 3] = H[q]
    np.testing.assert_allclose(D, D.T, atol=1e-12 * np.abs(D).max())
    h = 1e-6
    xf = x.reshape(-1)
    touched = sorted({int(vf[0, 0]), *map(int, F[vf[0, 1]])})
    for c in [3 * touched[0], 3 * touched[1] + 2, 3 * touched[-1] + 1, 0]:
        xp = xf.copy()
        xm = xf.copy()
        xp[c] += h
        xm[c] -= h
        gp, _, Ep = ev(xp.reshape(-1, 3))
        gm, _, Em = ev(xm.reshape(-1, 3))
        assert g.reshape(-1)[c] == pytest.approx((Ep - Em) / (2 * h), abs=1e-6)
        np.testing.assert_allclose(D[:, c], (gp - gm).reshape(-1) / (2 * h), atol=1e-5)


def test_random_vf_inputs():
    import mesh_inputs as mi
    n = 12
    _, F = mi.grid_mesh(n, 3)
    vf = mi.random_vf(n, 500, 3, 0)
    assert vf.shape == (500, 2) and vf.dtype == np.int32
    p, f = vf[:, 0], vf[:, 1]
    assert not (p[:, None] == F[f]).any()
    a = F[f, 0]
    assert (np.abs(p % n - a % n) <= 2).all() and (np.abs(p // n - a // n) <= 2).all()
    pairs = mi.vf_pairs(vf, F)
    np.testing.assert_array_equal(pairs[:, 0], np.repeat(p, 3))
    np.testing.assert_array_equal(pairs[:, 1], F[f].reshape(-1))
    np.testing.assert_array_equal(mi.random_vf(n, 500, 3, 0), vf)
