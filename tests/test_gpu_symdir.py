"""Symmetric-Dirichlet parameterization (dof 2, 2x2 blocks) and the
matrix-free Hessian-vector product: CUDA path vs the fp64 oracle."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, assert_close, gpu_pattern, to_dev

pytestmark = pytest.mark.gpu
FULL = 1
PATCH = 4  # the patch-staged kernel instead of the row-streaming one
GEN = 8  # the energy as a plain expression (MAD_EVAL_GENERIC_AD)


def setup(n, dtype, seed=1004, **kw):
    import hessian_assembly_b200 as mad
    ps = mi.param_static(n, seed, np.dtype(dtype))
    ctx = mad.Context(ps["V"], ps["F"], 2, dtype, part_xyz=ps["X"], **kw)
    return ctx, ps


def terms_for(ps, dtype, flags=0):
    import hessian_assembly_b200 as mad
    return mad.Terms(mask=4, flags=flags, face_Minv=to_dev(ps["Minv"].reshape(-1, 4), dtype),
                     face_area=to_dev(ps["area"], dtype))


def check(orc, n, dtype, flags=0, seed=1004, **kw):
    import torch
    ctx, ps = setup(n, dtype, seed, **kw)
    V = ps["V"]
    tt = getattr(torch, dtype)
    terms = terms_for(ps, dtype, flags)
    x = to_dev(ps["UV"], dtype)
    g = torch.full((V, 2), float("nan"), dtype=tt, device="cuda")
    H = torch.full((ctx.info.capacity_blocks, 2, 2), float("nan"), dtype=tt, device="cuda")
    e = torch.zeros(1, dtype=torch.float64, device="cuda")
    ctx.mad_eval(x, terms, g, H, e)
    v = mi.probe_vector(V, 2, seed + 1, np.dtype(dtype))
    y = torch.full((V, 2), float("nan"), dtype=tt, device="cuda")
    ctx.mad_hvp(x, terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, ps["F"])
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(V, 2, ps["UV"], 4, orp, oci, F=ps["F"], Minv=ps["Minv"],
                          area=ps["area"])
    assert_close("g", g.cpu().numpy(), og, dtype)
    assert_close("H", H[:nnzb].cpu().numpy(), oH, dtype)
    assert abs(e.item() - oE) <= ETOL[dtype] * abs(oE)
    oy = orc.bsr_mv(V, 2, orp, oci, oH, v)
    assert_close("y", y.cpu().numpy(), oy, dtype)
    return ctx


@pytest.mark.parametrize("flags", [0, FULL, PATCH, PATCH | FULL, GEN])
def test_symdir_small(orc, flags):
    check(orc, 10, "float32", flags)


@pytest.mark.parametrize("flags", [0, FULL, PATCH, PATCH | FULL, GEN])
def test_symdir_fp64(orc, flags):
    check(orc, 37, "float64", flags)


@pytest.mark.parametrize("flags", [0, PATCH])
def test_symdir_500x500_full(orc, flags):
    ctx = check(orc, 500, "float32", flags)
    assert ctx.info.n_patches > 100


def test_symdir_500x500_generic_ad(orc):
    check(orc, 500, "float32", GEN, seed=2005)


def test_symdir_500x500_full_ad(orc):
    check(orc, 500, "float32", FULL, seed=2004)


def test_symdir_bfs_partition(orc):
    import hessian_assembly_b200 as mad
    import torch
    n = 60
    ps = mi.param_static(n, 3, np.float64)
    ctx = mad.Context(ps["V"], ps["F"], 2, "float64")  # no positions: graph growth
    terms = terms_for(ps, "float64")
    g = torch.zeros((ps["V"], 2), dtype=torch.float64, device="cuda")
    H = torch.zeros((ctx.info.capacity_blocks, 2, 2), dtype=torch.float64, device="cuda")
    ctx.mad_eval(to_dev(ps["UV"]), terms, g, H)
    rp, ci, nnzb = gpu_pattern(ctx)
    og, oH, oE = orc.eval(ps["V"], 2, ps["UV"], 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])
    assert_close("g", g.cpu().numpy(), og, "float64")
    assert_close("H", H[:nnzb].cpu().numpy(), oH, "float64")


def test_hvp_cloth_with_springs_and_inertia(orc):
    import hessian_assembly_b200 as mad
    import torch
    from _parity import cloth_context, cloth_terms
    n = 50
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 5, 0, np.float64)
    v = mi.probe_vector(st["V"], 3, 6, np.float64)
    y = torch.zeros((st["V"], 3), dtype=torch.float64, device="cuda")
    ctx.mad_hvp(to_dev(x), cloth_terms(st, "float64", 3), to_dev(v), y)
    rp, ci = orc.pattern(st["V"], st["F"])
    og, oH, oE = orc.eval(st["V"], 3, x, 3, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"],
                          xt=st["xt"], w=st["w"])
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(st["V"], 3, rp, ci, oH, v), "float64")


def fan_problem(m, seed, dtype):
    """A hub vertex 0 with m faces around it (rim on the unit circle): the
    hub's row holds m faces, more than one row of the face table."""
    rng = np.random.default_rng(seed)
    ang = 2 * np.pi * np.arange(m) / m
    X = np.concatenate([[[0.0, 0.0]], np.stack([np.cos(ang), np.sin(ang)], 1)])
    F = np.array([[0, 1 + i, 1 + (i + 1) % m] for i in range(m)], np.int32)
    Dm = np.stack([X[F[:, 1]] - X[F[:, 0]], X[F[:, 2]] - X[F[:, 0]]], axis=2)
    Minv = np.linalg.inv(Dm)
    area = 0.5 * np.abs(np.linalg.det(Dm))
    UV = X + 0.02 * rng.standard_normal(X.shape)
    return X, F, Minv.astype(dtype), area.astype(dtype), UV.astype(dtype)


@pytest.mark.parametrize("dtype", ["float32", "float64"])
@pytest.mark.parametrize("flags", [0, FULL, PATCH])
def test_symdir_high_valence_fan(orc, dtype, flags):
    import hessian_assembly_b200 as mad
    import torch
    m = 40
    X, F, Minv, area, UV = fan_problem(m, 11, np.dtype(dtype))
    V = m + 1
    ctx = mad.Context(V, F, 2, dtype, part_xyz=X)
    terms = mad.Terms(mask=4, flags=flags, face_Minv=to_dev(Minv.reshape(-1, 4), dtype),
                      face_area=to_dev(area, dtype))
    tt = getattr(torch, dtype)
    g = torch.full((V, 2), float("nan"), dtype=tt, device="cuda")
    H = torch.full((ctx.info.capacity_blocks, 2, 2), float("nan"), dtype=tt, device="cuda")
    e = torch.zeros(1, dtype=torch.float64, device="cuda")
    ctx.mad_eval(to_dev(UV, dtype), terms, g, H, e)
    v = mi.probe_vector(V, 2, 12, np.dtype(dtype))
    y = torch.full((V, 2), float("nan"), dtype=tt, device="cuda")
    ctx.mad_hvp(to_dev(UV, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    rp, ci, nnzb = gpu_pattern(ctx)
    og, oH, oE = orc.eval(V, 2, UV, 4, rp, ci, F=F, Minv=Minv, area=area)
    assert_close("g", g.cpu().numpy(), og, dtype)
    assert_close("H", H[:nnzb].cpu().numpy(), oH, dtype)
    assert abs(e.item() - oE) <= ETOL[dtype] * abs(oE)
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 2, rp, ci, oH, v), dtype)


@pytest.mark.parametrize("flags", [0, PATCH])
def test_symdir_with_springs_inertia_and_pairs(orc, flags):
    """All four term types on a dof-2 mesh: edge terms store their blocks,
    face terms add to them, pair blocks sit at shifted positions."""
    import hessian_assembly_b200 as mad
    import torch
    n, dtype = 24, "float64"
    ps = mi.param_static(n, 31, np.float64)
    V, F, X, UV = ps["V"], ps["F"], ps["X"], ps["UV"]
    ctx = mad.Context(V, F, 2, dtype, part_xyz=X, max_pairs=200)
    edges = ctx.mad_edges().cpu().numpy()
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1)
    xt = X + 0.01 * mi.probe_vector(V, 2, 32, np.float64)
    k, w, kp = 3.0, 50.0, 7.0
    rng = np.random.default_rng(33)
    pairs = []
    while len(pairs) < 80:
        a, b = rng.integers(0, V, 2)
        if a != b and not mi.grid_adjacent(n, a, b):
            pairs.append((min(a, b), max(a, b)))
    pairs = np.unique(np.array(pairs, np.int32), axis=0)
    prest = 0.9 * np.linalg.norm(UV[pairs[:, 0]] - UV[pairs[:, 1]], axis=1)
    ctx.mad_add_pairs(to_dev(pairs), to_dev(prest))
    mask = 1 | 2 | 4 | 8
    terms = mad.Terms(mask=mask, flags=flags, spring_rest=to_dev(L0), spring_k=k,
                      inertia_xt=to_dev(xt), inertia_w=w,
                      face_Minv=to_dev(ps["Minv"].reshape(-1, 4)), face_area=to_dev(ps["area"]),
                      pair_k=kp)
    g = torch.full((V, 2), float("nan"), dtype=torch.float64, device="cuda")
    H = torch.full((ctx.info.capacity_blocks, 2, 2), float("nan"), dtype=torch.float64,
                   device="cuda")
    e = torch.zeros(1, dtype=torch.float64, device="cuda")
    ctx.mad_eval(to_dev(UV), terms, g, H, e)
    v = mi.probe_vector(V, 2, 34, np.float64)
    y = torch.full((V, 2), float("nan"), dtype=torch.float64, device="cuda")
    ctx.mad_hvp(to_dev(UV), terms, to_dev(v), y)
    torch.cuda.synchronize()
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F, pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(V, 2, UV, mask, orp, oci, edges=edges, L0=L0, k=k, xt=xt, w=w, F=F,
                          Minv=ps["Minv"], area=ps["area"], pairs=pairs, prest=prest, kp=kp)
    assert_close("g", g.cpu().numpy(), og, dtype)
    assert_close("H", H[:nnzb].cpu().numpy(), oH, dtype)
    assert abs(e.item() - oE) <= ETOL[dtype] * abs(oE)
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 2, orp, oci, oH, v), dtype)


@pytest.mark.parametrize("dtype", ["float32", "float64"])
def test_symdir_unaligned_caller_arrays(orc, dtype):
    """x and v handed in at an odd element offset (not aligned to a vertex's
    pair of values): the per-face passes fall back to element loads and the
    results match the aligned call."""
    import hessian_assembly_b200 as mad
    import torch
    n = 12
    ps = mi.param_static(n, 2400, np.dtype(dtype))
    V = ps["V"]
    ctx = mad.Context(V, ps["F"], 2, dtype, part_xyz=ps["X"])
    terms = terms_for(ps, dtype)
    tt = getattr(torch, dtype)
    v = mi.probe_vector(V, 2, 2401, np.dtype(dtype))
    xa = to_dev(ps["UV"], dtype)
    va = to_dev(v, dtype)
    xb_buf = torch.zeros(2 * V + 1, dtype=tt, device="cuda")
    vb_buf = torch.zeros(2 * V + 1, dtype=tt, device="cuda")
    xb_buf[1:] = xa.reshape(-1)
    vb_buf[1:] = va.reshape(-1)
    xb, vb = xb_buf[1:], vb_buf[1:]
    assert xb.data_ptr() % (2 * xb.element_size()) != 0
    out = []
    for x_, v_ in ((xa, va), (xb, vb)):
        g = torch.zeros((V, 2), dtype=tt, device="cuda")
        H = torch.zeros((ctx.info.capacity_blocks, 2, 2), dtype=tt, device="cuda")
        y = torch.zeros((V, 2), dtype=tt, device="cuda")
        ctx.mad_eval(x_, terms, g, H)
        ctx.mad_hvp(x_, terms, v_, y)
        torch.cuda.synchronize()
        out.append((g.cpu().numpy(), H.cpu().numpy(), y.cpu().numpy()))
    for a, b in zip(out[0], out[1]):
        np.testing.assert_array_equal(a, b)
