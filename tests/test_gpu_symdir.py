"""Symmetric-Dirichlet parameterization (dof 2, 2x2 blocks) and the
matrix-free Hessian-vector product: CUDA path vs the fp64 oracle."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, assert_close, gpu_pattern, to_dev

pytestmark = pytest.mark.gpu
FULL = 1


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


@pytest.mark.parametrize("flags", [0, FULL])
def test_symdir_small(orc, flags):
    check(orc, 10, "float32", flags)


@pytest.mark.parametrize("flags", [0, FULL])
def test_symdir_fp64(orc, flags):
    check(orc, 37, "float64", flags)


def test_symdir_500x500_full(orc):
    ctx = check(orc, 500, "float32")
    assert ctx.info.n_patches > 100


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
