"""ARAP parameterization (dof 2, the same face inputs as symmetric
Dirichlet) through the row-streaming kernel, the per-face Hessian-vector
pass and the allocation-free energy, alone and summed with symmetric
Dirichlet, springs, inertia and runtime pairs, against the fp64 oracle."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, assert_close, gpu_pattern, to_dev
from test_gpu_symdir import fan_problem, setup

pytestmark = pytest.mark.gpu
FULL = 1
PATCH = 4
ARAP = 32
SYMDIR = 4


def run(orc, ctx, V, F, UV, Minv, area, mask, dtype, flags=0, seed=7, extra=None, oextra=None,
        pattern=None):
    import hessian_assembly_b200 as mad
    import torch
    tt = getattr(torch, dtype)
    terms = mad.Terms(mask=mask, flags=flags, face_Minv=to_dev(Minv.reshape(-1, 4), dtype),
                      face_area=to_dev(area, dtype), **(extra or {}))
    x = to_dev(UV, dtype)
    g = torch.full((V, 2), float("nan"), dtype=tt, device="cuda")
    H = torch.full((ctx.info.capacity_blocks, 2, 2), float("nan"), dtype=tt, device="cuda")
    e = torch.zeros(1, dtype=torch.float64, device="cuda")
    ctx.mad_eval(x, terms, g, H, e)
    v = mi.probe_vector(V, 2, seed, np.dtype(dtype))
    y = torch.full((V, 2), float("nan"), dtype=tt, device="cuda")
    ctx.mad_hvp(x, terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    rp, ci, nnzb = gpu_pattern(ctx)
    if pattern is not None:
        np.testing.assert_array_equal(rp, pattern[0])
        np.testing.assert_array_equal(ci, pattern[1])
    og, oH, oE = orc.eval(V, 2, UV, mask, rp, ci, F=F, Minv=Minv, area=area, **(oextra or {}))
    assert_close("g", g.cpu().numpy(), og, dtype)
    assert_close("H", H[:nnzb].cpu().numpy(), oH, dtype)
    assert abs(e.item() - oE) <= ETOL[dtype] * abs(oE)
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 2, rp, ci, oH, v), dtype)
    return terms, oE


@pytest.mark.parametrize("flags", [0, FULL, 8])
@pytest.mark.parametrize("mask", [ARAP, ARAP | SYMDIR])
@pytest.mark.parametrize("dtype", ["float32", "float64"])
def test_arap_grid(orc, dtype, mask, flags):
    ctx, ps = setup(37, dtype, seed=3001)
    run(orc, ctx, ps["V"], ps["F"], ps["UV"], ps["Minv"], ps["area"], mask, dtype, flags,
        pattern=orc.pattern(ps["V"], ps["F"]))


def test_arap_500x500_fp32(orc):
    ctx, ps = setup(500, "float32", seed=3002)
    run(orc, ctx, ps["V"], ps["F"], ps["UV"], ps["Minv"], ps["area"], ARAP, "float32")


@pytest.mark.parametrize("dtype", ["float32", "float64"])
@pytest.mark.parametrize("flags", [0, FULL])
def test_arap_high_valence_fan(orc, dtype, flags):
    import hessian_assembly_b200 as mad
    m = 40
    X, F, Minv, area, UV = fan_problem(m, 3003, np.dtype(dtype))
    ctx = mad.Context(m + 1, F, 2, dtype, part_xyz=X)
    run(orc, ctx, m + 1, F, UV, Minv, area, ARAP | SYMDIR, dtype, flags)


def test_arap_with_springs_inertia_and_pairs(orc):
    import hessian_assembly_b200 as mad
    n, dtype = 24, "float64"
    ps = mi.param_static(n, 3004, np.float64)
    V, F, X, UV = ps["V"], ps["F"], ps["X"], ps["UV"]
    ctx = mad.Context(V, F, 2, dtype, part_xyz=X, max_pairs=200)
    edges = ctx.mad_edges().cpu().numpy()
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1)
    xt = X + 0.01 * mi.probe_vector(V, 2, 3005, np.float64)
    rng = np.random.default_rng(3006)
    pairs = []
    while len(pairs) < 80:
        a, b = rng.integers(0, V, 2)
        if a != b and not mi.grid_adjacent(n, a, b):
            pairs.append((min(a, b), max(a, b)))
    pairs = np.unique(np.array(pairs, np.int32), axis=0)
    prest = 0.9 * np.linalg.norm(UV[pairs[:, 0]] - UV[pairs[:, 1]], axis=1)
    ctx.mad_add_pairs(to_dev(pairs), to_dev(prest))
    k, w, kp = 3.0, 50.0, 7.0
    run(orc, ctx, V, F, UV, ps["Minv"], ps["area"], 1 | 2 | 8 | ARAP, dtype,
        extra=dict(spring_rest=to_dev(L0), spring_k=k, inertia_xt=to_dev(xt), inertia_w=w,
                   pair_k=kp),
        oextra=dict(edges=edges, L0=L0, k=k, xt=xt, w=w, pairs=pairs, prest=prest, kp=kp),
        pattern=orc.pattern(V, F, pairs))


@pytest.mark.parametrize("mask", [ARAP, ARAP | SYMDIR])
def test_arap_noalloc_energy(orc, mask):
    import hessian_assembly_b200 as mad
    import torch
    ctx, ps = setup(30, "float64", seed=3007)
    terms, oE = run(orc, ctx, ps["V"], ps["F"], ps["UV"], ps["Minv"], ps["area"], mask,
                    "float64")
    e = torch.zeros(1, dtype=torch.float64, device="cuda")
    st = mad.mad_energy_noalloc(ps["V"], 2, to_dev(ps["UV"]), terms, e, F=to_dev(ps["F"]))
    assert st == mad.MAD_OK
    torch.cuda.synchronize()
    assert abs(e.item() - oE) <= ETOL["float64"] * abs(oE)


def test_arap_refusals():
    import hessian_assembly_b200 as mad
    import torch
    ctx, ps = setup(8, "float32", seed=3008)
    tp = mad.Terms(mask=ARAP, flags=PATCH, face_Minv=to_dev(ps["Minv"].reshape(-1, 4)),
                   face_area=to_dev(ps["area"]))
    g = torch.zeros((ps["V"], 2), device="cuda")
    H = torch.zeros((ctx.info.capacity_blocks, 2, 2), device="cuda")
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_eval(to_dev(ps["UV"]), tp, g, H)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_jacobian_shape(ARAP)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    st = mi.cloth_static(6, np.float32)
    c3 = mad.Context(st["V"], st["F"], 3, "float32")
    t3 = mad.Terms(mask=ARAP, face_Minv=to_dev(ps["Minv"].reshape(-1, 4)[:len(st["F"])]),
                   face_area=to_dev(ps["area"][:len(st["F"])]))
    with pytest.raises(mad.MadError) as ei:
        c3.mad_eval(to_dev(mi.cloth_x(6, 1, 0, np.float32)), t3,
                    torch.zeros((st["V"], 3), device="cuda"),
                    torch.zeros((c3.info.capacity_blocks, 3, 3), device="cuda"))
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
