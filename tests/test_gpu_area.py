"""Area preservation on 3D triangles (a face term with a 9-variable stencil,
3x3 blocks among three vertices) through the row-streaming kernel, the
per-face Hessian-vector pass and the allocation-free energy, against the fp64
oracle."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, assert_close, cloth_context, gpu_pattern, run_eval, to_dev

pytestmark = pytest.mark.gpu
FULL = 1
GEN = 8
KA = 2.0e3


def rest_area(X, F):
    return 0.5 * np.linalg.norm(np.cross(X[F[:, 1]] - X[F[:, 0]], X[F[:, 2]] - X[F[:, 0]]), axis=1)


def area_terms(st, dtype, mask, flags=0):
    import hessian_assembly_b200 as mad
    A0 = rest_area(st["X"], st["F"]).astype(dtype)
    return mad.Terms(mask=mask, flags=flags, spring_rest=to_dev(st["L0"], dtype),
                     spring_k=st["k"], inertia_xt=to_dev(st["xt"], dtype), inertia_w=st["w"],
                     face_area=to_dev(A0, dtype), area_k=KA, pair_k=mi.PAIR_K), A0


def check(orc, n, dtype, mask=1 | 2 | 16, flags=0, seed=5000, pairs=None):
    import torch
    ctx, st = cloth_context(n, dtype, max_pairs=0 if pairs is None else len(pairs) + 8)
    x = mi.cloth_x(n, seed, 0, np.dtype(dtype))
    # a visible membrane strain: stretch the sheet a little
    x = (x * np.array([1.02, 0.99, 1.0])).astype(dtype)
    prest = None
    if pairs is not None:
        prest = mi.pair_rest(x, pairs, np.dtype(dtype))
        ctx.mad_add_pairs(to_dev(pairs), to_dev(prest, dtype))
    terms, A0 = area_terms(st, dtype, mask, flags)
    g, H, E = run_eval(ctx, x, terms, dtype)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(st["V"], st["F"], pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(st["V"], 3, x, mask, orp, oci, edges=st["edges"], L0=st["L0"],
                          k=st["k"], xt=st["xt"], w=st["w"], F=st["F"], area=A0, ka=KA,
                          pairs=pairs, prest=prest, kp=mi.PAIR_K)
    assert_close("g", g, og, dtype)
    assert_close("H", H[:nnzb], oH, dtype)
    assert abs(E - oE) <= ETOL[dtype] * abs(oE)
    v = mi.probe_vector(st["V"], 3, seed + 1, np.dtype(dtype))
    y = torch.full((st["V"], 3), float("nan"), dtype=getattr(torch, dtype), device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(st["V"], 3, orp, oci, oH, v), dtype)
    return ctx, st, x, terms, oE


@pytest.mark.parametrize("flags", [0, FULL, GEN])
@pytest.mark.parametrize("mask", [16, 1 | 2 | 16])
def test_area_cloth_fp64(orc, mask, flags):
    check(orc, 20, "float64", mask, flags)


def test_area_cloth_300x300_fp32(orc):
    check(orc, 300, "float32")


def test_area_cloth_1000x1000_fp32(orc):
    # the timed configuration (springs + inertia + area on the 1000^2 cloth)
    check(orc, 1000, "float32", seed=1007)


def test_area_cloth_300x300_fp32_generic_ad(orc):
    check(orc, 300, "float32", flags=GEN, seed=5003)


def test_area_with_pairs(orc):
    pairs = mi.random_pairs(24, 60, 5001, 0)
    check(orc, 24, "float64", 1 | 2 | 8 | 16, pairs=pairs)


def test_area_fan_overflow_rows(orc):
    """A hub shared by 40 faces in 3D: its row holds more faces than the slot
    table; rim vertices are lifted so every face is strained."""
    import hessian_assembly_b200 as mad
    import torch
    m = 40
    ang = 2 * np.pi * np.arange(m) / m
    X = np.concatenate([[[0.0, 0.0, 0.0]], np.stack([np.cos(ang), np.sin(ang), 0 * ang], 1)])
    F = np.array([[0, 1 + i, 1 + (i + 1) % m] for i in range(m)], np.int32)
    V = m + 1
    rng = np.random.default_rng(5002)
    x = X + 0.05 * rng.standard_normal(X.shape)
    A0 = rest_area(X, F)
    ctx = mad.Context(V, F, 3, "float64", part_xyz=X)
    terms = mad.Terms(mask=16, face_area=to_dev(A0), area_k=KA)
    g, H, E = run_eval(ctx, x, terms, "float64")
    rp, ci, nnzb = gpu_pattern(ctx)
    og, oH, oE = orc.eval(V, 3, x, 16, rp, ci, F=F, area=A0, ka=KA)
    assert_close("g", g, og, "float64")
    assert_close("H", H[:nnzb], oH, "float64")
    v = rng.standard_normal((V, 3))
    y = torch.zeros((V, 3), dtype=torch.float64, device="cuda")
    ctx.mad_hvp(to_dev(x), terms, to_dev(v), y)
    torch.cuda.synchronize()
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 3, rp, ci, oH, v), "float64")


def test_area_noalloc_energy(orc):
    import hessian_assembly_b200 as mad
    import torch
    ctx, st, x, terms, oE = check(orc, 16, "float64")
    e = torch.zeros(1, dtype=torch.float64, device="cuda")
    st_code = mad.mad_energy_noalloc(st["V"], 3, to_dev(x), terms, e, edges=ctx.mad_edges(),
                                     F=to_dev(st["F"]))
    assert st_code == mad.MAD_OK
    torch.cuda.synchronize()
    assert abs(e.item() - oE) <= ETOL["float64"] * abs(oE)


def test_area_refusals():
    import hessian_assembly_b200 as mad
    import torch
    ctx, st = cloth_context(6, "float32")
    terms, _ = area_terms(st, "float32", 16, flags=mad.MAD_EVAL_PATCH_STAGED)
    g = torch.zeros((st["V"], 3), device="cuda")
    H = torch.zeros((ctx.info.capacity_blocks, 3, 3), device="cuda")
    x = to_dev(mi.cloth_x(6, 1, 0, np.float32))
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_eval(x, terms, g, H)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_jacobian_shape(16)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    ps = mi.param_static(6, 3, np.float32)
    c2 = mad.Context(ps["V"], ps["F"], 2, "float32")
    t2 = mad.Terms(mask=16, face_area=to_dev(ps["area"]), area_k=1.0)
    with pytest.raises(mad.MadError) as ei:
        c2.mad_eval(to_dev(ps["UV"]), t2, torch.zeros((ps["V"], 2), device="cuda"),
                    torch.zeros((c2.info.capacity_blocks, 2, 2), device="cuda"))
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
