"""Mass-spring cloth (springs + inertia): CUDA path vs the fp64 oracle.

Cases: the 10x10 and 100x100 grids in fp32 and fp64, the 1000x1000 grid at
full size (every entry of g and H compared), both seeding strategies, both
patch builders, single- vs many-patch partitions, a permuted vertex
numbering, single term types, and run-to-run determinism.
"""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import (assert_close, check_cloth, cloth_context, cloth_terms, gpu_pattern,
                     run_eval, to_dev)

pytestmark = pytest.mark.gpu

FULL = 1  # MAD_EVAL_FULL_STENCIL_AD
SCAT = 2  # MAD_EVAL_EDGE_SCATTER
PATCH = 4  # MAD_EVAL_PATCH_STAGED
GEN = 8  # MAD_EVAL_GENERIC_AD


@pytest.mark.parametrize("flags", [0, FULL, SCAT, FULL | SCAT, PATCH, PATCH | FULL, GEN])
@pytest.mark.parametrize("part", ["rcb", "bfs"])
def test_cloth_10x10(orc, flags, part):
    check_cloth(orc, 10, "float32", flags=flags, part=part, seed=1001)


@pytest.mark.parametrize("dtype", ["float32", "float64"])
@pytest.mark.parametrize("flags", [0, FULL, SCAT, PATCH, GEN])
def test_cloth_100x100(orc, dtype, flags):
    check_cloth(orc, 100, dtype, flags=flags, seed=1002)


@pytest.mark.parametrize("mask", [1, 2])
@pytest.mark.parametrize("flags", [0, SCAT, PATCH])
def test_single_term_types(orc, mask, flags):
    check_cloth(orc, 23, "float32", mask=mask, flags=flags)


@pytest.mark.parametrize("patch_faces", [4, 37, 100000])
@pytest.mark.parametrize("flags", [0, PATCH])
def test_partition_granularity(orc, patch_faces, flags):
    # the largest patches (100000 faces asked, capped at 256 owned vertices),
    # tiny patches (4), and an odd size
    check_cloth(orc, 17, "float64", patch_faces=patch_faces, flags=flags)


def test_cloth_1000x1000_full(orc):
    r = check_cloth(orc, 1000, "float32", seed=1003, step=0)
    assert r["ctx"].info.n_patches > 1000


def test_cloth_1000x1000_second_step_and_full_ad(orc):
    check_cloth(orc, 1000, "float32", seed=1003, step=7, flags=FULL)


def test_cloth_1000x1000_generic_ad(orc):
    # the spring energy as a plain expression, differentiated by the AD types alone
    check_cloth(orc, 1000, "float32", seed=1003, step=11, flags=GEN)


def test_generic_ad_refusals():
    import hessian_assembly_b200 as mad
    import torch
    ctx, st = cloth_context(6)
    x = to_dev(mi.cloth_x(6, 1, 0, np.float32))
    g = torch.zeros((st["V"], 3), device="cuda")
    H = torch.zeros((ctx.info.capacity_blocks, 3, 3), device="cuda")
    for flags, code in ((GEN | FULL, mad.MAD_ERR_INVALID_ARG), (GEN | PATCH, mad.MAD_ERR_UNIMPLEMENTED),
                        (GEN | SCAT, mad.MAD_ERR_UNIMPLEMENTED)):
        with pytest.raises(mad.MadError) as ei:
            ctx.mad_eval(x, cloth_terms(st, "float32", 3, flags), g, H)
        assert ei.value.status == code


def test_cloth_1000x1000_scatter(orc):
    check_cloth(orc, 1000, "float32", seed=1003, step=3, flags=SCAT)


def test_cloth_1000x1000_patch_staged(orc):
    check_cloth(orc, 1000, "float32", seed=1003, step=5, flags=PATCH)


@pytest.mark.parametrize("n,dtype,slot_bytes", [(40, "float64", 4), (190, "float32", 8)])
def test_permuted_vertex_numbering(orc, n, dtype, slot_bytes):
    # A random numbering: at 40^2 every column and edge id of a tile still
    # lies within 16 bits (compact row tables, irregular deltas); at 190^2
    # (36,100 vertices) they do not, and the wide tables are used.
    import hessian_assembly_b200 as mad
    st = mi.cloth_static(n, np.float64)
    V = st["V"]
    perm = np.random.default_rng(3).permutation(V)   # new id of old vertex
    inv = np.argsort(perm)
    F = perm[st["F"]].astype(np.int32)
    X = st["X"][inv]
    ctx = mad.Context(V, F, 3, dtype, part_xyz=X)
    assert ctx.info.row_slot_bytes == slot_bytes
    e = np.sort(perm[mi.grid_edges(n)], axis=1)
    edges = e[np.lexsort((e[:, 1], e[:, 0]))].astype(np.int32)
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1).astype(dtype)
    x = mi.cloth_x(n, 9, 0, np.float64)[inv].astype(dtype)
    xt = X.astype(dtype)
    terms = mad.Terms(mask=3, spring_rest=to_dev(L0), spring_k=st["k"], inertia_xt=to_dev(xt),
                      inertia_w=st["w"])
    g, H, E = run_eval(ctx, x, terms, dtype)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(V, 3, x, 3, orp, oci, edges=edges, L0=L0, k=st["k"], xt=xt, w=st["w"])
    assert_close("g", g, og, dtype)
    assert_close("H", H[:nnzb], oH, dtype)


def test_grid_uses_compact_row_tables():
    ctx, _ = cloth_context(1000)
    assert ctx.info.row_slot_bytes == 4
    ctx.close()


def test_deterministic_run_to_run():
    n = 200
    ctx, st = cloth_context(n)
    x = mi.cloth_x(n, 4, 0, np.float32)
    terms = cloth_terms(st, "float32", 3)
    g1, H1, E1 = run_eval(ctx, x, terms, "float32")
    g2, H2, E2 = run_eval(ctx, x, terms, "float32")
    nnzb = ctx.info.nnzb_base  # blocks past nnzb are capacity slack (untouched)
    assert np.array_equal(g1, g2) and np.array_equal(H1[:nnzb], H2[:nnzb]) and E1 == E2


def test_missing_term_array_is_rejected():
    import hessian_assembly_b200 as mad
    import torch
    ctx, st = cloth_context(5)
    terms = mad.Terms(mask=1, spring_k=1.0)  # no rest lengths
    x = torch.zeros((25, 3), device="cuda")
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_eval(x, terms, torch.zeros_like(x), torch.zeros((ctx.info.capacity_blocks, 3, 3), device="cuda"))
    assert ei.value.status == mad.MAD_ERR_INVALID_ARG
    terms = mad.Terms(mask=4)  # symmetric Dirichlet needs dof 2
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_eval(x, terms, torch.zeros_like(x), torch.zeros((ctx.info.capacity_blocks, 3, 3), device="cuda"))
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED


def test_eval_host_matches_device(orc):
    import torch
    n = 30
    ctx, st = cloth_context(n)
    x = mi.cloth_x(n, 2, 0, np.float32)
    terms = cloth_terms(st, "float32", 3)
    g, H, E = run_eval(ctx, x, terms, "float32")
    nnzb = ctx.info.nnzb_base
    hx = torch.from_numpy(x).pin_memory()
    hg = torch.zeros((st["V"], 3)).pin_memory()
    hH = torch.zeros((nnzb, 3, 3)).pin_memory()
    he = torch.zeros(1, dtype=torch.float64)
    ctx.mad_eval_host(hx, terms, hg, hH, he)
    assert np.array_equal(hg.numpy(), g)
    assert np.array_equal(hH.numpy(), H[:nnzb])
    assert he.item() == E


@pytest.mark.parametrize("n,dtype", [(100, "float64"), (1000, "float32")])
def test_cloth_hvp(orc, n, dtype):
    """The matrix-free product of springs + inertia (at 1000^2 the benched
    size) against the oracle's assembled H applied to the same direction."""
    import torch
    ctx, st = cloth_context(n, dtype)
    x = mi.cloth_x(n, 1010, 0, np.dtype(dtype))
    v = mi.probe_vector(st["V"], 3, 1011, np.dtype(dtype))
    terms = cloth_terms(st, dtype, 3)
    y = torch.full((st["V"], 3), float("nan"), dtype=getattr(torch, dtype), device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    orp, oci = orc.pattern(st["V"], st["F"])
    _, oH, _ = orc.eval(st["V"], 3, x, 3, orp, oci, edges=st["edges"], L0=st["L0"], k=st["k"],
                        xt=st["xt"], w=st["w"])
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(st["V"], 3, orp, oci, oH, v), dtype)
