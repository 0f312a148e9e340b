"""Vertex-face terms (dof 3, a 4-vertex stencil with 12 variables) on the
cloth: the pattern holds the three (vertex, corner) pairs of each term,
inserted with mad_add_pairs; the terms are evaluated by their own pass after
the row kernel.  Parity of g, H, the energy and the Hessian-vector product
against the fp64 oracle, plus the refusals."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, assert_close, cloth_context, gpu_pattern, run_eval, to_dev

pytestmark = pytest.mark.gpu
VF = 64
KC = 50.0


def vf_terms_for(n, nvf, seed):
    st = mi.cloth_static(n, np.float64)
    F = st["F"]
    rng = np.random.default_rng(seed)
    vf = []
    while len(vf) < nvf:
        p, f = int(rng.integers(0, st["V"])), int(rng.integers(0, len(F)))
        if p not in F[f]:
            vf.append((p, f))
    vf = np.array(vf, np.int32)
    rest = 0.01 * rng.standard_normal(len(vf))
    pairs = np.array([(p, F[f][c]) for p, f in vf for c in range(3)], np.int32)
    return vf, rest, pairs


def check(orc, n, dtype, nvf, seed, mask=1 | 2 | VF, flags=0):
    import hessian_assembly_b200 as mad
    import torch
    vf, rest, pairs = vf_terms_for(n, nvf, seed)
    ctx, st = cloth_context(n, dtype, max_pairs=len(pairs) + 8, slack=0.6)
    ctx.mad_add_pairs(to_dev(pairs), to_dev(np.zeros(len(pairs)), dtype))
    x = mi.cloth_x(n, seed, 0, np.dtype(dtype))
    x = (x + 0.02 * mi.grid_spacing(n) * np.random.default_rng(seed + 1).standard_normal(x.shape)
         ).astype(dtype)
    terms = mad.Terms(mask=mask, flags=flags, spring_rest=to_dev(st["L0"], dtype), spring_k=st["k"],
                      inertia_xt=to_dev(st["xt"], dtype), inertia_w=st["w"],
                      vf=to_dev(vf), vf_rest=to_dev(rest, dtype), vf_k=KC)
    g, H, E = run_eval(ctx, x, terms, dtype)
    assert ctx.mad_status_sync() == mad.MAD_OK
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(st["V"], st["F"], pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(st["V"], 3, x, mask, orp, oci, edges=st["edges"], L0=st["L0"],
                          k=st["k"], xt=st["xt"], w=st["w"], F=st["F"], vf=vf,
                          vf_rest=rest.astype(dtype), kc=KC)
    assert_close("g", g, og, dtype)
    assert_close("H", H[:nnzb], oH, dtype)
    assert abs(E - oE) <= ETOL[dtype] * abs(oE)
    v = mi.probe_vector(st["V"], 3, seed + 2, np.dtype(dtype))
    y = torch.full((st["V"], 3), float("nan"), dtype=getattr(torch, dtype), device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(st["V"], 3, orp, oci, oH, v), dtype)
    return ctx


@pytest.mark.parametrize("dtype", ["float32", "float64"])
def test_vf_cloth(orc, dtype):
    check(orc, 30, dtype, 200, 6001)


@pytest.mark.parametrize("dtype", ["float32", "float64"])
def test_vf_cloth_generic_ad(orc, dtype):
    check(orc, 30, dtype, 200, 6004, flags=8)


def test_vf_only_terms(orc):
    # no row-kernel terms: rows are zeroed, the vertex-face pass alone adds
    check(orc, 20, "float64", 120, 6002, mask=VF)


def test_vf_many_terms_fp32(orc):
    check(orc, 200, "float32", 20000, 6003)


def test_vf_refusals():
    import hessian_assembly_b200 as mad
    import torch
    ctx, st = cloth_context(8, "float32", max_pairs=64)
    vf, rest, pairs = vf_terms_for(8, 4, 6004)
    x = to_dev(mi.cloth_x(8, 1, 0, np.float32))
    g = torch.zeros((st["V"], 3), device="cuda")
    H = torch.zeros((ctx.info.capacity_blocks, 3, 3), device="cuda")
    t = mad.Terms(mask=VF | 8, vf=to_dev(vf), vf_rest=to_dev(rest, "float32"), vf_k=1.0)
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_eval(x, t, g, H)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_jacobian_shape(VF)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    # blocks missing from the pattern (the pairs were not inserted): status error
    t = mad.Terms(mask=VF, vf=to_dev(vf), vf_rest=to_dev(rest, "float32"), vf_k=1.0)
    ctx.mad_eval(x, t, g, H)
    assert ctx.mad_status_sync() == mad.MAD_ERR_INDEX


# ---- installed sets (mad_add_vf): gathered per row, no atomics -------------

def check_installed(orc, n, dtype, nvf, seed, mask=1 | 2 | VF, flags=0, vf=None, rest=None):
    import hessian_assembly_b200 as mad
    import torch
    if vf is None:
        vf, rest, _ = vf_terms_for(n, nvf, seed)
    st = mi.cloth_static(n, np.float64)
    pairs = mi.vf_pairs(vf, st["F"])
    ctx, st = cloth_context(n, dtype, max_pairs=3 * len(vf) + 8, slack=0.6)
    ctx.mad_add_vf(to_dev(vf))
    assert ctx.mad_status_sync() == mad.MAD_OK
    x = mi.cloth_x(n, seed, 0, np.dtype(dtype))
    x = (x + 0.02 * mi.grid_spacing(n) * np.random.default_rng(seed + 1).standard_normal(x.shape)
         ).astype(dtype)
    terms = mad.Terms(mask=mask, flags=flags, spring_rest=to_dev(st["L0"], dtype),
                      spring_k=st["k"], inertia_xt=to_dev(st["xt"], dtype), inertia_w=st["w"],
                      vf=None, vf_rest=to_dev(rest, dtype), vf_k=KC)
    g, H, E = run_eval(ctx, x, terms, dtype)
    assert ctx.mad_status_sync() == mad.MAD_OK
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(st["V"], st["F"], pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(st["V"], 3, x, mask, orp, oci, edges=st["edges"], L0=st["L0"],
                          k=st["k"], xt=st["xt"], w=st["w"], F=st["F"], vf=vf,
                          vf_rest=rest.astype(dtype), kc=KC)
    assert_close("g", g, og, dtype)
    assert_close("H", H[:nnzb], oH, dtype)
    assert abs(E - oE) <= ETOL[dtype] * abs(oE)
    v = mi.probe_vector(st["V"], 3, seed + 2, np.dtype(dtype))
    y = torch.full((st["V"], 3), float("nan"), dtype=getattr(torch, dtype), device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(st["V"], 3, orp, oci, oH, v), dtype)
    return ctx, x, terms, g, H


@pytest.mark.parametrize("dtype", ["float32", "float64"])
@pytest.mark.parametrize("flags", [0, 8])
def test_vf_installed_cloth(orc, dtype, flags):
    check_installed(orc, 30, dtype, 200, 6101, flags=flags)


def test_vf_installed_only_terms(orc):
    check_installed(orc, 20, "float64", 120, 6102, mask=VF)


def test_vf_installed_1000x1000_benched_size(orc):
    # the timed configuration: 10^5 terms on the 1000^2 cloth
    n = 1000
    vf = mi.random_vf(n, 100_000, 1009, 0)
    rest = 0.001 * np.random.default_rng(1010).standard_normal(len(vf))
    check_installed(orc, n, "float32", 0, 6103, vf=vf, rest=rest)


def test_vf_installed_is_reproducible():
    n = 60
    vf, rest, _ = vf_terms_for(n, 900, 6104)
    import hessian_assembly_b200 as mad
    ctx, st = cloth_context(n, "float32", max_pairs=3 * len(vf) + 8, slack=0.6)
    ctx.mad_add_vf(to_dev(vf))
    x = mi.cloth_x(n, 6104, 0, np.float32)
    terms = mad.Terms(mask=1 | 2 | VF, spring_rest=to_dev(st["L0"], "float32"), spring_k=st["k"],
                      inertia_xt=to_dev(st["xt"], "float32"), inertia_w=st["w"],
                      vf_rest=to_dev(rest, "float32"), vf_k=KC)
    g1, H1, E1 = run_eval(ctx, x, terms, "float32")
    g2, H2, E2 = run_eval(ctx, x, terms, "float32")
    _, _, nnzb = gpu_pattern(ctx)
    assert np.array_equal(g1, g2) and np.array_equal(H1[:nnzb], H2[:nnzb]) and E1 == E2


def test_vf_installed_bad_terms_and_replacement(orc):
    import hessian_assembly_b200 as mad
    n = 16
    vf, rest, _ = vf_terms_for(n, 40, 6105)
    st = mi.cloth_static(n, np.float64)
    bad = vf.copy()
    bad[3, 0] = st["F"][bad[3, 1]][0]   # the vertex is a corner of its face
    bad[7, 1] = len(st["F"])            # face index out of range
    good = np.ones(len(vf), bool)
    good[[3, 7]] = False
    ctx, st = cloth_context(n, "float64", max_pairs=3 * len(vf) + 8, slack=0.6)
    ctx.mad_add_vf(to_dev(bad))
    assert ctx.mad_status_sync() == mad.MAD_ERR_INDEX
    x = mi.cloth_x(n, 6105, 0, np.float64)
    terms = mad.Terms(mask=VF, vf_rest=to_dev(rest), vf_k=KC)
    g, H, E = run_eval(ctx, x, terms, "float64")
    # the skipped terms' pairs are not in the pattern; the others evaluate as a set of their own
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(st["V"], st["F"], mi.vf_pairs(vf[good], st["F"]))
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(st["V"], 3, x, VF, orp, oci, F=st["F"], vf=vf[good],
                          vf_rest=rest[good], kc=KC)
    assert_close("g", g, og, "float64")
    assert_close("H", H[:nnzb], oH, "float64")
    # a new pair set drops the installed terms: vf = NULL is refused
    ctx.mad_add_pairs(to_dev(np.array([[0, 5]], np.int32)), to_dev(np.ones(1)))
    with pytest.raises(mad.MadError) as ei:
        run_eval(ctx, x, terms, "float64")
    assert ei.value.status == mad.MAD_ERR_INVALID_ARG
    # more terms than max_pairs / 3
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_add_vf(to_dev(np.zeros((len(vf) + 10, 2), np.int32)))
    assert ei.value.status == mad.MAD_ERR_CAPACITY


def test_vf_installed_on_permuted_numbering(orc):
    """Installed vertex-face terms on a randomly renumbered 190^2 cloth, whose
    column deltas pass 16 bits: the wide-table row kernel gathers the shares
    (the compact one does on grid numberings); eval and product vs the oracle."""
    import hessian_assembly_b200 as mad
    import torch
    n, dtype = 190, "float32"
    st = mi.cloth_static(n, np.float64)
    V = st["V"]
    perm = np.random.default_rng(7).permutation(V)   # new id of old vertex
    inv = np.argsort(perm)
    F = perm[st["F"]].astype(np.int32)
    X = st["X"][inv]
    vf0 = mi.random_vf(n, 1500, 6107, 0)
    vf = np.stack([perm[vf0[:, 0]], vf0[:, 1]], axis=1).astype(np.int32)  # faces keep their ids
    rest = 0.001 * np.random.default_rng(6108).standard_normal(len(vf))
    ctx = mad.Context(V, F, 3, dtype, part_xyz=X, max_pairs=3 * len(vf) + 8, slack=0.6)
    assert ctx.info.row_slot_bytes == 8
    ctx.mad_add_vf(to_dev(vf))
    assert ctx.mad_status_sync() == mad.MAD_OK
    e = np.sort(perm[mi.grid_edges(n)], axis=1)
    edges = e[np.lexsort((e[:, 1], e[:, 0]))].astype(np.int32)
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1)
    x = mi.cloth_x(n, 6107, 0, np.float64)[inv]
    x = (x + 0.02 * mi.grid_spacing(n) * np.random.default_rng(6109).standard_normal(x.shape)
         ).astype(dtype)
    xt = X
    mask = 1 | 2 | VF
    terms = mad.Terms(mask=mask, spring_rest=to_dev(L0, dtype), spring_k=st["k"],
                      inertia_xt=to_dev(xt, dtype), inertia_w=st["w"], vf=None,
                      vf_rest=to_dev(rest, dtype), vf_k=KC)
    g, H, E = run_eval(ctx, x, terms, dtype)
    assert ctx.mad_status_sync() == mad.MAD_OK
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F, mi.vf_pairs(vf, F))
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(V, 3, x, mask, orp, oci, edges=edges, L0=L0.astype(dtype), k=st["k"],
                          xt=xt.astype(dtype), w=st["w"], F=F, vf=vf,
                          vf_rest=rest.astype(dtype), kc=KC)
    assert_close("g", g, og, dtype)
    assert_close("H", H[:nnzb], oH, dtype)
    assert abs(E - oE) <= ETOL[dtype] * abs(oE)
    v = mi.probe_vector(V, 3, 6110, np.dtype(dtype))
    y = torch.full((V, 3), float("nan"), dtype=torch.float32, device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 3, orp, oci, oH, v), dtype)
