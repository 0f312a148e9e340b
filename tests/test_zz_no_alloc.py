"""mad_energy_noalloc: the total energy without a context and without any
device allocation.

It is for callers that cannot allocate device memory: code whose GPU memory is
owned by another allocator, and loops that must not allocate once set up.
Such callers cannot create a context, because mad_create allocates. The entry
point keeps its per-block partial sums in a fixed device array of the library.
The array is shared by all calls and keeps the previous call's values, so each
test calls the entry point twice in a row (different inputs, the second call
smaller where that matters) and compares both results with the energy
mad_eval returns for the same inputs and with the fp64 oracle's energy. It
uses the same energy tolerance as the other parity tests.

This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, cloth_context, cloth_terms, gpu_pattern, run_eval, to_dev


def rel(a, b):
    return abs(a - b) / max(abs(b), 1e-300)


def noalloc(V, dof, x, terms, dtype, **kw):
    import torch

    import hessian_assembly_b200 as mad
    e = torch.full((1,), float("nan"), dtype=torch.float64, device="cuda")
    st_code = mad.mad_energy_noalloc(V, dof, to_dev(x, dtype), terms, e, **kw)
    assert st_code == mad.MAD_OK
    torch.cuda.synchronize()
    return e.item()


@pytest.mark.gpu
def test_noalloc_energy_matches_eval_cloth_with_pairs_twice(orc):
    import hessian_assembly_b200 as mad
    n = 40
    ctx, st = cloth_context(n, "float32")
    mask = mad.MAD_TERM_SPRING | mad.MAD_TERM_INERTIA | mad.MAD_TERM_PAIR
    terms = cloth_terms(st, "float32", mask)
    edges = ctx.mad_edges()
    for step in (0, 1):
        x = mi.cloth_x(n, 2024, step, np.float32)
        pairs = mi.random_pairs(n, 60 + 20 * step, 2024, step)
        rest = mi.pair_rest(x, pairs, np.float32)
        dp, dr = to_dev(pairs), to_dev(rest)
        ctx.mad_add_pairs(dp, dr)
        _, _, e_ref = run_eval(ctx, x, terms, "float32")
        rp, ci, _ = gpu_pattern(ctx)
        _, _, e_orc = orc.eval(st["V"], 3, x, mask, rp, ci, edges=st["edges"], L0=st["L0"],
                               k=st["k"], xt=st["xt"], w=st["w"], pairs=pairs, prest=rest,
                               kp=mi.PAIR_K)
        e = noalloc(st["V"], 3, x, terms, "float32", edges=edges, pairs=dp, pair_rest=dr)
        assert rel(e, e_orc) <= ETOL["float32"], (step, e, e_orc)
        assert rel(e, e_ref) <= ETOL["float32"], (step, e, e_ref)


@pytest.mark.gpu
@pytest.mark.parametrize("mask", [4, 32, 4 | 32])  # SymDir, ARAP, both summed per face
def test_noalloc_energy_matches_eval_param_fp64_twice(orc, mask):
    import hessian_assembly_b200 as mad
    for n in (30, 17):  # a smaller second call must not pick up stale sums
        ps = mi.param_static(n, 77 + n, np.float64)
        ctx = mad.Context(ps["V"], ps["F"], 2, "float64", part_xyz=ps["X"])
        terms = mad.Terms(mask=mask, face_Minv=to_dev(ps["Minv"].reshape(-1, 4)),
                          face_area=to_dev(ps["area"]))
        _, _, e_ref = run_eval(ctx, ps["UV"], terms, "float64")
        rp, ci, _ = gpu_pattern(ctx)
        _, _, e_orc = orc.eval(ps["V"], 2, ps["UV"], mask, rp, ci, F=ps["F"], Minv=ps["Minv"],
                               area=ps["area"])
        e = noalloc(ps["V"], 2, ps["UV"], terms, "float64", F=to_dev(ps["F"]))
        assert rel(e, e_orc) <= ETOL["float64"], (n, e, e_orc)
        assert rel(e, e_ref) <= ETOL["float64"], (n, e, e_ref)


@pytest.mark.gpu
def test_noalloc_energy_springs_inertia_dof2_twice(orc):
    """Springs and inertia on a dof-2 mesh (the UV grid)."""
    import hessian_assembly_b200 as mad
    for n in (25, 12):
        ps = mi.param_static(n, 91 + n, np.float64)
        X = ps["X"]
        ctx = mad.Context(ps["V"], ps["F"], 2, "float64", part_xyz=X)
        edges = ctx.mad_edges()
        ed = edges.cpu().numpy()
        L0 = np.linalg.norm(X[ed[:, 0]] - X[ed[:, 1]], axis=1)
        terms = mad.Terms(mask=3, spring_rest=to_dev(L0), spring_k=50.0, inertia_xt=to_dev(X),
                          inertia_w=3.0)
        _, _, e_ref = run_eval(ctx, ps["UV"], terms, "float64")
        rp, ci, _ = gpu_pattern(ctx)
        _, _, e_orc = orc.eval(ps["V"], 2, ps["UV"], 3, rp, ci, edges=ed, L0=L0, k=50.0, xt=X,
                               w=3.0)
        e = noalloc(ps["V"], 2, ps["UV"], terms, "float64", edges=edges)
        assert rel(e, e_orc) <= ETOL["float64"], (n, e, e_orc)
        assert rel(e, e_ref) <= ETOL["float64"], (n, e, e_ref)


@pytest.mark.gpu
def test_noalloc_energy_area_dof3_twice(orc):
    """Area preservation (a dof-3 face term) with springs and inertia."""
    import hessian_assembly_b200 as mad
    for n in (18, 9):
        ctx, st = cloth_context(n, "float64")
        X, F = st["X"], st["F"]
        A0 = 0.5 * np.linalg.norm(np.cross(X[F[:, 1]] - X[F[:, 0]], X[F[:, 2]] - X[F[:, 0]]),
                                  axis=1)
        x = mi.cloth_x(n, 3030, n, np.float64) * np.array([1.02, 0.99, 1.0])
        terms = mad.Terms(mask=1 | 2 | 16, spring_rest=to_dev(st["L0"]), spring_k=st["k"],
                          inertia_xt=to_dev(st["xt"]), inertia_w=st["w"], face_area=to_dev(A0),
                          area_k=2.0e3)
        _, _, e_ref = run_eval(ctx, x, terms, "float64")
        rp, ci, _ = gpu_pattern(ctx)
        _, _, e_orc = orc.eval(st["V"], 3, x, 1 | 2 | 16, rp, ci, edges=st["edges"],
                               L0=st["L0"], k=st["k"], xt=st["xt"], w=st["w"], F=F, area=A0,
                               ka=2.0e3)
        e = noalloc(st["V"], 3, x, terms, "float64", edges=ctx.mad_edges(), F=to_dev(F))
        assert rel(e, e_orc) <= ETOL["float64"], (n, e, e_orc)
        assert rel(e, e_ref) <= ETOL["float64"], (n, e, e_ref)


@pytest.mark.gpu
def test_noalloc_index_out_of_range_gives_nan():
    """A vertex index outside [0, V) is skipped by the kernel's own check and
    shows up as a NaN energy; the next call with good input is finite again."""
    import hessian_assembly_b200 as mad
    n = 12
    st = mi.cloth_static(n, np.float32)
    x = mi.cloth_x(n, 5, 0, np.float32)
    terms = cloth_terms(st, "float32", mad.MAD_TERM_SPRING)
    bad = st["edges"].copy()
    bad[7, 1] = st["V"]  # one past the last vertex
    e = noalloc(st["V"], 3, x, terms, "float32", edges=to_dev(bad))
    assert np.isnan(e)
    e = noalloc(st["V"], 3, x, terms, "float32", edges=to_dev(st["edges"]))
    assert np.isfinite(e)


def test_noalloc_rejects_sizes_beyond_its_fixed_scratch():
    """More than 65,536 x 256 terms is refused before any device work."""
    import hessian_assembly_b200 as mad
    lib = mad.load_library()
    t = mad.mad_terms(mask=mad.MAD_TERM_SPRING | mad.MAD_TERM_INERTIA,
                      spring_rest=ctypes.c_void_p(256), inertia_xt=ctypes.c_void_p(256))
    fake = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    st = lib.mad_energy_noalloc(10_000_000, 3, mad.MAD_F32, fake, ctypes.byref(t), 7_000_000,
                                fake, 0, None, 0, None, None, fake, None)
    assert st == mad.MAD_ERR_CAPACITY
    st = lib.mad_energy_noalloc(-1, 3, mad.MAD_F32, fake, ctypes.byref(t), 0, None, 0, None, 0,
                                None, None, fake, None)
    assert st == mad.MAD_ERR_INVALID_ARG
