"""mad_energy_noalloc: the total energy without a context and without any
device allocation.

It is for callers that cannot allocate device memory: code whose GPU memory is
owned by another allocator, and loops that must not allocate once set up.
Such callers cannot create a context, because mad_create allocates. The entry
point keeps its per-block partial sums in a fixed device array of the library.
The array is shared by all calls and keeps the previous call's values, so each
test calls the entry point twice in a row and compares both results with the
energy mad_eval returns for the same inputs. It uses the same energy tolerance
as the other parity tests.

This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, cloth_context, cloth_terms, run_eval, to_dev


def rel(a, b):
    return abs(a - b) / max(abs(b), 1e-300)


@pytest.mark.gpu
def test_noalloc_energy_matches_eval_cloth_with_pairs_twice():
    import torch

    import hessian_assembly_b200 as mad
    n = 40
    ctx, st = cloth_context(n, "float32")
    terms = cloth_terms(st, "float32", mad.MAD_TERM_SPRING | mad.MAD_TERM_INERTIA |
                        mad.MAD_TERM_PAIR)
    edges = ctx.mad_edges()
    for step in (0, 1):
        x = mi.cloth_x(n, 2024, step, np.float32)
        pairs = mi.random_pairs(n, 60 + 20 * step, 2024, step)
        rest = mi.pair_rest(x, pairs, np.float32)
        dp, dr = to_dev(pairs), to_dev(rest)
        ctx.mad_add_pairs(dp, dr)
        _, _, e_ref = run_eval(ctx, x, terms, "float32")
        e = torch.full((1,), float("nan"), dtype=torch.float64, device="cuda")
        st_code = mad.mad_energy_noalloc(st["V"], 3, to_dev(x), terms, e, edges=edges,
                                         pairs=dp, pair_rest=dr)
        assert st_code == mad.MAD_OK
        torch.cuda.synchronize()
        assert rel(e.item(), e_ref) <= ETOL["float32"], (step, e.item(), e_ref)


@pytest.mark.gpu
def test_noalloc_energy_matches_eval_symdir_fp64_twice():
    import torch

    import hessian_assembly_b200 as mad
    for n in (30, 17):  # a smaller second call must not pick up stale sums
        ps = mi.param_static(n, 77 + n, np.float64)
        ctx = mad.Context(ps["V"], ps["F"], 2, "float64", part_xyz=ps["X"])
        terms = mad.Terms(mask=mad.MAD_TERM_SYMDIR,
                          face_Minv=to_dev(ps["Minv"].reshape(-1, 4)), face_area=to_dev(ps["area"]))
        _, _, e_ref = run_eval(ctx, ps["UV"], terms, "float64")
        e = torch.zeros(1, dtype=torch.float64, device="cuda")
        st_code = mad.mad_energy_noalloc(ps["V"], 2, to_dev(ps["UV"]), terms, e,
                                         F=to_dev(ps["F"]))
        assert st_code == mad.MAD_OK
        torch.cuda.synchronize()
        assert rel(e.item(), e_ref) <= ETOL["float64"], (n, e.item(), e_ref)


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
