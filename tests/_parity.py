"""Shared helpers for the GPU parity tests: build seeded workloads, run them
through the C ABI (via the Python binding) and compare with the fp64 oracle.

Tolerances: fp32 max|gpu - oracle| <= 2e-5 * max|oracle| per array, fp64
<= 1e-12 * max|oracle|; CSR row_ptr / col_idx bit-exact.
"""
import numpy as np

import mesh_inputs as mi

TOL = {"float32": 2e-5, "float64": 1e-12}
ETOL = {"float32": 1e-5, "float64": 1e-10}


def torch_mod():
    import torch
    return torch


def max_rel(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max() if ref.size else 0.0
    err = np.abs(gpu - ref).max() if ref.size else 0.0
    return err / scale if scale > 0 else err


def assert_close(name, gpu, ref, dtype):
    r = max_rel(gpu, ref)
    assert r <= TOL[dtype], f"{name}: max rel err {r:.3e} > {TOL[dtype]:.0e}"
    return r


def to_dev(a, dtype=None):
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(getattr(torch, dtype))
    return t.cuda()


def grid_part_xyz(n):
    X, _ = mi.grid_mesh(n, 3)
    return X


def cloth_context(n, dtype="float32", part="rcb", **kw):
    import hessian_assembly_b200 as mad
    st = mi.cloth_static(n, np.dtype(dtype))
    xyz = grid_part_xyz(n) if part == "rcb" else None
    ctx = mad.Context(st["V"], st["F"], 3, dtype, part_xyz=xyz, **kw)
    return ctx, st


def cloth_terms(st, dtype, mask, flags=0):
    import hessian_assembly_b200 as mad
    return mad.Terms(mask=mask, flags=flags, spring_rest=to_dev(st["L0"], dtype),
                     spring_k=st["k"], inertia_xt=to_dev(st["xt"], dtype),
                     inertia_w=st["w"], pair_k=mi.PAIR_K)


def gpu_pattern(ctx):
    torch = torch_mod()
    rp, ci, nz = ctx.mad_pattern()
    torch.cuda.synchronize()
    nnzb = int(nz.cpu()[0])
    return rp.cpu().numpy().copy(), ci[:nnzb].cpu().numpy().copy(), nnzb


def run_eval(ctx, x_np, terms, dtype, energy=True):
    torch = torch_mod()
    V = ctx.info.V
    dof = ctx.info.dof
    x = to_dev(x_np, dtype)
    g = torch.full((V, dof), float("nan"), dtype=getattr(torch, dtype), device="cuda")
    H = torch.full((max(ctx.info.capacity_blocks, 1), dof, dof), float("nan"),
                   dtype=getattr(torch, dtype), device="cuda")
    e = torch.zeros(1, dtype=torch.float64, device="cuda") if energy else None
    ctx.mad_eval(x, terms, g, H, e)
    torch.cuda.synchronize()
    return g.cpu().numpy(), H.cpu().numpy(), (float(e.cpu()[0]) if energy else None)


def check_cloth(orc, n, dtype="float32", mask=3, flags=0, step=0, seed=1002, part="rcb",
                pairs=None, prest=None, ctx=None, st=None, **kw):
    """Full-array parity of one cloth evaluation; returns the error summary."""
    if ctx is None:
        ctx, st = cloth_context(n, dtype, part, **kw)
    x = mi.cloth_x(n, seed, step, np.dtype(dtype))
    terms = cloth_terms(st, dtype, mask, flags)
    g, H, E = run_eval(ctx, x, terms, dtype)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(st["V"], st["F"], pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(st["V"], 3, x, mask, orp, oci, edges=st["edges"], L0=st["L0"],
                          k=st["k"], xt=st["xt"], w=st["w"], pairs=pairs, prest=prest,
                          kp=mi.PAIR_K)
    rg = assert_close("g", g, og, dtype)
    rH = assert_close("H", H[:nnzb], oH, dtype)
    rE = abs(E - oE) / max(abs(oE), 1e-300)
    assert rE <= ETOL[dtype], f"energy rel err {rE:.3e}"
    return {"g": rg, "H": rH, "E": rE, "ctx": ctx}
