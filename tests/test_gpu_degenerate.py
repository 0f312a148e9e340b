"""Degenerate meshes through every entry point: vertices without faces
(inertia only, diagonal pattern) and the empty mesh."""
import numpy as np
import pytest

from _parity import assert_close, gpu_pattern, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["float32", "float64"])
def test_isolated_vertices_eval_hvp_jacobian_energy(orc, dtype):
    import hessian_assembly_b200 as mad
    import torch
    V = 1000
    rng = np.random.default_rng(4000)
    x = rng.standard_normal((V, 3)).astype(dtype)
    xt = rng.standard_normal((V, 3)).astype(dtype)
    v = rng.standard_normal((V, 3)).astype(dtype)
    w = 7.0
    ctx = mad.Context(V, np.zeros((0, 3), np.int32), 3, dtype)
    assert ctx.info.E == 0 and ctx.info.nnzb_base == V
    terms = mad.Terms(mask=mad.MAD_TERM_SPRING | mad.MAD_TERM_INERTIA, spring_rest=None,
                      inertia_xt=to_dev(xt, dtype), inertia_w=w)
    tt = getattr(torch, dtype)
    g = torch.full((V, 3), float("nan"), dtype=tt, device="cuda")
    H = torch.full((ctx.info.capacity_blocks, 3, 3), float("nan"), dtype=tt, device="cuda")
    e = torch.zeros(1, dtype=torch.float64, device="cuda")
    ctx.mad_eval(to_dev(x, dtype), terms, g, H, e)
    y = torch.full((V, 3), float("nan"), dtype=tt, device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    rp, ci, nnzb = gpu_pattern(ctx)
    np.testing.assert_array_equal(rp, np.arange(V + 1))
    np.testing.assert_array_equal(ci, np.arange(V))
    og, oH, oE = orc.eval(V, 3, x, 2, rp, ci, xt=xt, w=w)
    assert_close("g", g.cpu().numpy(), og, dtype)
    assert_close("H", H[:nnzb].cpu().numpy(), oH, dtype)
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 3, rp, ci, oH, v), dtype)
    assert abs(e.item() - oE) <= 1e-5 * abs(oE)
    # the Jacobian: one row per coordinate, its single nonzero sqrt(w)
    rows, nnz = ctx.mad_jacobian_shape(3)
    assert (rows, nnz) == (3 * V, 3 * V)
    jrp = torch.zeros(rows + 1, dtype=torch.int64, device="cuda")
    jci = torch.zeros(nnz, dtype=torch.int32, device="cuda")
    r = torch.zeros(rows, dtype=tt, device="cuda")
    J = torch.zeros(nnz, dtype=tt, device="cuda")
    ctx.mad_jacobian_pattern(3, jrp, jci)
    ctx.mad_jacobian(to_dev(x, dtype), terms, r, J)
    torch.cuda.synchronize()
    orr, orp, oci, oJ = orc.jacobian(V, 3, x, 3, edges=np.zeros((0, 2), np.int32),
                                     L0=np.zeros(0), k=1.0, xt=xt, w=w)
    np.testing.assert_array_equal(jrp.cpu().numpy(), orp)
    np.testing.assert_array_equal(jci.cpu().numpy(), oci)
    assert_close("r", r.cpu().numpy(), orr, dtype)
    assert_close("J", J.cpu().numpy(), oJ, dtype)


def test_empty_mesh_every_entry_point():
    import hessian_assembly_b200 as mad
    import torch
    ctx = mad.Context(0, np.zeros((0, 3), np.int32), 3, "float32")
    terms = mad.Terms(mask=3)
    e = torch.full((1,), float("nan"), dtype=torch.float64, device="cuda")
    z = torch.empty((0, 3), dtype=torch.float32, device="cuda")
    zH = torch.empty((0, 3, 3), dtype=torch.float32, device="cuda")
    ctx.mad_eval(z, terms, z, zH, e)
    ctx.mad_hvp(z, terms, z, z)
    assert ctx.mad_jacobian_shape(3) == (0, 0)
    jrp = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    ctx.mad_jacobian_pattern(3, jrp, None)
    ctx.mad_jacobian(z, terms, None, None)
    torch.cuda.synchronize()
    assert e.item() == 0.0
    assert jrp.item() == 0
    assert ctx.mad_status_sync() == 0
