"""Residuals and sparse Jacobian of the vector-valued objective (scalar CSR,
term-major rows) through the C ABI, against the fp64 oracle: pattern
bit-exact, values within the parity tolerance.  J^T r = g is checked against
mad_eval's gradient, which holds at any size."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import assert_close, cloth_context, cloth_terms, run_eval, to_dev

pytestmark = pytest.mark.gpu


def gpu_jacobian(ctx, x, terms, dtype):
    import torch
    rows, nnz = ctx.mad_jacobian_shape(terms.mask)
    tt = getattr(torch, dtype)
    rp = torch.full((rows + 1,), -1, dtype=torch.int64, device="cuda")
    ci = torch.full((max(nnz, 1),), -1, dtype=torch.int32, device="cuda")
    r = torch.full((max(rows, 1),), float("nan"), dtype=tt, device="cuda")
    J = torch.full((max(nnz, 1),), float("nan"), dtype=tt, device="cuda")
    ctx.mad_jacobian_pattern(terms.mask, rp, ci)
    ctx.mad_jacobian(to_dev(x, dtype), terms, r, J)
    torch.cuda.synchronize()
    return (rp.cpu().numpy(), ci[:nnz].cpu().numpy(), r[:rows].cpu().numpy(),
            J[:nnz].cpu().numpy())


def check_cloth(orc, n, dtype, mask=3, seed=2100):
    ctx, st = cloth_context(n, dtype)
    x = mi.cloth_x(n, seed, 0, np.dtype(dtype))
    terms = cloth_terms(st, dtype, mask)
    rp, ci, r, J = gpu_jacobian(ctx, x, terms, dtype)
    orr, orp, oci, oJ = orc.jacobian(st["V"], 3, x, mask, edges=st["edges"], L0=st["L0"],
                                     k=st["k"], xt=st["xt"], w=st["w"])
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    assert_close("r", r, orr, dtype)
    assert_close("J", J, oJ, dtype)
    return ctx, st, x, terms, (rp, ci, r, J)


@pytest.mark.parametrize("n,dtype", [(10, "float32"), (100, "float32"), (100, "float64")])
@pytest.mark.parametrize("mask", [1, 2, 3])
def test_cloth_jacobian(orc, n, dtype, mask):
    check_cloth(orc, n, dtype, mask)


def test_cloth_jacobian_1000x1000_full(orc):
    check_cloth(orc, 1000, "float32")


def test_cloth_jacobian_transpose_residual_is_gradient():
    """J^T r = g (mad_eval's gradient) at the full 1000^2 size."""
    import scipy.sparse as sp
    n, dtype = 1000, "float32"
    ctx, st = cloth_context(n, dtype)
    x = mi.cloth_x(n, 2101, 0, np.float32)
    terms = cloth_terms(st, dtype, 3)
    rp, ci, r, J = gpu_jacobian(ctx, x, terms, dtype)
    g, _, _ = run_eval(ctx, x, terms, dtype, energy=False)
    Jm = sp.csr_matrix((J.astype(np.float64), ci, rp), shape=(len(r), st["V"] * 3))
    gt = Jm.T @ r.astype(np.float64)
    assert_close("J^T r", gt.astype(np.float32), g.reshape(-1).astype(np.float64), dtype)


@pytest.mark.parametrize("n,dtype", [(30, "float64"), (500, "float32")])
def test_symdir_jacobian(orc, n, dtype):
    import hessian_assembly_b200 as mad
    ps = mi.param_static(n, 2200 + n, np.dtype(dtype))
    ctx = mad.Context(ps["V"], ps["F"], 2, dtype, part_xyz=ps["X"])
    terms = mad.Terms(mask=4, face_Minv=to_dev(ps["Minv"].reshape(-1, 4), dtype),
                      face_area=to_dev(ps["area"], dtype))
    rp, ci, r, J = gpu_jacobian(ctx, ps["UV"], terms, dtype)
    orr, orp, oci, oJ = orc.jacobian(ps["V"], 2, ps["UV"], 4, F=ps["F"], Minv=ps["Minv"],
                                     area=ps["area"])
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    assert_close("r", r, orr, dtype)
    assert_close("J", J, oJ, dtype)


def test_jacobian_with_all_mesh_terms_dof2(orc):
    """Springs, inertia and faces together on a dof-2 mesh: three segments."""
    import hessian_assembly_b200 as mad
    n = 20
    ps = mi.param_static(n, 2300, np.float64)
    V, X = ps["V"], ps["X"]
    ctx = mad.Context(V, ps["F"], 2, "float64", part_xyz=X)
    edges = ctx.mad_edges().cpu().numpy()
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1)
    xt = X + 0.01 * mi.probe_vector(V, 2, 2301, np.float64)
    terms = mad.Terms(mask=7, spring_rest=to_dev(L0), spring_k=3.0, inertia_xt=to_dev(xt),
                      inertia_w=5.0, face_Minv=to_dev(ps["Minv"].reshape(-1, 4)),
                      face_area=to_dev(ps["area"]))
    rp, ci, r, J = gpu_jacobian(ctx, ps["UV"], terms, "float64")
    orr, orp, oci, oJ = orc.jacobian(V, 2, ps["UV"], 7, edges=edges, L0=L0, k=3.0, xt=xt, w=5.0,
                                     F=ps["F"], Minv=ps["Minv"], area=ps["area"])
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    assert_close("r", r, orr, "float64")
    assert_close("J", J, oJ, "float64")


def test_jacobian_shapes_and_refusals():
    import hessian_assembly_b200 as mad
    ctx, st = cloth_context(5, "float32")
    V, E = st["V"], len(st["edges"])
    assert ctx.mad_jacobian_shape(0) == (0, 0)
    assert ctx.mad_jacobian_shape(1) == (E, 6 * E)
    assert ctx.mad_jacobian_shape(2) == (3 * V, 3 * V)
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_jacobian_shape(8)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_jacobian_shape(4)  # symmetric Dirichlet needs dof 2
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
