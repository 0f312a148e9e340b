"""GPU-built block-CSR pattern and edge list are bit-exact with the oracle."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import gpu_pattern

pytestmark = pytest.mark.gpu


def _ctx(V, F, dof=3, **kw):
    import hessian_assembly_b200 as mad
    return mad.Context(V, F, dof, "float32", **kw)


@pytest.mark.parametrize("n", [2, 3, 10, 100])
def test_grid_pattern_and_edges(orc, n):
    X, F = mi.grid_mesh(n)
    V = n * n
    ctx = _ctx(V, F, part_xyz=X)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    assert nnzb == V + 2 * (2 * n * (n - 1) + (n - 1) ** 2)
    assert ctx.info.nnzb_base == nnzb
    np.testing.assert_array_equal(ctx.mad_edges().cpu().numpy(), orc.edges(V, F))
    assert ctx.info.capacity_blocks == int(np.ceil(1.1 * nnzb))


def test_random_mesh_with_isolated_vertices(orc):
    rng = np.random.default_rng(5)
    V = 300
    F = np.array([rng.choice(250, 3, replace=False) for _ in range(400)], np.int32)  # 250..299 isolated
    ctx = _ctx(V, F)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    np.testing.assert_array_equal(ctx.mad_edges().cpu().numpy(), orc.edges(V, F))


def test_no_faces_gives_diagonal_pattern(orc):
    ctx = _ctx(7, np.zeros((0, 3), np.int32))
    rp, ci, nnzb = gpu_pattern(ctx)
    np.testing.assert_array_equal(rp, np.arange(8))
    np.testing.assert_array_equal(ci, np.arange(7))
    assert ctx.info.E == 0


def test_empty_mesh():
    ctx = _ctx(0, np.zeros((0, 3), np.int32))
    assert ctx.info.V == 0 and ctx.info.nnzb_base == 0 and ctx.info.n_patches == 0


def test_high_valence_fan(orc):
    # one hub vertex shared by 300 faces (row length 301 + 1)
    m = 300
    F = np.array([[0, 1 + i, 1 + (i + 1) % m] for i in range(m)], np.int32)
    V = m + 1
    ctx = _ctx(V, F)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
