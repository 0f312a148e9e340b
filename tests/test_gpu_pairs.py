"""Runtime vertex-vertex pairs: GPU insertion into the double-buffered CSR
and assembly with all terms, vs the fp64 oracle (pattern bit-exact)."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import assert_close, check_cloth, cloth_context, cloth_terms, gpu_pattern, run_eval, to_dev

pytestmark = pytest.mark.gpu
FULL = 1
SCAT = 2
PATCH = 4


def add_pairs(ctx, pairs, rest, dtype):
    ctx.mad_add_pairs(to_dev(np.asarray(pairs, np.int32)), to_dev(np.asarray(rest), dtype))


def pair_case(orc, n, P, dtype="float32", seed=1005, step=0, flags=0, **kw):
    ctx, st = cloth_context(n, dtype, **kw)
    x = mi.cloth_x(n, seed, step, np.dtype(dtype))
    pairs = mi.random_pairs(n, P, seed, step)
    rest = mi.pair_rest(x, pairs, np.dtype(dtype))
    add_pairs(ctx, pairs, rest, dtype)
    assert ctx.mad_status_sync() == 0
    return check_cloth(orc, n, dtype, mask=11, flags=flags, step=step, seed=seed, pairs=pairs,
                       prest=rest, ctx=ctx, st=st)


@pytest.mark.parametrize("flags", [0, FULL, SCAT, PATCH, 8])
def test_pairs_small(orc, flags):
    pair_case(orc, 30, 60, flags=flags)


def test_pairs_fp64(orc):
    pair_case(orc, 40, 150, "float64")


@pytest.mark.parametrize("flags", [0, PATCH])
def test_pairs_1000x1000_full(orc, flags):
    r = pair_case(orc, 1000, 100000, flags=flags)
    rp, ci, nnzb = gpu_pattern(r["ctx"])
    assert nnzb == 6992002 + 200000


def test_replace_semantics_and_double_buffer(orc):
    n = 25
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 1, 0, np.float64)
    for step in range(3):
        pairs = mi.random_pairs(n, 40 + 10 * step, 7, step)
        rest = mi.pair_rest(x, pairs, np.float64)
        add_pairs(ctx, pairs, rest, "float64")
        check_cloth(orc, n, "float64", mask=11, seed=1, pairs=pairs, prest=rest, ctx=ctx, st=st)
    # n = 0 restores the mesh pattern
    ctx.mad_add_pairs(None, None)
    check_cloth(orc, n, "float64", mask=11, seed=1, ctx=ctx, st=st)


def test_duplicates_edge_coincidence_and_shared_rows(orc):
    n = 12
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 3, 0, np.float64)
    pairs = np.array([[0, 50], [50, 0], [0, 50],      # duplicates (both orders)
                      [0, 1], [13, 12],               # on mesh edges
                      [0, 99], [0, 143], [5, 99],     # rows 0 and 99 gain several blocks
                      [143, 70], [70, 143]], np.int32)
    rest = np.linspace(0.05, 0.3, len(pairs))
    add_pairs(ctx, pairs, rest, "float64")
    assert ctx.mad_status_sync() == 0
    check_cloth(orc, n, "float64", mask=11, seed=3, pairs=pairs, prest=rest, ctx=ctx, st=st)


@pytest.mark.parametrize("flags", [0, PATCH])
def test_many_pairs_on_one_vertex_spill_rows(orc, flags):
    # vertex 0 gains 300 blocks: more than the shared-memory reserve, so its
    # row (and the rows staged after it) is assembled in place in global memory
    n = 30
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 4, 0, np.float64)
    far = np.array([v for v in range(n * n) if not mi.grid_adjacent(n, 0, v) and v != 0][:300])
    pairs = np.stack([np.zeros_like(far), far], 1).astype(np.int32)
    rest = mi.pair_rest(x, pairs, np.float64)
    add_pairs(ctx, pairs, rest, "float64")
    check_cloth(orc, n, "float64", mask=11, seed=4, pairs=pairs, prest=rest, ctx=ctx, st=st,
                flags=flags)


def test_bad_index_sets_status_and_is_skipped(orc):
    n = 10
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 5, 0, np.float64)
    good = np.array([[0, 55], [3, 77]], np.int32)
    bad = np.array([[0, 100], [7, 7], [-1, 4]], np.int32)
    pairs = np.concatenate([good[:1], bad, good[1:]])
    rest = np.full(len(pairs), 0.2)
    add_pairs(ctx, pairs, rest, "float64")
    assert ctx.mad_status_sync() == 5  # MAD_ERR_INDEX
    assert ctx.mad_status_sync() == 0  # cleared
    check_cloth(orc, n, "float64", mask=11, seed=5, pairs=good, prest=np.full(2, 0.2), ctx=ctx, st=st)


def test_capacity_overflow_keeps_previous_pattern(orc):
    import hessian_assembly_b200 as mad
    n = 10
    ctx, st = cloth_context(n, "float64", slack=0.02, max_pairs=64)  # 12 spare blocks
    x = mi.cloth_x(n, 6, 0, np.float64)
    p1 = mi.random_pairs(n, 4, 6, 0)
    r1 = mi.pair_rest(x, p1, np.float64)
    add_pairs(ctx, p1, r1, "float64")
    assert ctx.mad_status_sync() == 0
    p2 = mi.random_pairs(n, 30, 6, 1)  # 60 new blocks > 12 spare
    add_pairs(ctx, p2, mi.pair_rest(x, p2, np.float64), "float64")
    assert ctx.mad_status_sync() == mad.MAD_ERR_CAPACITY
    check_cloth(orc, n, "float64", mask=11, seed=6, pairs=p1, prest=r1, ctx=ctx, st=st)
    with pytest.raises(mad.MadError) as ei:
        add_pairs(ctx, mi.random_pairs(n, 65, 6, 2), np.ones(65), "float64")
    assert ei.value.status == mad.MAD_ERR_CAPACITY


def test_hvp_with_pairs(orc):
    import torch
    n = 30
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 8, 0, np.float64)
    pairs = mi.random_pairs(n, 80, 8, 0)
    rest = mi.pair_rest(x, pairs, np.float64)
    add_pairs(ctx, pairs, rest, "float64")
    v = mi.probe_vector(st["V"], 3, 9, np.float64)
    y = torch.zeros((st["V"], 3), dtype=torch.float64, device="cuda")
    ctx.mad_hvp(to_dev(x), cloth_terms(st, "float64", 11), to_dev(v), y)
    rp, ci = orc.pattern(st["V"], st["F"], pairs)
    og, oH, oE = orc.eval(st["V"], 3, x, 11, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"],
                          xt=st["xt"], w=st["w"], pairs=pairs, prest=rest, kp=mi.PAIR_K)
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(st["V"], 3, rp, ci, oH, v), "float64")


def test_first_insertion_overflow_restores_mesh_pattern(orc):
    import hessian_assembly_b200 as mad
    n = 10
    ctx, st = cloth_context(n, "float64", slack=0.02, max_pairs=64)
    x = mi.cloth_x(n, 10, 0, np.float64)
    p = mi.random_pairs(n, 30, 10, 0)  # 60 new blocks > 12 spare, from the mesh pattern
    add_pairs(ctx, p, mi.pair_rest(x, p, np.float64), "float64")
    assert ctx.mad_status_sync() == mad.MAD_ERR_CAPACITY
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(st["V"], st["F"])
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    check_cloth(orc, n, "float64", mask=3, seed=10, ctx=ctx, st=st)


@pytest.mark.parametrize("mask", [3, 2 | 8, 1 | 8])
@pytest.mark.parametrize("flags", [0, PATCH])
def test_inserted_blocks_with_partial_term_sets(orc, mask, flags):
    # inserted blocks without pair terms stay zero; without edge terms every
    # block of a row starts at zero
    n = 20
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 11, 0, np.float64)
    pairs = mi.random_pairs(n, 50, 11, 0)
    rest = mi.pair_rest(x, pairs, np.float64)
    add_pairs(ctx, pairs, rest, "float64")
    check_cloth(orc, n, "float64", mask=mask, flags=flags, seed=11, pairs=pairs, prest=rest,
                ctx=ctx, st=st)


def test_rows_at_the_register_merge_limits(orc):
    # vertex 0 gets 8 pair entries (two of them repeated), vertex 1 gets 9:
    # one row at the limit of the in-register merge, one just past it
    n = 16
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 12, 0, np.float64)
    far0 = [v for v in range(40, 200) if not mi.grid_adjacent(n, 0, v)][:6]
    far1 = [v for v in range(60, 240) if not mi.grid_adjacent(n, 1, v) and v not in far0][:9]
    pairs = [[0, v] for v in far0] + [[far0[0], 0], [0, far0[3]]] + [[1, v] for v in far1]
    pairs = np.array(pairs, np.int32)
    rest = np.linspace(0.1, 0.4, len(pairs))
    add_pairs(ctx, pairs, rest, "float64")
    assert ctx.mad_status_sync() == 0
    check_cloth(orc, n, "float64", mask=11, seed=12, pairs=pairs, prest=rest, ctx=ctx, st=st)


def test_pairs_on_a_long_mesh_row(orc):
    """A fan hub whose mesh row (41 blocks) is longer than the columns the
    register merge holds, with pairs on the hub and between rim vertices."""
    import hessian_assembly_b200 as mad
    m = 40
    ang = 2 * np.pi * np.arange(m) / m
    X = np.concatenate([[[0.0, 0.0, 0.0]], np.stack([np.cos(ang), np.sin(ang), 0 * ang], 1)])
    F = np.array([[0, 1 + i, 1 + (i + 1) % m] for i in range(m)], np.int32)
    V = m + 1
    ctx = mad.Context(V, F, 3, "float64", part_xyz=X)
    edges = ctx.mad_edges().cpu().numpy()
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1)
    rng = np.random.default_rng(13)
    x = X + 0.01 * rng.standard_normal(X.shape)
    xt = X.copy()
    # hub pairs are all on mesh edges; rim pairs are new blocks
    pairs = np.array([[0, 5], [0, 17], [3, 9], [3, 25], [9, 3], [30, 10]], np.int32)
    prest = 0.9 * np.linalg.norm(x[pairs[:, 0]] - x[pairs[:, 1]], axis=1)
    ctx.mad_add_pairs(to_dev(pairs), to_dev(prest))
    terms = mad.Terms(mask=11, spring_rest=to_dev(L0), spring_k=10.0, inertia_xt=to_dev(xt),
                      inertia_w=3.0, pair_k=5.0)
    g, H, E = run_eval(ctx, x, terms, "float64")
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F, pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(V, 3, x, 11, orp, oci, edges=edges, L0=L0, k=10.0, xt=xt, w=3.0,
                          pairs=pairs, prest=prest, kp=5.0)
    assert_close("g", g, og, "float64")
    assert_close("H", H[:nnzb], oH, "float64")
    assert ctx.mad_status_sync() == 0


def test_inserted_blocks_before_a_long_mesh_row(orc):
    """A fan hub (mesh row of 41 blocks) that gains blocks with lower
    columns: every mesh block of the hub row, those past position 31 too,
    moves behind the inserted ones."""
    import hessian_assembly_b200 as mad
    m = 40
    ang = 2 * np.pi * np.arange(m) / m
    tri = np.array([[3.0, 0.0, 0.0], [3.5, 0.0, 0.0], [3.0, 0.5, 0.0]])
    hub = np.array([[0.0, 0.0, 0.0]])
    rim = np.stack([np.cos(ang), np.sin(ang), 0 * ang], 1)
    X = np.concatenate([tri, hub, rim])
    F = np.array([[0, 1, 2]] + [[3, 4 + i, 4 + (i + 1) % m] for i in range(m)], np.int32)
    V = 4 + m
    ctx = mad.Context(V, F, 3, "float64", part_xyz=X)
    edges = ctx.mad_edges().cpu().numpy()
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1)
    rng = np.random.default_rng(14)
    x = X + 0.01 * rng.standard_normal(X.shape)
    xt = X.copy()
    # the hub (3) gains columns 0 and 1 ahead of its mesh row; rim vertex 20
    # gains column 2; row 2 gains column 20 after its mesh columns
    pairs = np.array([[3, 1], [0, 3], [2, 20], [1, 3]], np.int32)
    prest = 0.9 * np.linalg.norm(x[pairs[:, 0]] - x[pairs[:, 1]], axis=1)
    ctx.mad_add_pairs(to_dev(pairs), to_dev(prest))
    terms = mad.Terms(mask=11, spring_rest=to_dev(L0), spring_k=10.0, inertia_xt=to_dev(xt),
                      inertia_w=3.0, pair_k=5.0)
    g, H, E = run_eval(ctx, x, terms, "float64")
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F, pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    assert orp[4] - orp[3] == 43  # the hub row: 2 inserted + 41 mesh blocks
    og, oH, oE = orc.eval(V, 3, x, 11, orp, oci, edges=edges, L0=L0, k=10.0, xt=xt, w=3.0,
                          pairs=pairs, prest=prest, kp=5.0)
    assert_close("g", g, og, "float64")
    assert_close("H", H[:nnzb], oH, "float64")
    assert ctx.mad_status_sync() == 0


@pytest.mark.parametrize("n,dtype,slot_bytes", [(40, "float64", 4), (190, "float32", 8)])
def test_pairs_on_permuted_numbering(orc, n, dtype, slot_bytes):
    """Pairs on a randomly renumbered cloth: at 40^2 the compact row tables
    (irregular deltas), at 190^2 the wide ones (deltas past 16 bits), so both
    row kernels' pair paths run; eval and the product against the oracle."""
    import hessian_assembly_b200 as mad
    import torch
    st = mi.cloth_static(n, np.float64)
    V = st["V"]
    perm = np.random.default_rng(5).permutation(V)   # new id of old vertex
    inv = np.argsort(perm)
    F = perm[st["F"]].astype(np.int32)
    X = st["X"][inv]
    ctx = mad.Context(V, F, 3, dtype, part_xyz=X)
    assert ctx.info.row_slot_bytes == slot_bytes
    e = np.sort(perm[mi.grid_edges(n)], axis=1)
    edges = e[np.lexsort((e[:, 1], e[:, 0]))].astype(np.int32)
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1).astype(dtype)
    x = mi.cloth_x(n, 15, 0, np.float64)[inv].astype(dtype)
    xt = X.astype(dtype)
    pairs = perm[mi.random_pairs(n, 4 * n, 15, 0)].astype(np.int32)
    prest = mi.pair_rest(x, pairs, np.dtype(dtype))
    add_pairs(ctx, pairs, prest, dtype)
    assert ctx.mad_status_sync() == 0
    terms = mad.Terms(mask=11, spring_rest=to_dev(L0), spring_k=st["k"], inertia_xt=to_dev(xt),
                      inertia_w=st["w"], pair_k=mi.PAIR_K)
    g, H, E = run_eval(ctx, x, terms, dtype)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F, pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(V, 3, x, 11, orp, oci, edges=edges, L0=L0, k=st["k"], xt=xt, w=st["w"],
                          pairs=pairs, prest=prest, kp=mi.PAIR_K)
    assert_close("g", g, og, dtype)
    assert_close("H", H[:nnzb], oH, dtype)
    # the product: y = H v with the oracle's assembled H
    v = np.random.default_rng(16).standard_normal((V, 3)).astype(dtype)
    tdt = getattr(torch, dtype)
    y = torch.zeros((V, 3), dtype=tdt, device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    oy = orc.bsr_mv(V, 3, orp, oci, oH, v.astype(np.float64))
    assert_close("y", y.cpu().numpy(), oy, dtype)


@pytest.mark.parametrize("dtype", ["float32", "float64"])
def test_pairs_dof2_compact_rows(orc, dtype):
    """Springs, inertia and pairs on a 2-D grid (no face terms): the compact
    row kernel's pair path at dof 2, with the gathered partner entries in
    their 2-D layout; eval and the product against the oracle."""
    import hessian_assembly_b200 as mad
    import torch
    n = 40
    ps = mi.param_static(n, 41, np.float64)
    V, F, X, UV = ps["V"], ps["F"], ps["X"], ps["UV"]
    ctx = mad.Context(V, F, 2, dtype, part_xyz=X, max_pairs=400)
    assert ctx.info.row_slot_bytes == 4
    edges = ctx.mad_edges().cpu().numpy()
    L0 = np.linalg.norm(X[edges[:, 0]] - X[edges[:, 1]], axis=1)
    xt = X + 0.01 * mi.probe_vector(V, 2, 42, np.float64)
    rng = np.random.default_rng(43)
    pairs = []
    while len(pairs) < 300:
        a, b = rng.integers(0, V, 2)
        if a != b and not mi.grid_adjacent(n, a, b):
            pairs.append((a, b))
    pairs = np.array(pairs, np.int32)
    prest = 0.9 * np.linalg.norm(UV[pairs[:, 0]] - UV[pairs[:, 1]], axis=1)
    add_pairs(ctx, pairs, prest, dtype)
    assert ctx.mad_status_sync() == 0
    mask = 1 | 2 | 8
    terms = mad.Terms(mask=mask, spring_rest=to_dev(L0, dtype), spring_k=3.0,
                      inertia_xt=to_dev(xt, dtype), inertia_w=50.0, pair_k=7.0)
    x = UV.astype(dtype)
    g, H, E = run_eval(ctx, x, terms, dtype)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(V, F, pairs)
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(V, 2, x, mask, orp, oci, edges=edges, L0=L0.astype(dtype), k=3.0,
                          xt=xt.astype(dtype), w=50.0, pairs=pairs, prest=prest.astype(dtype),
                          kp=7.0)
    assert_close("g", g, og, dtype)
    assert_close("H", H[:nnzb], oH, dtype)
    v = mi.probe_vector(V, 2, 44, np.dtype(dtype))
    tdt = getattr(torch, dtype)
    y = torch.full((V, 2), float("nan"), dtype=tdt, device="cuda")
    ctx.mad_hvp(to_dev(x, dtype), terms, to_dev(v, dtype), y)
    torch.cuda.synchronize()
    assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 2, orp, oci, oH, v), dtype)
