"""Owner-computes sharding on one GPU: every shard's rows evaluated one after
another with mad_eval_shard, reading the positions of the other shards
through their own device buffers (the pointers a peer GPU would pass), and
the rows stitched back together.

The stitched g and H are compared with the fp64 oracle (pattern bit-exact,
values within the parity tolerance) and with the unsharded mad_eval, which
they must equal bit for bit: a row's terms and their order do not depend on
which shard evaluates it.
"""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import ETOL, assert_close, cloth_context, cloth_terms, gpu_pattern, run_eval, to_dev

pytestmark = pytest.mark.gpu


def run_shards(ctx, st, x, terms, dtype, nranks, separate=True):
    import torch

    import hessian_assembly_b200 as mad
    V = st["V"]
    rb, bb = mad.mad_shard_plan(V, st["F"], nranks)
    tdt = getattr(torch, dtype)
    xd = to_dev(x, dtype)
    # each shard's positions in a buffer of its own (as on its own GPU), or
    # slices of one buffer
    parts = [xd[rb[r]:rb[r + 1]].clone() if separate else xd[rb[r]:rb[r + 1]]
             for r in range(nranks)]
    gs, Hs, E = [], [], 0.0
    for r in range(nranks):
        nr, nb = int(rb[r + 1] - rb[r]), int(bb[r + 1] - bb[r])
        g = torch.full((max(nr, 1), 3), float("nan"), dtype=tdt, device="cuda")
        H = torch.full((max(nb, 1), 3, 3), float("nan"), dtype=tdt, device="cuda")
        e = torch.zeros(1, dtype=torch.float64, device="cuda")
        ctx.mad_eval_shard(rb, parts, r, terms, g, H, e)
        torch.cuda.synchronize()
        gs.append(g[:nr].cpu().numpy())
        Hs.append(H[:nb].cpu().numpy())
        E += e.item()
    return np.concatenate(gs), np.concatenate(Hs), E, rb


@pytest.mark.parametrize("n,dtype,nranks", [(100, "float32", 2), (100, "float64", 3),
                                            (37, "float32", 8), (1000, "float32", 8)])
def test_shards_stitch_to_the_oracle_and_to_eval(orc, n, dtype, nranks):
    ctx, st = cloth_context(n, dtype)
    x = mi.cloth_x(n, 4242, 1, np.dtype(dtype))
    terms = cloth_terms(st, dtype, 3)
    g, H, E, rb = run_shards(ctx, st, x, terms, dtype, nranks)
    rp, ci, nnzb = gpu_pattern(ctx)
    orp, oci = orc.pattern(st["V"], st["F"])
    np.testing.assert_array_equal(rp, orp)
    np.testing.assert_array_equal(ci, oci)
    og, oH, oE = orc.eval(st["V"], 3, x, 3, orp, oci, edges=st["edges"], L0=st["L0"],
                          k=st["k"], xt=st["xt"], w=st["w"])
    assert_close("g", g, og, dtype)
    assert_close("H", H, oH, dtype)
    assert abs(E - oE) <= ETOL[dtype] * abs(oE)
    g1, H1, _ = run_eval(ctx, x, terms, dtype)
    assert np.array_equal(g, g1) and np.array_equal(H, H1[:nnzb])


def test_shards_of_one_buffer_and_full_stencil_ad(orc):
    n = 64
    ctx, st = cloth_context(n, "float64")
    x = mi.cloth_x(n, 9, 0, np.float64)
    terms = cloth_terms(st, "float64", 3, flags=1)
    g, H, _, _ = run_shards(ctx, st, x, terms, "float64", 5, separate=False)
    g1, H1, _ = run_eval(ctx, x, terms, "float64")
    assert np.array_equal(g, g1) and np.array_equal(H, H1[:ctx.info.nnzb_base])


def test_shard_refusals():
    import torch

    import hessian_assembly_b200 as mad
    n = 40
    ctx, st = cloth_context(n, "float32")
    x = to_dev(mi.cloth_x(n, 1, 0, np.float32))
    g = torch.zeros((st["V"], 3), device="cuda")
    H = torch.zeros((ctx.info.nnzb_base, 3, 3), device="cuda")
    terms = cloth_terms(st, "float32", 3)
    for rb, code in (([0, 50, st["V"]], mad.MAD_ERR_INVALID_ARG),   # not a multiple of 32
                     ([0, 64, 32, st["V"]], mad.MAD_ERR_INVALID_ARG),  # decreasing
                     ([0, 64, st["V"] - 1], mad.MAD_ERR_INVALID_ARG)):  # does not end at V
        with pytest.raises(mad.MadError) as ei:
            ctx.mad_eval_shard(rb, [x] * (len(rb) - 1), 0, terms, g, H)
        assert ei.value.status == code
    rb = [0, 640, st["V"]]
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_eval_shard(rb, [x, x], 0, mad.Terms(mask=8, pair_k=1.0), g, H)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
    pairs = mi.random_pairs(n, 10, 3, 0)
    ctx.mad_add_pairs(to_dev(pairs), to_dev(np.ones(10, np.float32)))
    with pytest.raises(mad.MadError) as ei:
        ctx.mad_eval_shard(rb, [x, x], 0, terms, g, H)
    assert ei.value.status == mad.MAD_ERR_UNIMPLEMENTED
