"""Owner-computes sharding, host side: the row ranges of mad_shard_plan and
the halos of mad_shard_halo, checked against the fp64 oracle's pattern, and
the halo exchange they imply, run as world_size-2 gloo ranks on CPU.

A shard owns the rows [row_begin[r], row_begin[r+1]) of the block-CSR
Hessian; its Hessian values are the pattern's blocks [row_ptr[row_begin[r]],
row_ptr[row_begin[r+1]]) and its rows read the positions of the vertices in
its halo, which other shards own.
"""
import os

import numpy as np
import pytest

import mesh_inputs as mi


def brute_halo(rp, ci, lo, hi):
    cols = ci[rp[lo]:rp[hi]]
    return np.unique(cols[(cols < lo) | (cols >= hi)])


def random_mesh(V, nF, seed):
    rng = np.random.default_rng(seed)
    F = []
    while len(F) < nF:
        f = rng.integers(0, V, 3)
        if len(set(f.tolist())) == 3:
            F.append(f)
    return np.array(F, np.int32)


@pytest.mark.parametrize("n,nranks", [(10, 1), (10, 3), (100, 2), (100, 8), (257, 5)])
def test_plan_ranges_and_blocks(orc, n, nranks):
    import hessian_assembly_b200 as mad
    st = mi.cloth_static(n, np.float32)
    V = st["V"]
    rb, bb = mad.mad_shard_plan(V, st["F"], nranks)
    rp, ci = orc.pattern(V, st["F"])
    assert rb[0] == 0 and rb[-1] == V and np.all(np.diff(rb) >= 0)
    assert all(b % 32 == 0 or b == V for b in rb)
    np.testing.assert_array_equal(bb, rp[rb])
    # balance: every range is within one tile of rows of the even share
    nnzb = rp[V]
    tile_blocks = 32 * int(np.max(np.diff(rp)))
    for r in range(nranks):
        if V >= 32 * nranks * 4:
            assert abs((bb[r + 1] - bb[r]) - nnzb / nranks) <= tile_blocks


@pytest.mark.parametrize("n,lo,hi", [(10, 0, 32), (10, 32, 64), (40, 320, 800), (40, 0, 1600),
                                     (40, 1600, 1600)])
def test_halo_is_the_ranges_outside_columns(orc, n, lo, hi):
    import hessian_assembly_b200 as mad
    st = mi.cloth_static(n, np.float32)
    rp, ci = orc.pattern(st["V"], st["F"])
    h = mad.mad_shard_halo(st["V"], st["F"], lo, hi)
    np.testing.assert_array_equal(h, brute_halo(rp, ci, lo, hi))


def test_halo_random_mesh(orc):
    import hessian_assembly_b200 as mad
    V = 500
    F = random_mesh(V, 700, 11)  # unordered numbering: halos far from the range
    rp, ci = orc.pattern(V, F)
    rb, bb = mad.mad_shard_plan(V, F, 4)
    np.testing.assert_array_equal(bb, rp[rb])
    for r in range(4):
        np.testing.assert_array_equal(mad.mad_shard_halo(V, F, rb[r], rb[r + 1]),
                                      brute_halo(rp, ci, rb[r], rb[r + 1]))


def test_plan_rejects_bad_arguments():
    import hessian_assembly_b200 as mad
    st = mi.cloth_static(5, np.float32)
    for nranks in (0, 65):
        with pytest.raises(mad.MadError):
            mad.mad_shard_plan(st["V"], st["F"], nranks)
    bad = st["F"].copy()
    bad[0, 0] = st["V"]
    with pytest.raises(mad.MadError):
        mad.mad_shard_plan(st["V"], bad, 2)
    with pytest.raises(mad.MadError):
        mad.mad_shard_halo(st["V"], st["F"], 10, 5)


# ---------------------------------------------------------------- gloo ranks

def _exchange_rank(rank, world, port, n, out):
    """One gloo rank: plan, ask each owner for the positions of its halo
    vertices (the requests, then the answers, routed rank to rank), and check
    that the answers are the global positions."""
    import torch
    import torch.distributed as dist

    import hessian_assembly_b200 as mad
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        st = mi.cloth_static(n, np.float32)
        V = st["V"]
        x = mi.cloth_x(n, 77, 0, np.float64)      # every rank can build the global x ...
        rb, bb = mad.mad_shard_plan(V, st["F"], world)
        own = x[rb[rank]:rb[rank + 1]]            # ... but serves only its own part
        halo = mad.mad_shard_halo(V, st["F"], rb[rank], rb[rank + 1])
        owner = np.searchsorted(rb, halo, side="right") - 1
        assert np.all(owner != rank)

        def exchange(lists, dtype):
            """lists[s] goes to rank s; returns what each rank sent here (gloo
            has no all_to_all: padded all_gathers of every rank's lists)."""
            cnt = torch.tensor([len(a) for a in lists], dtype=torch.int64)
            cnts = [torch.zeros(world, dtype=torch.int64) for _ in range(world)]
            dist.all_gather(cnts, cnt)
            m = max(1, int(max(int(c.max()) for c in cnts)))
            buf = torch.zeros(world, m, dtype=dtype)
            for s, a in enumerate(lists):
                buf[s, :len(a)] = torch.as_tensor(a, dtype=dtype)
            bufs = [torch.zeros(world, m, dtype=dtype) for _ in range(world)]
            dist.all_gather(bufs, buf)
            return [bufs[s][rank, :int(cnts[s][rank])].numpy() for s in range(world)]

        # requests: the halo vertices of each owner
        req = [halo[owner == s].astype(np.int64) for s in range(world)]
        got = exchange(req, torch.int64)
        # answers: this rank's positions at the requested vertices
        ans = []
        for s in range(world):
            v = got[s]
            assert np.all((v >= rb[rank]) & (v < rb[rank + 1])), "request for a vertex not owned"
            ans.append(own[v - rb[rank]].reshape(-1))
        back = exchange(ans, torch.float64)
        for s in range(world):
            np.testing.assert_array_equal(back[s].reshape(-1, 3), x[req[s]])
        # every block of the pattern is owned by exactly one rank
        nb = torch.tensor([bb[rank + 1] - bb[rank]], dtype=torch.int64)
        dist.all_reduce(nb)
        assert int(nb) == bb[-1]
        out.put((rank, len(halo), None))
    except Exception as e:  # reported to the parent
        out.put((rank, -1, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n", [64, 130])
def test_halo_exchange_two_gloo_ranks(n):
    import multiprocessing as mp
    import socket
    ctx = mp.get_context("spawn")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    q = ctx.Queue()
    ps = [ctx.Process(target=_exchange_rank, args=(r, 2, port, n, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = [q.get(timeout=120) for _ in ps]
    for p in ps:
        p.join(timeout=60)
    for rank, nh, err in res:
        assert err is None, f"rank {rank}: {err}"
        assert nh > 0
