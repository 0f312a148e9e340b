"""Stream capture: mad_eval, mad_add_pairs and mad_hvp recorded in a CUDA
graph and replayed with new inputs copied into the captured buffers give the
oracle's results at every replay."""
import numpy as np
import pytest

import mesh_inputs as mi
from _parity import assert_close, cloth_context, cloth_terms, gpu_pattern, to_dev

pytestmark = pytest.mark.gpu


def _capture(fn):
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # one uncaptured run first
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    return graph


def test_eval_graph_replay(orc):
    import torch
    n, dtype = 60, "float32"
    ctx, st = cloth_context(n, dtype)
    V = st["V"]
    terms = cloth_terms(st, dtype, 3)
    x = torch.zeros((V, 3), dtype=torch.float32, device="cuda")
    g = torch.zeros((V, 3), dtype=torch.float32, device="cuda")
    H = torch.zeros((ctx.info.capacity_blocks, 3, 3), dtype=torch.float32, device="cuda")
    graph = _capture(lambda: ctx.mad_eval(x, terms, g, H))
    rp, ci = orc.pattern(V, st["F"])
    for step in range(3):
        xs = mi.cloth_x(n, 3100, step, np.float32)
        x.copy_(to_dev(xs, dtype))
        graph.replay()
        torch.cuda.synchronize()
        og, oH, _ = orc.eval(V, 3, xs, 3, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"],
                             xt=st["xt"], w=st["w"])
        assert_close("g", g.cpu().numpy(), og, dtype)
        assert_close("H", H[:len(ci)].cpu().numpy(), oH, dtype)


def test_pairs_and_eval_graph_replay(orc):
    import torch
    n, dtype, P = 40, "float64", 100
    ctx, st = cloth_context(n, dtype, max_pairs=P)
    V = st["V"]
    terms = cloth_terms(st, dtype, 11)
    x = torch.zeros((V, 3), dtype=torch.float64, device="cuda")
    ij = torch.zeros((P, 2), dtype=torch.int32, device="cuda")
    rest = torch.zeros(P, dtype=torch.float64, device="cuda")
    g = torch.zeros((V, 3), dtype=torch.float64, device="cuda")
    H = torch.zeros((ctx.info.capacity_blocks, 3, 3), dtype=torch.float64, device="cuda")
    # valid inputs for the uncaptured run
    pairs0 = mi.random_pairs(n, P, 3200, 99)
    x0 = mi.cloth_x(n, 3200, 99, np.float64)
    x.copy_(to_dev(x0))
    ij.copy_(to_dev(pairs0))
    rest.copy_(to_dev(mi.pair_rest(x0, pairs0, np.float64)))

    def step():
        ctx.mad_add_pairs(ij, rest)
        ctx.mad_eval(x, terms, g, H)

    graph = _capture(step)
    for s_ in range(3):
        xs = mi.cloth_x(n, 3200, s_, np.float64)
        pairs = mi.random_pairs(n, P, 3200, s_)
        pr = mi.pair_rest(xs, pairs, np.float64)
        x.copy_(to_dev(xs))
        ij.copy_(to_dev(pairs))
        rest.copy_(to_dev(pr))
        graph.replay()
        torch.cuda.synchronize()
        assert ctx.mad_status_sync() == 0
        rp, ci, nnzb = gpu_pattern(ctx)
        orp, oci = orc.pattern(V, st["F"], pairs)
        np.testing.assert_array_equal(rp, orp)
        np.testing.assert_array_equal(ci, oci)
        og, oH, _ = orc.eval(V, 3, xs, 11, orp, oci, edges=st["edges"], L0=st["L0"], k=st["k"],
                             xt=st["xt"], w=st["w"], pairs=pairs, prest=pr, kp=mi.PAIR_K)
        assert_close("g", g.cpu().numpy(), og, dtype)
        assert_close("H", H[:nnzb].cpu().numpy(), oH, dtype)


def test_symdir_hvp_graph_replay(orc):
    import hessian_assembly_b200 as mad
    import torch
    n, dtype = 30, "float64"
    ps = mi.param_static(n, 3300, np.float64)
    V = ps["V"]
    ctx = mad.Context(V, ps["F"], 2, dtype, part_xyz=ps["X"])
    terms = mad.Terms(mask=4, face_Minv=to_dev(ps["Minv"].reshape(-1, 4)),
                      face_area=to_dev(ps["area"]))
    x = to_dev(ps["UV"])
    v = torch.zeros((V, 2), dtype=torch.float64, device="cuda")
    y = torch.zeros((V, 2), dtype=torch.float64, device="cuda")
    graph = _capture(lambda: ctx.mad_hvp(x, terms, v, y))
    rp, ci = orc.pattern(V, ps["F"])
    og, oH, _ = orc.eval(V, 2, ps["UV"], 4, rp, ci, F=ps["F"], Minv=ps["Minv"], area=ps["area"])
    for s_ in range(2):
        vv = mi.probe_vector(V, 2, 3301 + s_, np.float64)
        v.copy_(to_dev(vv))
        graph.replay()
        torch.cuda.synchronize()
        assert_close("y", y.cpu().numpy(), orc.bsr_mv(V, 2, rp, ci, oH, vv), dtype)
