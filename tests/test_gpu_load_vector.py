"""GPU parity of the fused calls around the context's expert load vector.

In ue_rebalance, ue_rebalance_ex and ue_rebalance_dispatch the load grid also
adds every rank's counts into a load vector held by the context, and the
planner reads it (instead of summing counts) and writes the zeros back for the
next call.  These tests run sequences that would expose a vector left
non-zero: shapes that change E and N on one context, the three fused calls
interleaved with the separate calls, a CUDA graph replayed over new ids, and
bad ids.  Every result is compared bit for bit with the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_load_ue_b200 import inputs, ue

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    c = ue.Context(0)
    yield c
    c.close()


def _ids(E, N, tpr, s, seed, K=8):
    w = inputs.Workload("lv", E=E, K=K, N=N, R=1, tokens_per_rank=tpr, s=s, base_seed=seed)
    return inputs.topk_ids(w, 0)


def _fused(ctx, ids_np, E, N, R, call="rebalance", variant=0):
    T, K = ids_np.shape
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np)).cuda()
    counts = torch.full((N, E), -7, dtype=torch.int32, device="cuda")
    bad = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.full((T, K), -5, dtype=torch.int32, device="cuda")
    if call == "rebalance":
        ue.ue_rebalance(ctx, cfg, ids, counts, bad, plan, phys)
    elif call == "ex":
        ue.ue_rebalance_ex(ctx, cfg, ids, counts, bad, plan, phys, variant)
    else:
        disp = ue.Dispatch(cfg, with_gates=False)
        ue.ue_rebalance_dispatch(ctx, cfg, ids, counts, bad, plan, phys, disp)
    torch.cuda.synchronize()
    return counts.cpu().numpy(), bad.cpu().numpy(), plan.to_host(), phys.cpu().numpy()


def _check(ctx, ids_np, E, N, R, call="rebalance", variant=0):
    counts, bad, pl, phys = _fused(ctx, ids_np, E, N, R, call, variant)
    ref = oracle.rebalance(ids_np, E, N, R, variant)
    assert np.array_equal(counts, ref["counts"]), "counts"
    assert np.array_equal(bad, ref["bad"]), "bad"
    assert np.array_equal(pl["load"], ref["load"]), "load"
    for f in oracle.PLAN_FIELDS:
        assert np.array_equal(pl[f], ref["plan"][f]), f
    assert np.array_equal(pl["rank_off"], ref["rank_off"]), "rank_off"
    assert np.array_equal(phys, ref["phys"]), "phys"


def test_shapes_change_on_one_context(ctx):
    # Wider, then narrower, then wider again: a vector left non-zero past the
    # narrow shape's E, or by it below, would show up in the next plan.
    seq = [(256, 64, 1, 4096, 1.2), (64, 8, 2, 512, 1.0), (1024, 128, 1, 1024, 1.6), (256, 64, 1, 4096, 0.0),
           (128, 32, 2, 8192, 1.2), (1024, 1024, 1, 64, 0.8), (256, 256, 1, 16384, 1.2), (64, 8, 2, 512, 1.0)]
    for i, (E, N, R, tpr, s) in enumerate(seq):
        _check(ctx, _ids(E, N, tpr, s, 40 + i), E, N, R)


def test_fused_and_separate_calls_interleaved(ctx):
    E, N, R = 256, 64, 1
    for i in range(3):
        ids_np = _ids(E, N, 4096, 1.2, 60 + i)
        _check(ctx, ids_np, E, N, R, call="rebalance")
        # separate calls do not touch the vector
        T, K = ids_np.shape
        cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
        ids = torch.from_numpy(ids_np).cuda()
        counts = torch.empty((N, E), dtype=torch.int32, device="cuda")
        ue.ue_load(ctx, cfg, ids, counts, None)
        plan = ue.Plan(cfg)
        ue.ue_plan(ctx, cfg, counts, plan)
        torch.cuda.synchronize()
        _check(ctx, ids_np, E, N, R, call="dispatch")
        _check(ctx, ids_np, E, N, R, call="ex", variant=3)


def test_bad_ids_are_not_loads(ctx):
    E, N, R = 256, 64, 1
    ids_np = _ids(E, N, 4096, 1.2, 77).copy()
    rng = np.random.default_rng(5)
    pos = rng.choice(ids_np.size, size=2000, replace=False)
    ids_np.reshape(-1)[pos] = rng.choice([-1, E, E + 7, 1 << 30], size=pos.size)
    for _ in range(2):
        _check(ctx, ids_np, E, N, R)


def test_cuda_graph_replays_over_new_ids(ctx):
    E, N, R = 256, 64, 1
    T, K = 64 * 4096, 8
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ids = torch.empty((T, K), dtype=torch.int32, device="cuda")
    counts = torch.empty((N, E), dtype=torch.int32, device="cuda")
    bad = torch.empty((N,), dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.empty((T, K), dtype=torch.int32, device="cuda")
    st = torch.cuda.Stream()
    ids.copy_(torch.from_numpy(_ids(E, N, 4096, 1.2, 90)))
    with torch.cuda.stream(st):
        ue.ue_rebalance(ctx, cfg, ids, counts, bad, plan, phys, stream=st)   # warm-up outside the capture
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        ue.ue_rebalance(ctx, cfg, ids, counts, bad, plan, phys, stream=st)
    for k, s in enumerate((1.2, 0.0, 1.6, 0.8)):
        ids_np = _ids(E, N, 4096, s, 91 + k)
        ids.copy_(torch.from_numpy(ids_np))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.rebalance(ids_np, E, N, R)
        assert np.array_equal(counts.cpu().numpy(), ref["counts"])
        assert np.array_equal(plan["load"].cpu().numpy(), ref["load"])
        for f in oracle.PLAN_FIELDS:
            assert np.array_equal(plan[f].cpu().numpy(), ref["plan"][f]), f
        assert np.array_equal(phys.cpu().numpy(), ref["phys"])
    del g
