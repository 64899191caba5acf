"""GPU parity of the persistent reroute over pieces (large microbatches).

When a CTA's share of a rank's ids in the rank-per-cluster reroute would be
large (more than 64 Ki ids: many ranks, or many tokens per rank), the library
cuts each rank's ids into pieces: the load kernel writes the occurrences before
every piece and the persistent reroute routes each piece with a table, ranking
only the experts whose quota boundary falls inside it.  Every case here takes
that path (checked on the kernels the call launches) and is compared bit for
bit with the oracle.
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


def _launched(fn):
    """Names of the kernels fn launches (CUDA profiler activity)."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return " ".join(e.name for e in prof.events() if e.device_type.name == "CUDA")


def _run(ctx, ids_np, E, N, R, fused=True, phys_offset=0):
    T, K = ids_np.shape
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np)).cuda()
    counts = torch.full((N, E), -7, dtype=torch.int32, device="cuda")
    bad = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    for t in plan.tensors.values():
        t.fill_(-99)
    buf = torch.full((T * K + phys_offset,), -5, dtype=torch.int32, device="cuda")
    phys = buf[phys_offset:].view(T, K)
    if fused:
        names = _launched(lambda: ue.ue_rebalance(ctx, cfg, ids, counts, bad, plan, phys))
    else:
        ue.ue_load(ctx, cfg, ids, counts, bad)
        ue.ue_plan(ctx, cfg, counts, plan)
        names = _launched(lambda: ue.ue_reroute(ctx, cfg, ids, plan, phys))
    assert "k_reroute_pieces" in names, names
    return counts.cpu().numpy(), bad.cpu().numpy(), plan.to_host(), phys.cpu().numpy()


def _check(ctx, ids, E, N, R, **kw):
    counts, bad, pl, phys = _run(ctx, ids, E, N, R, **kw)
    ref = oracle.rebalance(ids, E, N, R)
    assert np.array_equal(counts, ref["counts"]), "counts"
    assert np.array_equal(bad, ref["bad"]), "bad"
    for f in oracle.PLAN_FIELDS:
        assert np.array_equal(pl[f], ref["plan"][f]), f
    assert np.array_equal(pl["rank_off"], ref["rank_off"]), "rank_off"
    assert np.array_equal(phys, ref["phys"]), "phys"
    return ref


def colocated_boundaries(E, Q, d, K=8):
    """E experts, one per rank (N = E), whose quota boundaries all fall inside
    the same E/2 consecutive ids.  Loads: experts below E/2 get Q + d, the
    others Q - d, so Q is the quota, every expert below E/2 overflows by d onto
    one replica, and its home range ends at its Q-th occurrence.  Order:
    Q - d rounds of every expert, then 2d rounds of the experts below E/2; the
    Q-th occurrence of expert e is then id (Q - d) * E + d * E/2 + e."""
    half = E // 2
    full = np.tile(np.arange(E, dtype=np.int32), Q - d)
    tail = np.tile(np.arange(half, dtype=np.int32), 2 * d)
    ids = np.concatenate([full, tail])
    assert ids.size % K == 0
    return ids.reshape(-1, K)


@pytest.mark.parametrize("E", [256, 512])
def test_pieces_colocated_boundaries(ctx, E):
    Q, d = 131072, 1024
    ids = colocated_boundaries(E, Q, d)
    ref = _check(ctx, ids, E, E, 1)
    pl = ref["plan"]
    assert int(pl["info"][3]) == E // 2          # every overloaded expert is replicated once
    assert (pl["info"][2] & 1) == 0
    assert int(pl["info"][6]) == Q               # and the plan is perfectly balanced


@pytest.mark.parametrize("tpr,n,s", [(32768, 128, 1.2), (16384, 256, 0.0), (131072, 8, 1.6), (24576, 128, 0.8)])
def test_pieces_sweep_points(ctx, tpr, n, s):
    w = inputs.Workload(f"pieces-{tpr}-{n}-{s}", E=256, K=8, N=n, R=1, tokens_per_rank=tpr, s=s, base_seed=7)
    ids_d = inputs.topk_ids_device(w, 0, "cuda")
    torch.cuda.synchronize()
    _check(ctx, ids_d.cpu().numpy(), w.E, w.N, w.R)


def _ragged_ids(T, K, E, seed, bad_frac=0.0):
    rng = np.random.default_rng(seed)
    p = (rng.permutation(E) + 1.0) ** -1.3
    ids = rng.choice(E, size=(T, K), p=p / p.sum()).astype(np.int32)
    if bad_frac:
        m = rng.random((T, K)) < bad_frac
        ids[m] = rng.choice([-1, -1000, E, E + 5, 2**31 - 1], size=int(m.sum()))
    return ids


@pytest.mark.parametrize("T,K,E,N,R", [
    (160 * 10001, 7, 320, 160, 1),    # ids per rank not a multiple of 4: scalar path
    (200 * 14000, 5, 200, 200, 2),    # odd K, R = 2
    (256 * 16384, 8, 256, 256, 0),    # no redundant slots: every expert has one replica
    (8 * 80000, 8, 64, 8, 4),         # few ranks, many tokens each
])
def test_pieces_edge_shapes(ctx, T, K, E, N, R):
    ids = _ragged_ids(T, K, E, seed=T + K)
    _check(ctx, ids, E, N, R)


def test_pieces_bad_ids(ctx):
    ids = _ragged_ids(256 * 16384, 8, 256, seed=3, bad_frac=0.03)
    ref = _check(ctx, ids, 256, 256, 1)
    assert ref["bad"].sum() > 0


@pytest.mark.parametrize("phys_offset", [0, 1])
def test_pieces_separate_steps(ctx, phys_offset):
    # ue_reroute alone computes the piece rows itself; a phys buffer that is
    # not 16-byte aligned takes the scalar path.
    w = inputs.Workload("pieces-separate", E=256, K=8, N=256, R=1, tokens_per_rank=16384, s=1.2, base_seed=2)
    ids = inputs.topk_ids_device(w, 0, "cuda").cpu().numpy()
    _check(ctx, ids, w.E, w.N, w.R, fused=False, phys_offset=phys_offset)


def test_pieces_plan_variants(ctx):
    w = inputs.Workload("pieces-variants", E=256, K=8, N=256, R=1, tokens_per_rank=16384, s=1.6, base_seed=5)
    ids_np = inputs.topk_ids_device(w, 0, "cuda").cpu().numpy()
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    ids = torch.from_numpy(ids_np).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.empty_like(ids)
    for v in (1, 2, 3):
        names = _launched(lambda: ue.ue_rebalance_ex(ctx, cfg, ids, counts, None, plan, phys, v))
        assert "k_reroute_pieces" in names
        ref = oracle.rebalance(ids_np, w.E, w.N, w.R, variant=v)
        pl = plan.to_host()
        for f in oracle.PLAN_FIELDS:
            assert np.array_equal(pl[f], ref["plan"][f]), (v, f)
        assert np.array_equal(phys.cpu().numpy(), ref["phys"]), v


@pytest.mark.parametrize("E,N,R,tpr,s", [
    (1024, 1024, 1, 16384, 1.2),     # the largest E and N: the workspace caps the pieces per rank
    (1024, 8, 4, 131072, 0.8),       # 128 home experts per rank, four redundant slots each
])
def test_pieces_widest_shapes(ctx, E, N, R, tpr, s):
    w = inputs.Workload(f"pieces-wide-{E}-{N}", E=E, K=8, N=N, R=R, tokens_per_rank=tpr, s=s, base_seed=11)
    ids_d = inputs.topk_ids_device(w, 0, "cuda")
    torch.cuda.synchronize()
    _check(ctx, ids_d.cpu().numpy(), w.E, w.N, w.R)
