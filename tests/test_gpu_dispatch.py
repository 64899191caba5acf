"""GPU parity of the dispatch layout (routing expansion grouped by physical slot)
against the CPU oracle: phys, slot_off, src_index and gates_out bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_load_ue_b200 import inputs, ue

pytestmark = pytest.mark.gpu

GUARD = 64


@pytest.fixture(scope="module")
def ctx():
    c = ue.Context(0)
    yield c
    c.close()


def run_dispatch(ctx, ids_np, E, N, R, gates_np=None, fused=True, plan_ids=None):
    """Device rebalance with the dispatch layout.  src_index / gates_out carry
    GUARD sentinel entries past T*K that the kernel must never touch."""
    T, K = ids_np.shape
    L = T * K
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np)).cuda()
    counts = torch.full((N, E), -7, dtype=torch.int32, device="cuda")
    bad = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.full_like(ids, -5)
    disp = ue.Dispatch(cfg, with_gates=gates_np is not None)
    src_big = torch.full((L + GUARD,), -3, dtype=torch.int32, device="cuda")
    gout_big = torch.full((L + GUARD,), -3.0, dtype=torch.float32, device="cuda")
    disp.src_index = src_big[:L]
    if gates_np is not None:
        disp.gates_out = gout_big[:L]
    disp.slot_off.fill_(-9)
    gates = None if gates_np is None else torch.from_numpy(np.ascontiguousarray(gates_np)).cuda()
    if plan_ids is not None:                    # a plan computed from other ids
        pids = torch.from_numpy(np.ascontiguousarray(plan_ids)).cuda()
        ue.ue_rebalance(ctx, cfg, pids, counts, bad, plan, phys)
        ue.ue_dispatch(ctx, cfg, ids, plan, phys, disp, gates)
    elif fused:
        ue.ue_rebalance_dispatch(ctx, cfg, ids, counts, bad, plan, phys, disp, gates)
    else:
        ue.ue_load(ctx, cfg, ids, counts, bad)
        ue.ue_plan(ctx, cfg, counts, plan)
        ue.ue_dispatch(ctx, cfg, ids, plan, phys, disp, gates)
    torch.cuda.synchronize()
    return {"phys": phys.cpu().numpy(), "slot_off": disp.slot_off.cpu().numpy(),
            "src_big": src_big.cpu().numpy(), "gout_big": gout_big.cpu().numpy(), "plan": plan.to_host(),
            "L": L, "S": cfg.S}


def assert_dispatch_equal(got, ids, E, N, R, gates=None):
    ref = oracle.rebalance(ids, E, N, R)
    assert np.array_equal(got["phys"], ref["phys"]), "phys"
    for f in oracle.PLAN_FIELDS:
        assert np.array_equal(got["plan"][f], ref["plan"][f]), f
    slot_off, src, gout = oracle.dispatch(ref["phys"], got["S"], gates)
    assert np.array_equal(got["slot_off"], slot_off), "slot_off"
    n, L = int(slot_off[-1]), got["L"]
    assert np.array_equal(got["src_big"][:n], src), "src_index"
    assert (got["src_big"][n:] == -3).all(), "src_index written past slot_off[S]"
    if gates is None:
        assert (got["gout_big"] == -3.0).all()
    else:
        assert np.array_equal(got["gout_big"][:n].view(np.uint32), gout.view(np.uint32)), "gates_out"
        assert (got["gout_big"][n:] == -3.0).all()
    assert n <= L


WORKLOADS = [(inputs.TINY, 0), (inputs.CLASS_106B, 3), (inputs.CLASS_671B, 0), (inputs.CLASS_671B, 11),
             (inputs.EXTREME, 2)]


@pytest.mark.parametrize("w,mb", WORKLOADS, ids=lambda x: getattr(x, "name", str(x)))
def test_dispatch_full_size(ctx, w, mb):
    ids = inputs.topk_ids(w, mb)
    gates = inputs.gates(ids, w, mb)
    assert_dispatch_equal(run_dispatch(ctx, ids, w.E, w.N, w.R, gates), ids, w.E, w.N, w.R, gates)


@pytest.mark.parametrize("w", [inputs.TINY, inputs.EXTREME], ids=lambda w: w.name)
def test_dispatch_separate_calls_and_no_gates(ctx, w):
    ids = inputs.topk_ids(w, 1)
    assert_dispatch_equal(run_dispatch(ctx, ids, w.E, w.N, w.R, None, fused=False), ids, w.E, w.N, w.R)


def test_dispatch_phys_equals_reroute(ctx):
    w = inputs.CLASS_671B
    ids = inputs.topk_ids(w, 5)
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    d_ids = torch.from_numpy(ids).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    p1 = torch.full_like(d_ids, -5)
    p2 = torch.full_like(d_ids, -6)
    ue.ue_rebalance(ctx, cfg, d_ids, counts, None, plan, p1)
    ue.ue_dispatch(ctx, cfg, d_ids, plan, p2, ue.Dispatch(cfg, with_gates=False))
    torch.cuda.synchronize()
    assert torch.equal(p1, p2)


def _ragged_ids(T, K, E, seed, bad_frac=0.0):
    rng = np.random.default_rng(seed)
    p = (rng.permutation(E) + 1.0) ** -1.3
    ids = rng.choice(E, size=(T, K), p=p / p.sum()).astype(np.int32)
    if bad_frac:
        m = rng.random((T, K)) < bad_frac
        ids[m] = rng.choice([-1, -1000, E, E + 5, 2**31 - 1], size=int(m.sum()))
    return ids


@pytest.mark.parametrize("T,K,E,N,R", [
    (0, 8, 64, 8, 2),               # empty microbatch: slot_off all zero
    (24, 1, 16, 4, 1),
    (3 * 37, 3, 24, 3, 2),          # unaligned rank boundaries (scalar path)
    (5 * 1001, 5, 40, 5, 3),
    (4096, 8, 64, 8, 0),            # no redundant slots
    (4096, 8, 64, 1, 2),            # a single rank
    (2048 * 8, 2, 1024, 1024, 4),   # maximum E, N and N*R (ids not staged)
    (8 * 5000, 8, 1024, 8, 2),
    (16 * 20000, 8, 256, 16, 1),    # CTA shares larger than the staging buffer
])
def test_dispatch_edge_shapes(ctx, T, K, E, N, R):
    ids = _ragged_ids(T, K, E, seed=T + 3 * K + E)
    gates = np.random.default_rng(T + 1).random((T, K), dtype=np.float32)
    assert_dispatch_equal(run_dispatch(ctx, ids, E, N, R, gates), ids, E, N, R, gates)


def test_dispatch_bad_ids_not_dispatched(ctx):
    ids = _ragged_ids(9 * 513, 5, 72, seed=4, bad_frac=0.05)
    gates = np.random.default_rng(2).random(ids.shape, dtype=np.float32)
    got = run_dispatch(ctx, ids, 72, 9, 2, gates)
    assert_dispatch_equal(got, ids, 72, 9, 2, gates)
    assert got["slot_off"][-1] == ((ids >= 0) & (ids < 72)).sum()


def test_dispatch_plan_from_other_ids_is_reported(ctx):
    E, N, R = 64, 8, 2
    ids = _ragged_ids(8 * 512, 8, E, seed=10)
    other = _ragged_ids(8 * 512, 8, E, seed=11)
    ctx.device_error()                         # clear
    got = run_dispatch(ctx, ids, E, N, R, None, plan_ids=other)
    assert ctx.device_error() & 2
    assert (got["src_big"][got["L"]:] == -3).all()
    assert got["slot_off"][-1] <= got["L"]
