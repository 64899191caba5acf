"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer steps (load, plan, reroute) and the weight copy must be bit-exact.
Gradient reduction must hold |gpu - oracle| <= 1e-5 * (|G0| + sum |g_i|) + 1e-30
per element (fp32 accumulation); with the same replica order it is in fact exact.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_load_ue_b200 import inputs, ue

pytestmark = pytest.mark.gpu

GRAD_RTOL = 1e-5


@pytest.fixture(scope="module")
def ctx():
    c = ue.Context(0)
    yield c
    c.close()


def run_rebalance(ctx, ids_np, E, N, R, fused=True, plan=None):
    T, K = ids_np.shape
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np)).cuda()
    counts = torch.full((N, E), -7, dtype=torch.int32, device="cuda")
    bad = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    plan = plan or ue.Plan(cfg)
    for t in plan.tensors.values():
        t.fill_(-99)
    phys = torch.full_like(ids, -5)
    if fused:
        ue.ue_rebalance(ctx, cfg, ids, counts, bad, plan, phys)
    else:
        ue.ue_load(ctx, cfg, ids, counts, bad)
        ue.ue_plan(ctx, cfg, counts, plan)
        ue.ue_reroute(ctx, cfg, ids, plan, phys)
    torch.cuda.synchronize()
    return {"counts": counts.cpu().numpy(), "bad": bad.cpu().numpy(), "plan": plan.to_host(),
            "phys": phys.cpu().numpy(), "plan_obj": plan, "cfg": cfg}


def assert_rebalance_equal(got, ids, E, N, R):
    ref = oracle.rebalance(ids, E, N, R)
    assert np.array_equal(got["counts"], ref["counts"]), "counts"
    assert np.array_equal(got["bad"], ref["bad"]), "bad"
    pl = got["plan"]
    for f in oracle.PLAN_FIELDS:
        assert np.array_equal(pl[f], ref["plan"][f]), f
    assert np.array_equal(pl["load"], ref["load"]), "load"
    assert np.array_equal(pl["rank_off"], ref["rank_off"]), "rank_off"
    assert np.array_equal(got["phys"], ref["phys"]), "phys"
    return ref


# ---- load + plan + reroute ---------------------------------------------------------

WORKLOADS = [
    (inputs.TINY, 0),
    (inputs.CLASS_106B, 0), (inputs.CLASS_106B, 9),
    (inputs.CLASS_671B, 0), (inputs.CLASS_671B, 15),
    (inputs.EXTREME, 0), (inputs.EXTREME, 4),
]


@pytest.mark.parametrize("w,mb", WORKLOADS, ids=lambda x: getattr(x, "name", str(x)))
def test_rebalance_full_size(ctx, w, mb):
    ids = inputs.topk_ids(w, mb)
    got = run_rebalance(ctx, ids, w.E, w.N, w.R)
    ref = assert_rebalance_equal(got, ids, w.E, w.N, w.R)
    if w.hot_fraction:
        assert ref["plan"]["info"][2] & 1      # the hot expert exhausts the slots


@pytest.mark.parametrize("w", [inputs.TINY, inputs.CLASS_671B, inputs.EXTREME], ids=lambda w: w.name)
def test_separate_steps_equal_fused(ctx, w):
    ids = inputs.topk_ids(w, 1)
    a = run_rebalance(ctx, ids, w.E, w.N, w.R, fused=True)
    b = run_rebalance(ctx, ids, w.E, w.N, w.R, fused=False)
    for k in ("counts", "bad", "phys"):
        assert np.array_equal(a[k], b[k])
    for f in ue.PLAN_FIELDS:
        assert np.array_equal(a["plan"][f], b["plan"][f])


SWEEP_POINTS = [(256, 256, 1.6), (32768, 8, 0.0), (4096, 64, 0.8), (1024, 128, 1.2), (16384, 32, 1.6),
                (256, 8, 1.2), (1024, 32, 0.0)]


@pytest.mark.parametrize("tpr,n,s", SWEEP_POINTS)
def test_rebalance_sweep_points(ctx, tpr, n, s):
    w = inputs.Workload(f"sweep-{tpr}-{n}-{s}", E=256, K=8, N=n, R=1, tokens_per_rank=tpr, s=s, base_seed=3)
    ids = inputs.topk_ids(w, 0)
    assert_rebalance_equal(run_rebalance(ctx, ids, w.E, w.N, w.R), ids, w.E, w.N, w.R)


def _ragged_ids(T, K, E, seed, bad_frac=0.0):
    rng = np.random.default_rng(seed)
    p = (rng.permutation(E) + 1.0) ** -1.3
    ids = rng.choice(E, size=(T, K), p=p / p.sum()).astype(np.int32)   # duplicates within a token allowed
    if bad_frac:
        m = rng.random((T, K)) < bad_frac
        ids[m] = rng.choice([-1, -1000, E, E + 5, 2**31 - 1], size=int(m.sum()))
    return ids


@pytest.mark.parametrize("T,K,E,N,R", [
    (0, 8, 64, 8, 2),          # empty microbatch
    (24, 1, 16, 4, 1),         # tiny, K = 1
    (3 * 37, 3, 24, 3, 2),     # odd K and tokens per rank: unaligned rank boundaries
    (5 * 1001, 5, 40, 5, 3),   # ragged CTA and warp shares
    (7 * 997, 7, 56, 7, 1),
    (4096, 8, 64, 8, 0),       # no redundant slots
    (4096, 8, 64, 1, 2),       # a single rank
    (2048 * 8, 2, 1024, 1024, 4),   # maximum E, N and N*R
    (8 * 5000, 8, 1024, 8, 2),      # maximum E with few ranks
    (64 * 33, 6, 192, 64, 2),
])
def test_rebalance_edge_shapes(ctx, T, K, E, N, R):
    ids = _ragged_ids(T, K, E, seed=T + K + E)
    assert_rebalance_equal(run_rebalance(ctx, ids, E, N, R), ids, E, N, R)


def test_rebalance_bad_ids(ctx):
    ids = _ragged_ids(9 * 513, 5, 72, seed=4, bad_frac=0.05)
    got = run_rebalance(ctx, ids, 72, 9, 2)
    assert got["bad"].sum() > 0
    assert_rebalance_equal(got, ids, 72, 9, 2)
    assert (got["phys"][(ids < 0) | (ids >= 72)] == -1).all()


def test_rebalance_one_hot_expert_runs_out(ctx):
    T, K, E, N, R = 4096, 4, 64, 16, 1
    ids = np.full((T, K), 5, np.int32)
    ids[:, 1:] = _ragged_ids(T, K - 1, E, seed=1)
    got = run_rebalance(ctx, ids, E, N, R)
    ref = assert_rebalance_equal(got, ids, E, N, R)
    assert ref["plan"]["info"][2] & 1


def test_rebalance_all_ids_identical(ctx):
    ids = np.full((8 * 1024, 8), 3, np.int32)
    assert_rebalance_equal(run_rebalance(ctx, ids, 32, 8, 4), ids, 32, 8, 4)


def test_plan_buffers_reused_across_microbatches(ctx):
    w = inputs.CLASS_671B
    plan = ue.Plan(ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T))
    for mb in (2, 3):
        ids = inputs.topk_ids(w, mb)
        assert_rebalance_equal(run_rebalance(ctx, ids, w.E, w.N, w.R, plan=plan), ids, w.E, w.N, w.R)


# ---- weight sync -----------------------------------------------------------------

def _plan_for(ctx, w, mb):
    ids = inputs.topk_ids(w, mb)
    got = run_rebalance(ctx, ids, w.E, w.N, w.R)
    return got["plan_obj"], got["plan"], got["cfg"]


def _check_sync_full(ctx, w, slot_bytes, mb=0):
    plan, pl, cfg = _plan_for(ctx, w, mb)
    g = torch.Generator(device="cuda").manual_seed(11)
    W = torch.randint(0, 256, (w.S, slot_bytes), dtype=torch.uint8, device="cuda", generator=g)
    before = W.cpu().numpy()
    ue.ue_sync(ctx, cfg, W, slot_bytes, plan)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    expect = before.copy()
    oracle.sync(expect, slot_bytes, w.E, w.N, w.R, pl["slot_expert"])
    assert np.array_equal(W.cpu().numpy(), expect)
    return pl


def test_sync_tiny_full(ctx):
    w = inputs.TINY
    pl = _check_sync_full(ctx, w, 2 * w.P)
    assert pl["info"][4] > 0


@pytest.mark.parametrize("slot_bytes", [16, 48 * 1024, 48 * 1024 + 16, 3 * 48 * 1024 - 32, 1 << 20])
def test_sync_ragged_tiles(ctx, slot_bytes):
    _check_sync_full(ctx, inputs.CLASS_671B.with_(tokens_per_rank=256), slot_bytes, mb=3)


def test_sync_store_depth_switch(ctx):
    # The sync's CTAs leave three store groups in flight when they stream 16 or
    # more tiles of 48 KiB, one otherwise: a slot size that gives about half the
    # CTAs 16 tiles and the others 15 runs both in one launch.
    w = inputs.TINY
    _, pl, _ = _plan_for(ctx, w, 0)
    M = int(pl["info"][3])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ntiles = -(-(15 * sms + sms // 2) // M)
    slot_bytes = ntiles * 48 * 1024 - 48            # a ragged last tile
    total = M * ntiles
    assert total // sms == 15 and total % sms > 0
    _check_sync_full(ctx, w, slot_bytes)


def test_sync_extreme_fanout(ctx):
    # the hot expert fans out to many replicas: each of its tiles is read once, written ~10 times
    w = inputs.EXTREME
    pl = _check_sync_full(ctx, w, 4 * 48 * 1024 + 1024)
    off = pl["rep_off"]
    assert (np.diff(off) - 1).max() >= 8


# ---- grad reduce ----------------------------------------------------------------

def _grad_tolerance_ok(got, expect, master0, grads_abs_sum):
    bound = GRAD_RTOL * (np.abs(master0).astype(np.float64) + grads_abs_sum) + 1e-30
    return np.all(np.abs(got.astype(np.float64) - expect.astype(np.float64)) <= bound)


def _grad_abs_sum(gw, pl, E, N, R, is_bf16):
    H, HR = E // N, E // N + R
    acc = np.zeros((E, gw.shape[1]), np.float64)
    g = (gw.astype(np.uint32) << 16).view(np.float32) if is_bf16 else gw
    off = pl["rep_off"]
    for e in range(E):
        for i in range(off[e] + 1, off[e + 1]):
            s = pl["rep_slot"][i]
            acc[e] += np.abs(g[(s // HR) * R + (s % HR - H)])
    return acc


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_grad_reduce_tiny_full(ctx, dtype):
    w = inputs.TINY
    plan, pl, cfg = _plan_for(ctx, w, 0)
    P = w.P
    gen = torch.Generator(device="cuda").manual_seed(21)
    master = torch.randn((w.E, P), generator=gen, device="cuda") * 1e-3
    gt = torch.float32 if dtype == "fp32" else torch.bfloat16
    grads = (torch.randn((w.N * w.R, P), generator=gen, device="cuda") * 1e-3).to(gt)
    m0 = master.cpu().numpy()
    gh = grads.cpu().numpy() if dtype == "fp32" else grads.view(torch.int16).cpu().numpy().view(np.uint16)
    ue.ue_grad_reduce(ctx, cfg, master, grads, P, plan)
    torch.cuda.synchronize()
    expect = m0.copy()
    oracle.grad_reduce(expect, gh, P, w.E, w.N, w.R, pl)
    got = master.cpu().numpy()
    assert _grad_tolerance_ok(got, expect, m0, _grad_abs_sum(gh, pl, w.E, w.N, w.R, dtype == "bf16"))
    assert np.array_equal(got, expect)          # same order of fp32 adds: bit-exact


@pytest.mark.parametrize("P", [8, 2040, 2048, 2056, 4096 + 8 * 37])
def test_grad_reduce_ragged_chunks(ctx, P):
    w = inputs.EXTREME.with_(tokens_per_rank=64)
    plan, pl, cfg = _plan_for(ctx, w, 2)
    gen = torch.Generator(device="cuda").manual_seed(P)
    master = torch.randn((w.E, P), generator=gen, device="cuda")
    grads = torch.randn((w.N * w.R, P), generator=gen, device="cuda")
    m0, gh = master.cpu().numpy(), grads.cpu().numpy()
    ue.ue_grad_reduce(ctx, cfg, master, grads, P, plan)
    torch.cuda.synchronize()
    expect = m0.copy()
    oracle.grad_reduce(expect, gh, P, w.E, w.N, w.R, pl)
    assert np.array_equal(master.cpu().numpy(), expect)


def test_grad_reduce_no_redundant_slots(ctx):
    ids = _ragged_ids(4096, 8, 64, seed=9)
    got = run_rebalance(ctx, ids, 64, 8, 0)
    master = torch.randn((64, 1024), device="cuda")
    m0 = master.clone()
    ue.ue_grad_reduce(ctx, got["cfg"], master, torch.empty(0, device="cuda"), 1024, got["plan_obj"])
    torch.cuda.synchronize()
    assert torch.equal(master, m0)
