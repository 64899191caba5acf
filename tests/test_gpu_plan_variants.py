"""GPU parity of the plan variants (UE_PLAN_REQUEUE, UE_PLAN_SPREAD and both)
against the CPU oracle: every plan array and the rerouted ids bit-exact."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from moe_expert_load_ue_b200 import inputs, ue

pytestmark = pytest.mark.gpu

VARIANTS = (ue.UE_PLAN_REQUEUE, ue.UE_PLAN_SPREAD, ue.UE_PLAN_REQUEUE | ue.UE_PLAN_SPREAD)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "plan_variant_cases.json")


@pytest.fixture(scope="module")
def ctx():
    c = ue.Context(0)
    yield c
    c.close()


def run_variant(ctx, ids_np, E, N, R, variant):
    T, K = ids_np.shape
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np)).cuda()
    counts = torch.full((N, E), -7, dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    for t in plan.tensors.values():
        t.fill_(-99)
    phys = torch.full_like(ids, -5)
    ue.ue_rebalance_ex(ctx, cfg, ids, counts, None, plan, phys, variant)
    torch.cuda.synchronize()
    return plan.to_host(), phys.cpu().numpy()


def assert_variant_equal(ctx, ids, E, N, R, variant):
    pl, phys = run_variant(ctx, ids, E, N, R, variant)
    ref = oracle.rebalance(ids, E, N, R, variant)
    for f in oracle.PLAN_FIELDS:
        assert np.array_equal(pl[f], ref["plan"][f]), (variant, f)
    assert np.array_equal(pl["load"], ref["load"])
    assert np.array_equal(phys, ref["phys"]), variant
    return ref


@pytest.mark.parametrize("w,mb", [(inputs.TINY, 0), (inputs.CLASS_106B, 2), (inputs.CLASS_671B, 0),
                                  (inputs.CLASS_671B, 7), (inputs.EXTREME, 0), (inputs.EXTREME, 5)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_variants_full_size(ctx, w, mb):
    ids = inputs.topk_ids(w, mb)
    for v in VARIANTS:
        assert_variant_equal(ctx, ids, w.E, w.N, w.R, v)


@pytest.mark.parametrize("tpr,n,s", [(256, 256, 1.6), (32768, 8, 0.0), (4096, 64, 0.8), (1024, 128, 1.2),
                                     (16384, 32, 1.6)])
def test_variants_sweep_points(ctx, tpr, n, s):
    w = inputs.Workload(f"sweep-{tpr}-{n}-{s}", E=256, K=8, N=n, R=1, tokens_per_rank=tpr, s=s, base_seed=4)
    ids = inputs.topk_ids(w, 0)
    for v in VARIANTS:
        assert_variant_equal(ctx, ids, w.E, w.N, w.R, v)


def _skewed_ids(T, K, E, seed, hot=2):
    rng = np.random.default_rng(seed)
    p = (rng.permutation(E) + 1.0) ** -1.5
    ids = rng.choice(E, size=(T, K), p=p / p.sum()).astype(np.int32)
    for h in rng.choice(E, size=hot, replace=False):
        ids[rng.random(T) < 0.35, rng.integers(K)] = h        # a few very hot experts: slots run out
    return ids


@pytest.mark.parametrize("T,K,E,N,R", [
    (4096, 8, 64, 8, 2),
    (4096, 8, 64, 16, 3),
    (3 * 37, 3, 24, 3, 2),
    (4096, 8, 64, 8, 0),            # no redundant slots: every variant is the base rule
    (4096, 8, 64, 1, 2),            # a single rank
    (2048 * 8, 2, 1024, 1024, 4),   # maximum E, N and N*R
    (8 * 5000, 8, 1024, 8, 2),
    (64 * 33, 6, 192, 64, 2),
    (32 * 400, 8, 128, 32, 4),
])
def test_variants_edge_shapes(ctx, T, K, E, N, R):
    ids = _skewed_ids(T, K, E, seed=T + E + N)
    for v in VARIANTS:
        assert_variant_equal(ctx, ids, E, N, R, v)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_variant_hand_cases_on_device(ctx, case):
    # counts with every token on rank 0 give the case's loads as column sums
    E, N, R = case["E"], case["N"], case["R"]
    cfg = ue.Config(E=E, N=N, R=R, K=1, T=0)
    counts = torch.zeros((N, E), dtype=torch.int32, device="cuda")
    counts[0] = torch.tensor(case["load"], dtype=torch.int32)
    for v, exp in case["variants"].items():
        plan = ue.Plan(cfg)
        ue.ue_plan_ex(ctx, cfg, counts, plan, int(v))
        torch.cuda.synchronize()
        pl = plan.to_host()
        assert pl["slot_expert"].tolist() == exp["slot_expert"], v
        assert pl["slot_quota"].tolist() == exp["slot_quota"], v
        assert pl["rank_load_after"].tolist() == exp["rank_load_after"], v
        assert int(pl["info"][2] & 1) == exp["flag"], v
