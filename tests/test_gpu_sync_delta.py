"""GPU parity of the incremental replica weight sync against the CPU oracle:
over a sequence of microbatch plans, each device call writes exactly the bytes
the oracle writes (bit-exact), and slots whose expert is unchanged are not
written."""
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


def _device_plan(ctx, w, mb, ids_np=None):
    ids_np = inputs.topk_ids(w, mb) if ids_np is None else ids_np
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=ids_np.shape[0])
    ids = torch.from_numpy(ids_np).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.empty_like(ids)
    ue.ue_rebalance(ctx, cfg, ids, counts, None, plan, phys)
    torch.cuda.synchronize()
    return cfg, plan


def _run_sequence(ctx, w, n_mb, slot_bytes, stationary_every=0):
    """Full sync for the first microbatch, then incremental syncs; the oracle
    replays the same sequence on a host copy.  With stationary_every = k,
    every k-th microbatch reuses the previous microbatch's routing (its plan
    is then identical and the sync must write nothing)."""
    g = torch.Generator(device="cuda").manual_seed(21)
    W = torch.randint(0, 256, (w.S, slot_bytes), dtype=torch.uint8, device="cuda", generator=g)
    host = W.cpu().numpy()
    prev_plan, prev_host = None, None
    ids_prev = None
    copied = []
    for mb in range(n_mb):
        ids_np = ids_prev if (stationary_every and mb % stationary_every == 1 and ids_prev is not None) \
            else inputs.topk_ids(w, mb)
        cfg, plan = _device_plan(ctx, w, mb, ids_np)
        pl = plan.to_host()
        ue.ue_sync_delta(ctx, cfg, W, slot_bytes, plan, None if prev_plan is None else prev_plan["slot_expert"])
        torch.cuda.synchronize()
        assert ctx.device_error() == 0
        n = oracle.sync_delta(host, slot_bytes, w.E, w.N, w.R, pl["slot_expert"], prev_host)
        assert np.array_equal(W.cpu().numpy(), host), mb
        copied.append(n)
        prev_plan, prev_host, ids_prev = plan, pl["slot_expert"], ids_np
    return copied


def test_sync_delta_tiny_stationary(ctx):
    # stationary popularity: the plans barely move, most slots are kept
    w = inputs.TINY
    copied = _run_sequence(ctx, w, 4, 48 * 1024 + 16, stationary_every=2)
    assert copied[0] > 0 and copied[1] == 0


@pytest.mark.parametrize("w", [inputs.CLASS_671B.with_(tokens_per_rank=512), inputs.EXTREME.with_(tokens_per_rank=256),
                               inputs.CLASS_106B.with_(tokens_per_rank=1024)], ids=lambda w: w.name)
def test_sync_delta_sequences(ctx, w):
    copied = _run_sequence(ctx, w, 5, 3 * 48 * 1024 - 32, stationary_every=3)
    assert copied[0] > 0


def test_sync_delta_null_prev_is_full_sync(ctx):
    w = inputs.TINY
    cfg, plan = _device_plan(ctx, w, 0)
    pl = plan.to_host()
    slot_bytes = 4096
    g = torch.Generator(device="cuda").manual_seed(3)
    W1 = torch.randint(0, 256, (w.S, slot_bytes), dtype=torch.uint8, device="cuda", generator=g)
    W2 = W1.clone()
    ue.ue_sync(ctx, cfg, W1, slot_bytes, plan)
    ue.ue_sync_delta(ctx, cfg, W2, slot_bytes, plan, None)
    torch.cuda.synchronize()
    assert torch.equal(W1, W2)
    # prev = the same plan: nothing to write
    W3 = W1.clone()
    W3[w.S - 1].zero_()      # a redundant slot now stale on purpose: the delta must not touch it
    ue.ue_sync_delta(ctx, cfg, W3, slot_bytes, plan, plan["slot_expert"])
    torch.cuda.synchronize()
    expect = W1.clone()
    expect[w.S - 1].zero_()
    assert torch.equal(W3, expect)
    assert pl["info"][4] > 0
