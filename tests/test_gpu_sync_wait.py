"""Bounded waits of the bulk-copy rings: the way out when a wait runs out.

Every mbarrier wait of the weight-sync kernels and of the gradient reduction
is bounded by the context's wait limit.  The diagnostic flag UE_WAIT_STALL_ONCE makes the first CTA of the
next sync wait once, with its first copies in flight, on a barrier that nothing
completes, so that the wait runs out without any fault: the kernel must set bit
0 of the status word, let its copies in flight land, drain its stores and
return, leaving the context and the GPU usable, so that the next sync on the
same context is byte-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_expert_load_ue_b200 import inputs, ue

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000        # 1 ms: far above one tile's copy, far below a hang


@pytest.fixture(scope="module")
def ctx():
    c = ue.Context(0)
    yield c
    c.close()


def _plan(ctx, w, mb=0):
    ids = torch.from_numpy(inputs.topk_ids(w, mb)).cuda()
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.empty_like(ids)
    ue.ue_rebalance(ctx, cfg, ids, counts, None, plan, phys)
    torch.cuda.synchronize()
    return cfg, plan, plan.to_host()


def _weights(w, slot_bytes, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randint(0, 256, (w.S, slot_bytes), dtype=torch.uint8, device="cuda", generator=g)


def test_short_limit_alone_gives_no_false_expiry(ctx):
    w = inputs.CLASS_671B.with_(tokens_per_rank=256)
    cfg, plan, pl = _plan(ctx, w)
    slot_bytes = 4 << 20
    W = _weights(w, slot_bytes, 1)
    expect = W.cpu().numpy()
    ctx.set_wait_limit(LIMIT_NS, 0)
    try:
        ue.ue_sync(ctx, cfg, W, slot_bytes, plan)
        torch.cuda.synchronize()
        assert ctx.device_error() == 0
    finally:
        ctx.set_wait_limit(2_000_000_000, 0)
    oracle.sync(expect, slot_bytes, w.E, w.N, w.R, pl["slot_expert"])
    assert np.array_equal(W.cpu().numpy(), expect)


@pytest.mark.parametrize("call", ["sync", "sync_delta", "sync_shard"])
def test_wait_runs_out_then_context_is_usable(ctx, call):
    w = inputs.CLASS_671B.with_(tokens_per_rank=256)
    cfg, plan, pl = _plan(ctx, w, 1)
    slot_bytes = 4 << 20          # several tiles per CTA, so copies are in flight at the stall
    G = 2
    SG = w.S // G

    def run(W):
        if call == "sync":
            ue.ue_sync(ctx, cfg, W, slot_bytes, plan)
        elif call == "sync_delta":
            ue.ue_sync_delta(ctx, cfg, W, slot_bytes, plan, None)
        else:
            for g in range(G):
                ue.ue_sync_shard(ctx, cfg, G, g, [W[h * SG] for h in range(G)], slot_bytes, plan, -1)

    W = _weights(w, slot_bytes, 2)
    ctx.set_wait_limit(LIMIT_NS, ue.UE_WAIT_STALL_ONCE)
    try:
        run(W)
        torch.cuda.synchronize()
        assert ctx.device_error() & 1, "the stalled wait must report that it gave up"
    finally:
        ctx.set_wait_limit(2_000_000_000, 0)
    # The flag cleared itself: the same call now completes, byte-exact.
    W = _weights(w, slot_bytes, 3)
    expect = W.cpu().numpy()
    run(W)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    oracle.sync(expect, slot_bytes, w.E, w.N, w.R, pl["slot_expert"])
    assert np.array_equal(W.cpu().numpy(), expect)


def test_grad_reduce_wait_runs_out_then_context_is_usable(ctx):
    w = inputs.CLASS_671B.with_(tokens_per_rank=256, rows=512, cols=512)
    cfg, plan, pl = _plan(ctx, w, 2)
    P = w.P
    g = torch.Generator(device="cuda").manual_seed(4)
    master = torch.randn((w.E, P), generator=g, device="cuda")
    grads = torch.randn((w.N * w.R, P), generator=g, device="cuda").to(torch.bfloat16)
    ctx.set_wait_limit(LIMIT_NS, ue.UE_WAIT_STALL_ONCE)
    try:
        ue.ue_grad_reduce(ctx, cfg, master, grads, P, plan)
        torch.cuda.synchronize()
        assert ctx.device_error() & 1, "the stalled wait must report that it gave up"
    finally:
        ctx.set_wait_limit(2_000_000_000, 0)
    master = torch.randn((w.E, P), generator=g, device="cuda")
    m0 = master.cpu().numpy()
    ue.ue_grad_reduce(ctx, cfg, master, grads, P, plan)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    expect = m0.copy()
    oracle.grad_reduce(expect, grads.view(torch.int16).cpu().numpy().view(np.uint16), P, w.E, w.N, w.R, pl)
    assert np.array_equal(master.cpu().numpy(), expect)
