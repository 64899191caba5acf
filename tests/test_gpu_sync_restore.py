"""GPU parity of the weight restore in backward (ue_sync_restore).

A stack of layers shares the redundant slots: forward syncs each layer's
replicas (incrementally, from the previous layer's plan), backward restores
each layer's replicas, last layer first, from the experts the slots hold.
After every call the whole weight buffer must equal the oracle's replay of the
same calls byte for byte.
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


def _layer_plans(ctx, w, n):
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    plans = []
    for mb in range(n):
        ids = torch.from_numpy(inputs.topk_ids(w, mb)).cuda()
        counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
        plan = ue.Plan(cfg)
        ue.ue_rebalance(ctx, cfg, ids, counts, None, plan, torch.empty_like(ids))
        plans.append(plan)
    torch.cuda.synchronize()
    return cfg, plans


@pytest.mark.parametrize("w", [inputs.TINY, inputs.CLASS_671B.with_(tokens_per_rank=256),
                               inputs.CLASS_106B.with_(tokens_per_rank=256), inputs.EXTREME.with_(tokens_per_rank=128)],
                         ids=lambda w: w.name)
def test_restore_layer_stack_matches_oracle(ctx, w):
    layers = 5
    cfg, plans = _layer_plans(ctx, w, layers)
    se = [p["slot_expert"].cpu().numpy() for p in plans]
    slot_bytes = 64 * 1024 + 16
    g = torch.Generator(device="cuda").manual_seed(7)
    W = torch.randint(0, 256, (w.S, slot_bytes), dtype=torch.uint8, device="cuda", generator=g)
    Wh = W.cpu().numpy()
    H, HR = w.H, w.H + w.R
    red = (np.arange(w.S) % HR) >= H
    held = np.full(w.S, -1, np.int32)
    for li in range(layers):          # forward
        prev = plans[li - 1]["slot_expert"] if li else None
        ue.ue_sync_delta(ctx, cfg, W, slot_bytes, plans[li], prev)
        oracle.sync_delta(Wh, slot_bytes, w.E, w.N, w.R, se[li], se[li - 1] if li else None)
        held = np.where(red & (se[li] >= 0), se[li], held)
    torch.cuda.synchronize()
    assert np.array_equal(W.cpu().numpy(), Wh)
    restored = 0
    for li in reversed(range(layers)):   # backward
        held_d = torch.from_numpy(held).cuda()
        ue.ue_sync_restore(ctx, cfg, W, slot_bytes, plans[li], held_d)
        restored += oracle.sync_restore(Wh, slot_bytes, w.E, w.N, w.R, se[li], held)
        torch.cuda.synchronize()
        assert np.array_equal(W.cpu().numpy(), Wh), f"layer {li}"
        held = np.where(red & (se[li] >= 0), se[li], held)
    assert restored > 0
    assert ctx.device_error() == 0


def test_restore_unknown_holder_is_full_sync(ctx):
    w = inputs.CLASS_671B.with_(tokens_per_rank=256)
    cfg, (plan,) = _layer_plans(ctx, w, 1)
    slot_bytes = 48 * 1024 * 3 - 16
    W = torch.randint(0, 256, (w.S, slot_bytes), dtype=torch.uint8, device="cuda",
                      generator=torch.Generator(device="cuda").manual_seed(9))
    expect = W.cpu().numpy()
    ue.ue_sync_restore(ctx, cfg, W, slot_bytes, plan, None)
    torch.cuda.synchronize()
    oracle.sync(expect, slot_bytes, w.E, w.N, w.R, plan["slot_expert"].cpu().numpy())
    assert np.array_equal(W.cpu().numpy(), expect)
