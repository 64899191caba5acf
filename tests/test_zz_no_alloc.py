"""ue_reroute_static: routing expansion for callers that cannot allocate.

Some callers cannot call cudaMalloc - an engine that reserves its whole
device-memory budget in its own pool at start-up, or a caller in a region of
its framework where allocation is not allowed - and so cannot create a context.
ue_reroute_static keeps its scratch in a device array the library holds, and
must give the same phys as ue_reroute.  Checked through the C ABI, bit for bit
(routing is integer work), on two calls in a row, the second on another shape,
so that what the first call leaves in the shared array cannot leak into the
second.  This file is collected last; it passes alone in a fresh process too
(the first call on the device does the set-up).
"""
import numpy as np
import pytest
import torch

from moe_expert_load_ue_b200 import inputs, ue


def _phys_both_ways(ctx, w, mb):
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    ids = torch.from_numpy(inputs.topk_ids(w, mb)).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    ue.ue_load(ctx, cfg, ids, counts, None)
    ue.ue_plan(ctx, cfg, counts, plan)
    ref = torch.full_like(ids, -5)
    ue.ue_reroute(ctx, cfg, ids, plan, ref)
    got = torch.full_like(ids, -7)
    ue.ue_reroute_static(cfg, ids, plan, got)
    torch.cuda.synchronize()
    return got.cpu().numpy(), ref.cpu().numpy()


@pytest.mark.gpu
def test_static_reroute_equals_reroute_twice():
    ctx = ue.Context(0)
    try:
        for w, mb in ((inputs.CLASS_671B, 3), (inputs.EXTREME, 5)):
            got, ref = _phys_both_ways(ctx, w, mb)
            assert (ref >= 0).all()
            assert np.array_equal(got, ref), w.name
    finally:
        ctx.close()


def test_static_reroute_refuses_beyond_its_scratch():
    # 2 * N * (E + 1) + 64 ints must fit 2^20: N = E = 1024 does not; refused
    # on the host before any device call, with the output untouched.
    import ctypes
    cfg = ue.Config(E=1024, N=1024, R=1, K=8, T=1024)
    ue.lib()
    arrays = [np.zeros(8, np.int32) for _ in ue.PLAN_FIELDS]
    pb = ue.UePlanBuffers(*[a.ctypes.data for a in arrays])
    ids = np.zeros(1024 * 8 + 4, np.int32)
    phys = np.full(1024 * 8, 3, np.int32)
    base = ids.ctypes.data
    aligned = base + (-base) % 16
    st = ue.lib().ue_reroute_static(ctypes.byref(cfg.c()), aligned, ctypes.byref(pb), phys.ctypes.data, None)
    assert st == ue.UE_ERR_INVALID_ARG
    assert "static scratch" in ue.lib().ue_last_error().decode()
    assert (phys == 3).all()
