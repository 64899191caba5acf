"""GPU parity of the calls across GPUs against the CPU oracle, with the G GPUs
emulated as parts of one device's memory (each call gets the parts' base
addresses exactly as it would get peer-mapped addresses).  Each call is an
independent launch; none waits on another.

- load / reroute of each GPU's ranks: counts rows and phys slices bit-exact;
- weight sync, relay rounds: after every round the slots equal the oracle's
  relay round (bit-exact), and after the last the single-GPU sync; the direct
  form in one call per GPU;
- gradient reduction on the home GPUs: bit-exact to the oracle (fp32, bf16).
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


def _rebalance_sharded(ctx, ids_np, E, N, R, G):
    T, K = ids_np.shape
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np)).cuda()
    counts = torch.full((N, E), -7, dtype=torch.int32, device="cuda")
    bad = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    n = T // G
    local = [ids[g * n:(g + 1) * n].clone() for g in range(G)]    # each GPU's own (aligned) buffer
    for g in reversed(range(G)):
        ue.ue_load_shard(ctx, cfg, G, g, local[g], counts, bad)
    plan = ue.Plan(cfg)
    ue.ue_plan(ctx, cfg, counts, plan)
    phys = torch.full_like(ids, -5)                               # slices: some not 16-byte aligned
    for g in range(G):
        ue.ue_reroute_shard(ctx, cfg, G, g, local[g], plan, phys[g * n:(g + 1) * n])
    torch.cuda.synchronize()
    return cfg, counts.cpu().numpy(), bad.cpu().numpy(), plan, phys.cpu().numpy()


SHARD_CASES = [(inputs.TINY, (1, 2, 4, 8)), (inputs.CLASS_671B, (2, 8, 64)), (inputs.EXTREME, (4, 128)),
               (inputs.CLASS_106B, (8,))]


@pytest.mark.parametrize("w,Gs", SHARD_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_load_and_reroute_shards(ctx, w, Gs):
    ids = inputs.topk_ids(w, 3)
    ref = oracle.rebalance(ids, w.E, w.N, w.R)
    for G in Gs:
        cfg, counts, bad, plan, phys = _rebalance_sharded(ctx, ids, w.E, w.N, w.R, G)
        assert np.array_equal(counts, ref["counts"]), G
        assert np.array_equal(bad, ref["bad"]), G
        pl = plan.to_host()
        for f in oracle.PLAN_FIELDS:
            assert np.array_equal(pl[f], ref["plan"][f]), (G, f)
        assert np.array_equal(phys, ref["phys"]), G


def test_load_and_reroute_shards_ragged_and_bad_ids(ctx):
    rng = np.random.default_rng(5)
    E, N, R, K = 48, 12, 2, 3
    T = N * 37                                   # unaligned rank shares
    ids = rng.integers(0, E, size=(T, K)).astype(np.int32)
    ids[rng.random((T, K)) < 0.03] = -1
    ids[5, 1] = E + 9
    ref = oracle.rebalance(ids, E, N, R)
    for G in (2, 3, 4, 6, 12):
        _, counts, bad, plan, phys = _rebalance_sharded(ctx, ids, E, N, R, G)
        assert np.array_equal(counts, ref["counts"]) and np.array_equal(bad, ref["bad"])
        assert np.array_equal(phys, ref["phys"])


def _sync_case(ctx, w, mb, G, slot_bytes, seed):
    ids = inputs.topk_ids(w, mb)
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    plan = ue.Plan(cfg)
    d_ids = torch.from_numpy(ids).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    ue.ue_rebalance(ctx, cfg, d_ids, counts, None, plan, torch.empty_like(d_ids))
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = torch.randint(0, 256, (cfg.S, slot_bytes), dtype=torch.uint8, device="cuda", generator=g)
    SG = cfg.S // G
    bases = [W[h * SG] for h in range(G)]
    return cfg, plan, W, bases


@pytest.mark.parametrize("w,mb,G", [(inputs.TINY, 0, 2), (inputs.TINY, 1, 8), (inputs.CLASS_671B, 2, 8),
                                    (inputs.CLASS_671B, 5, 64), (inputs.EXTREME, 1, 16), (inputs.EXTREME, 2, 128),
                                    (inputs.CLASS_106B, 4, 4)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_sync_relay_rounds(ctx, w, mb, G):
    slot_bytes = 2 * 48 * 1024 + 4096 + 16       # two full tiles and a ragged one
    cfg, plan, W, bases = _sync_case(ctx, w, mb, G, slot_bytes, seed=mb + 7)
    pl = plan.to_host()
    host = W.cpu().numpy()
    full = host.copy()
    oracle.sync(full, slot_bytes, w.E, w.N, w.R, pl["slot_expert"])
    rounds = ue.ue_relay_rounds(G)
    assert rounds == oracle.relay_rounds(G)
    for k in range(rounds):
        for g in reversed(range(G)):
            ue.ue_sync_shard(ctx, cfg, G, g, bases, slot_bytes, plan, k)
        torch.cuda.synchronize()
        assert ctx.device_error() == 0
        oracle.sync_relay(host, slot_bytes, w.E, w.N, w.R, pl["slot_expert"], G, k)
        assert np.array_equal(W.cpu().numpy(), host), k
    assert np.array_equal(host, full)


@pytest.mark.parametrize("w,G", [(inputs.TINY, 4), (inputs.CLASS_671B, 16), (inputs.EXTREME, 64)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_sync_direct_form(ctx, w, G):
    slot_bytes = 48 * 1024 + 32
    cfg, plan, W, bases = _sync_case(ctx, w, 6, G, slot_bytes, seed=2)
    pl = plan.to_host()
    host = W.cpu().numpy()
    for g in range(G):
        ue.ue_sync_shard(ctx, cfg, G, g, bases, slot_bytes, plan, -1)
    torch.cuda.synchronize()
    oracle.sync(host, slot_bytes, w.E, w.N, w.R, pl["slot_expert"])
    assert np.array_equal(W.cpu().numpy(), host)


def test_sync_shard_one_gpu_equals_sync(ctx):
    w = inputs.CLASS_106B
    slot_bytes = 3 * 48 * 1024 - 48
    cfg, plan, W, bases = _sync_case(ctx, w, 9, 1, slot_bytes, seed=4)
    W2 = W.clone()
    ue.ue_sync_shard(ctx, cfg, 1, 0, [W], slot_bytes, plan, 0)
    ue.ue_sync(ctx, cfg, W2, slot_bytes, plan)
    torch.cuda.synchronize()
    assert torch.equal(W, W2)


@pytest.mark.parametrize("w,G,dtype", [(inputs.TINY, 2, torch.float32), (inputs.TINY, 8, torch.bfloat16),
                                       (inputs.CLASS_671B, 8, torch.bfloat16), (inputs.EXTREME, 32, torch.float32),
                                       (inputs.CLASS_106B, 4, torch.float32)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_grad_reduce_shards(ctx, w, G, dtype):
    P = 3 * 1024 + 8 * 5                         # a ragged last chunk
    ids = inputs.topk_ids(w, 4)
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    plan = ue.Plan(cfg)
    d_ids = torch.from_numpy(ids).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    ue.ue_rebalance(ctx, cfg, d_ids, counts, None, plan, torch.empty_like(d_ids))
    gen = torch.Generator(device="cuda").manual_seed(11)
    master = torch.randn((w.E, P), device="cuda", generator=gen) * 1e-2
    grads = (torch.randn((w.N * w.R, P), device="cuda", generator=gen) * 1e-3).to(dtype)
    m_host = master.cpu().numpy().copy()
    g_host = grads.cpu().view(torch.int16).numpy().view(np.uint16) if dtype == torch.bfloat16 \
        else grads.cpu().numpy()
    EG, RG = w.E // G, (w.N // G) * w.R
    bases = [grads[h * RG] for h in range(G)]
    for g in range(G):
        ue.ue_grad_reduce_shard(ctx, cfg, G, g, master[g * EG:(g + 1) * EG], bases, dtype, P, plan)
    torch.cuda.synchronize()
    oracle.grad_reduce(m_host, np.ascontiguousarray(g_host), P, w.E, w.N, w.R, plan.to_host())
    got = master.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), m_host.view(np.uint32))


def test_shards_empty_microbatch_and_no_redundant_slots(ctx):
    # T = 0: the counts rows are written (zeros) and nothing else is touched
    E, N, R, K = 32, 8, 2, 4
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=0)
    counts = torch.full((N, E), -7, dtype=torch.int32, device="cuda")
    bad = torch.full((N,), -7, dtype=torch.int32, device="cuda")
    empty = torch.empty((0, K), dtype=torch.int32, device="cuda")
    for g in range(4):
        ue.ue_load_shard(ctx, cfg, 4, g, empty, counts, bad)
    plan = ue.Plan(cfg)
    ue.ue_plan(ctx, cfg, counts, plan)
    for g in range(4):
        ue.ue_reroute_shard(ctx, cfg, 4, g, empty, plan, empty)
    torch.cuda.synchronize()
    assert (counts == 0).all().item() and (bad == 0).all().item()
    # R = 0: no replica anywhere, the sync and the gradient reduction change nothing
    ids = np.random.default_rng(8).integers(0, 64, size=(8 * 64, 4)).astype(np.int32)
    cfg0, counts0, _, plan0, phys0 = _rebalance_sharded(ctx, ids, 64, 8, 0, 4)
    ref = oracle.rebalance(ids, 64, 8, 0)
    assert np.array_equal(phys0, ref["phys"])
    W = torch.randint(0, 256, (cfg0.S, 4096), dtype=torch.uint8, device="cuda")
    W0 = W.clone()
    bases = [W[h * (cfg0.S // 4)] for h in range(4)]
    for k in range(ue.ue_relay_rounds(4)):
        for g in range(4):
            ue.ue_sync_shard(ctx, cfg0, 4, g, bases, 4096, plan0, k)
    master = torch.randn((64, 64), device="cuda")
    m0 = master.clone()
    for g in range(4):
        ue.ue_grad_reduce_shard(ctx, cfg0, 4, g, master[g * 16:(g + 1) * 16], None, torch.float32, 64, plan0)
    torch.cuda.synchronize()
    assert torch.equal(W, W0) and torch.equal(master, m0)


def test_sharded_balancer_on_one_gpu(ctx):
    """The host sequence (ShardedBalancer with the device calls) for G = 1:
    rebalance, relay sync and gradient reduction equal the oracle."""
    from moe_expert_load_ue_b200.shard import DeviceOps, ShardedBalancer
    w = inputs.CLASS_106B
    ids = inputs.topk_ids(w, 2)
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    bal = ShardedBalancer(cfg, DeviceOps(ctx, cfg, 1, 0), G=1, g=0)
    d_ids = torch.from_numpy(ids).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    bad = torch.empty(w.N, dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.empty_like(d_ids)
    bal.rebalance(d_ids, counts, bad, plan, phys)
    slot_bytes = 48 * 1024 + 64
    W = torch.randint(0, 256, (cfg.S, slot_bytes), dtype=torch.uint8, device="cuda")
    host = W.cpu().numpy()
    bal.sync([W], slot_bytes, plan)
    P = 2048 + 16
    master = torch.randn((w.E, P), device="cuda") * 1e-2
    grads = torch.randn((w.N * w.R, P), device="cuda") * 1e-3
    m_host = master.cpu().numpy().copy()
    bal.grad_reduce(master, [grads], torch.float32, P, plan)
    torch.cuda.synchronize()
    ref = oracle.rebalance(ids, w.E, w.N, w.R)
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert np.array_equal(phys.cpu().numpy(), ref["phys"])
    oracle.sync(host, slot_bytes, w.E, w.N, w.R, ref["plan"]["slot_expert"])
    assert np.array_equal(W.cpu().numpy(), host)
    oracle.grad_reduce(m_host, grads.cpu().numpy(), P, w.E, w.N, w.R, ref["plan"])
    assert np.array_equal(master.cpu().numpy().view(np.uint32), m_host.view(np.uint32))
