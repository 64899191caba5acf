"""GPU parity at the workloads' full sizes, compared byte for byte.

Weight sync: every filled redundant slot equals its expert's home slot in full,
windows of every slot equal the oracle's sync, and every other slot (home
slots, empty redundant slots) is unchanged in full.

Gradient reduction: the whole master row of every replicated expert equals the
oracle's reduction (bit for bit, and within the 1e-5 contract), and every other
master row is unchanged in full.  The rows are compared in column chunks, so
the host holds one chunk of every row at a time.

Rebalance at the sweep's largest corner (256 ranks x 32,768 tokens per rank,
33.5 M assignments): every output array against the oracle.
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


def _free_gb():
    free, _ = torch.cuda.mem_get_info()
    return free / 2**30


def _rebalance(ctx, w, ids):
    cfg = ue.Config(E=w.E, N=w.N, R=w.R, K=w.K, T=w.T)
    ids_d = ids if isinstance(ids, torch.Tensor) else torch.from_numpy(ids).cuda()
    counts = torch.empty((w.N, w.E), dtype=torch.int32, device="cuda")
    bad = torch.empty(w.N, dtype=torch.int32, device="cuda")
    plan = ue.Plan(cfg)
    phys = torch.full_like(ids_d, -5)
    ue.ue_rebalance(ctx, cfg, ids_d, counts, bad, plan, phys)
    torch.cuda.synchronize()
    return cfg, plan, counts, bad, phys


def _home(e, w):
    return (e // w.H) * (w.H + w.R) + e % w.H


# ---- weight sync, whole slots ---------------------------------------------------

@pytest.mark.parametrize("w,mb", [(inputs.CLASS_671B, 0), (inputs.CLASS_106B, 5), (inputs.EXTREME, 3)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_sync_full_size_whole_slots(ctx, w, mb):
    slot_bytes = 2 * w.P
    if _free_gb() < 2 * w.S * slot_bytes / 2**30 + 4:
        pytest.skip("not enough device memory")
    cfg, plan, *_ = _rebalance(ctx, w, inputs.topk_ids(w, mb))
    pl = plan.to_host()
    W = torch.empty((w.S, slot_bytes), dtype=torch.uint8, device="cuda")
    W.view(torch.int32).random_(generator=torch.Generator(device="cuda").manual_seed(5 + mb))
    W0 = W.clone()
    width = 1 << 18
    rng = np.random.default_rng(mb)
    starts = sorted({0, slot_bytes - width} | {int(rng.integers(0, slot_bytes - width)) // 16 * 16
                                               for _ in range(2)})
    win = lambda X: np.concatenate([X[:, a:a + width].cpu().numpy() for a in starts], axis=1)
    expect = win(W0)
    ue.ue_sync(ctx, cfg, W, slot_bytes, plan)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    oracle.sync(expect, expect.shape[1], w.E, w.N, w.R, pl["slot_expert"])
    assert np.array_equal(win(W), expect)
    HR = w.H + w.R
    filled = 0
    for s in range(w.S):
        e = int(pl["slot_expert"][s])
        if s % HR >= w.H and e >= 0:
            assert torch.equal(W[s], W0[_home(e, w)]), f"slot {s} (expert {e}) differs from its home"
            filled += 1
        else:
            assert torch.equal(W[s], W0[s]), f"slot {s} must be untouched"
    assert filled == int(pl["info"][4]) > 0
    del W, W0
    torch.cuda.empty_cache()


# ---- gradient reduction, whole rows ------------------------------------------------

def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.cpu().numpy()


@pytest.mark.parametrize("w,mb", [(inputs.CLASS_671B, 0), (inputs.CLASS_106B, 7)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_grad_reduce_full_size_whole_rows(ctx, w, mb):
    P = w.P
    gdt = torch.bfloat16 if w.grad_dtype == "bf16" else torch.float32
    gsize = 2 if gdt == torch.bfloat16 else 4
    if _free_gb() < (2 * w.E * P * 4 + w.N * w.R * P * gsize) / 2**30 + 4:
        pytest.skip("not enough device memory")
    cfg, plan, *_ = _rebalance(ctx, w, inputs.topk_ids(w, mb))
    pl = plan.to_host()
    gen = torch.Generator(device="cuda").manual_seed(31 + mb)
    master = torch.empty((w.E, P), device="cuda")
    for e in range(w.E):
        master[e].normal_(0.0, 1e-3, generator=gen)
    grads = torch.empty((w.N * w.R, P), dtype=gdt, device="cuda")
    for r in range(w.N * w.R):
        grads[r].normal_(0.0, 1e-3, generator=gen)
    m0 = master.clone()
    ue.ue_grad_reduce(ctx, cfg, master, grads, P, plan)
    torch.cuda.synchronize()

    off = pl["rep_off"]
    rep = [e for e in range(w.E) if off[e + 1] - off[e] > 1]
    assert len(rep) == int(pl["info"][3]) > 0
    for e in sorted(set(range(w.E)) - set(rep)):
        assert torch.equal(master[e], m0[e]), f"master row {e} (no replica) must be untouched"

    rep_t = torch.tensor(rep, device="cuda")
    width = 1 << 20
    mh = np.zeros((w.E, width), np.float32)       # oracle input: the replicated rows of one column chunk
    for a in range(0, P, width):
        b = min(P, a + width)
        n = b - a
        before = m0[rep_t, a:b].cpu().numpy()
        gh = np.ascontiguousarray(_bits(grads[:, a:b]))
        mh[rep, :n] = before
        oracle.grad_reduce(mh, gh, n, w.E, w.N, w.R, pl)
        expect = mh[rep, :n]
        got = master[rep_t, a:b].cpu().numpy()
        if not np.array_equal(got, expect):
            # report the 1e-5 contract and the first differing element
            H, HR = w.H, w.H + w.R
            g = (gh.astype(np.uint32) << 16).view(np.float32) if gsize == 2 else gh
            abs_sum = np.zeros_like(before, dtype=np.float64)
            for i, e in enumerate(rep):
                for p in range(off[e] + 1, off[e + 1]):
                    s = pl["rep_slot"][p]
                    abs_sum[i] += np.abs(g[(s // HR) * w.R + (s % HR - H)])
            bound = GRAD_RTOL * (np.abs(before).astype(np.float64) + abs_sum) + 1e-30
            within = np.all(np.abs(got.astype(np.float64) - expect.astype(np.float64)) <= bound)
            idx = np.argwhere(got != expect)[0]
            pytest.fail(f"columns [{a}, {b}): expert {rep[idx[0]]} element {a + idx[1]}: "
                        f"{got[tuple(idx)]!r} != {expect[tuple(idx)]!r}; within 1e-5 contract: {within}")
    del master, grads, m0
    torch.cuda.empty_cache()


# ---- rebalance at the sweep's largest corner -----------------------------------------

@pytest.mark.parametrize("s", [0.0, 1.6])
def test_rebalance_sweep_corner_256_ranks_32768_tokens(ctx, s):
    w = inputs.Workload(f"sweep-corner-s{s}", E=256, K=8, N=256, R=1, tokens_per_rank=32768, s=s,
                        rows=2048, cols=1024, base_seed=4)
    ids_d = inputs.topk_ids_device(w, 0, "cuda")
    torch.cuda.synchronize()
    ids = ids_d.cpu().numpy()
    cfg, plan, counts, bad, phys = _rebalance(ctx, w, ids_d)
    ref = oracle.rebalance(ids, w.E, w.N, w.R)
    assert np.array_equal(counts.cpu().numpy(), ref["counts"]), "counts"
    assert np.array_equal(bad.cpu().numpy(), ref["bad"]), "bad"
    pl = plan.to_host()
    for f in oracle.PLAN_FIELDS:
        assert np.array_equal(pl[f], ref["plan"][f]), f
    assert np.array_equal(pl["load"], ref["load"]), "load"
    assert np.array_equal(pl["rank_off"], ref["rank_off"]), "rank_off"
    assert np.array_equal(phys.cpu().numpy(), ref["phys"]), "phys"
