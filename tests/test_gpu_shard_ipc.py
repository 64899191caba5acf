"""The calls across GPUs with real interprocess peer tables (CUDA IPC).

Two processes, one per simulated GPU, both on the one GPU of the test box,
each holding only its own shard: its ranks' tokens, its slots, its home
experts' master rows and its replica-gradient rows.  Each process maps the
other's slots and replica-gradient rows through CUDA IPC handles exchanged over
a gloo group (moe_expert_load_ue_b200.peer.PeerBuffers), and ShardedBalancer
issues load, the all-gather of the counts, plan and reroute, the weight sync
(relay rounds, then the direct form on fresh slots) and the home-GPU gradient
reduction, with host barriers after a stream synchronize.  No kernel waits on
another process's kernels.  The shards put together must equal the single-GPU
oracle bit for bit.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
E, N, R, K, T = 32, 8, 2, 4, 8 * 512
NB = 3 * 48 * 1024 + 16          # slot bytes: several bulk tiles and a ragged one
P = 4096 + 8                     # gradient elements per expert
G = 2


def _inputs():
    rng = np.random.default_rng(23)
    p = (rng.permutation(E) + 1.0) ** -1.5
    ids = np.stack([rng.choice(E, size=K, replace=False, p=p / p.sum()) for _ in range(T)]).astype(np.int32)
    S = N * (E // N + R)
    W0 = rng.integers(0, 256, size=(S, NB), dtype=np.uint8)
    m0 = rng.standard_normal((E, P)).astype(np.float32)
    g0 = (rng.standard_normal((N * R, P)) * 1e-3).astype(np.float32)
    return ids, W0, m0, g0


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from moe_expert_load_ue_b200 import ue
    from moe_expert_load_ue_b200.peer import PeerBuffers
    from moe_expert_load_ue_b200.shard import DeviceOps, ShardedBalancer
    try:
        dist.init_process_group("gloo", rank=rank, world_size=G, timeout=datetime.timedelta(seconds=60))
        torch.cuda.set_device(0)
        ids, W0, m0, g0 = _inputs()
        S = W0.shape[0]
        NG, SG, EG, TG = N // G, S // G, E // G, T // G
        RG = NG * R
        cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
        ctx = ue.Context(0)
        ids_l = torch.from_numpy(ids[rank * TG:(rank + 1) * TG]).cuda()
        counts = torch.full((N, E), -1, dtype=torch.int32, device="cuda")
        bad = torch.full((N,), -1, dtype=torch.int32, device="cuda")
        plan = ue.Plan(cfg)
        phys_l = torch.empty_like(ids_l)
        W_init = torch.from_numpy(W0[rank * SG:(rank + 1) * SG]).cuda()
        W_l = W_init.clone()
        master_l = torch.from_numpy(m0[rank * EG:(rank + 1) * EG]).cuda()
        grads_l = torch.from_numpy(g0[rank * RG:(rank + 1) * RG]).cuda()
        bal = ShardedBalancer(cfg, DeviceOps(ctx, cfg, G, rank), G=G, g=rank, device="cuda", host_staged=True)

        bal.rebalance(ids_l, counts, bad, plan, phys_l)
        pw = PeerBuffers(W_l)
        pg = PeerBuffers(grads_l)
        bal.sync(pw.ptrs, NB, plan, relay=True)
        W_relay = W_l.cpu().numpy()
        W_l.copy_(W_init)
        bal.barrier()                   # every process's slots are back to their first state
        bal.sync(pw.ptrs, NB, plan, relay=False)
        W_direct = W_l.cpu().numpy()
        bal.grad_reduce(master_l, pg.ptrs, torch.float32, P, plan)
        torch.cuda.synchronize()
        out = (rank, counts.cpu().numpy(), bad.cpu().numpy(), plan["slot_expert"].cpu().numpy(),
               phys_l.cpu().numpy(), W_relay, W_direct, master_l.cpu().numpy(), ctx.device_error())
        bal.barrier()                   # no process reads the other's buffers any more
        pw.close()
        pg.close()
        ctx.close()
        dist.destroy_process_group()
        q.put(out)
    except Exception as exc:            # report instead of hanging the parent
        q.put((rank, repr(exc)))
        raise


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_calls_over_cuda_ipc_match_the_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(G)]
    for p in procs:
        p.start()
    outs = sorted([q.get(timeout=300) for _ in procs], key=lambda o: o[0])
    for p in procs:
        p.join(timeout=120)
    for o in outs:
        assert len(o) > 2, f"rank {o[0]} failed: {o[1]}"
    for p in procs:
        assert p.exitcode == 0

    ids, W0, m0, g0 = _inputs()
    ref = oracle.rebalance(ids, E, N, R)
    for _, counts, bad, se, *_ in outs:
        assert np.array_equal(counts, ref["counts"]) and np.array_equal(bad, ref["bad"])
        assert np.array_equal(se, ref["plan"]["slot_expert"])
    assert np.array_equal(np.concatenate([o[4] for o in outs]), ref["phys"])
    Wref = W0.copy()
    oracle.sync(Wref, NB, E, N, R, ref["plan"]["slot_expert"])
    assert np.array_equal(np.concatenate([o[5] for o in outs]), Wref), "relay rounds"
    assert np.array_equal(np.concatenate([o[6] for o in outs]), Wref), "direct form"
    mref = m0.copy()
    oracle.grad_reduce(mref, g0, P, E, N, R, ref["plan"])
    assert np.array_equal(np.concatenate([o[7] for o in outs]), mref)
    assert all(o[8] == 0 for o in outs)
