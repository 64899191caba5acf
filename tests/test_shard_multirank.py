"""Host logic of the balancer across GPUs on CPU (gloo, world sizes 2 and 4).

`ShardedBalancer` issues the exchanges between GPUs around the sharded calls:
the all-gather of the counts rows before planning and the barriers that order
the relay rounds of the weight sync and fence the gradient reduction.  Here
each rank is a CPU process whose device steps are stand-ins built on the
oracle (test code), acting on buffers in shared memory the way the sharded
kernels act on peer memory: each rank writes only its own rows and slots.
Checked: every rank ends with the full counts and the same plan; the ranks'
phys slices, slots and master rows together equal the single-GPU oracle; and
no rank starts relay round k (or the gradient reduction) before every rank
has finished round k - 1 (the sync), which a missing barrier would break
because rank 0 is slowed down on purpose.  Before the sync every rank writes
new weights into its own home slots (an optimizer step), rank 0 late: the
replicas must hold the new weights, which a missing barrier before the first
round would break (a consumer would pull rank 0's old bytes).
"""
import os
import socket
import sys
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

E, N, R, K, T, NB, P = 32, 8, 2, 4, 8 * 96, 64, 40


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(17)
    p = (rng.permutation(E) + 1.0) ** -1.6
    ids = np.stack([rng.choice(E, size=K, replace=False, p=p / p.sum()) for _ in range(T)]).astype(np.int32)
    W = rng.integers(0, 256, size=(N * (E // N + R), NB), dtype=np.uint8)
    master = (rng.integers(-64, 64, size=(E, P)) / 256.0).astype(np.float32)
    grads = (rng.integers(-64, 64, size=(N * R, P)) / 1024.0).astype(np.float32)
    W_new = rng.integers(0, 256, size=W.shape, dtype=np.uint8)     # home slots after an optimizer step
    return ids, W, master, grads, W_new


class OracleOps:
    """Stand-ins for the sharded device calls of GPU g (test code)."""

    def __init__(self, g, G, ids_full, W, master, grads, log, t0):
        import oracle
        self.o, self.g, self.G = oracle, g, G
        self.ids_full, self.W, self.master, self.grads, self.log, self.t0 = ids_full, W, master, grads, log, t0
        self.NG = N // G

    def _stamp(self, k, i):
        self.log[self.g, k, i] = time.monotonic_ns() - self.t0

    def write_home(self, W_new):
        """This GPU's home slots get new weights (rank 0 late), log row 6."""
        self._stamp(6, 0)
        if self.g == 0:
            time.sleep(0.3)
        HR, SG = E // N + R, (N * (E // N + R)) // self.G
        for s in range(self.g * SG, (self.g + 1) * SG):
            if s % HR < E // N:
                self.W[s] = W_new[s]
        self._stamp(6, 1)

    def load(self, ids_local, counts, bad):
        c, b = self.o.load(ids_local.numpy(), E, self.NG)
        lo = self.g * self.NG
        counts[lo:lo + self.NG] = torch.from_numpy(c)
        bad[lo:lo + self.NG] = torch.from_numpy(b)

    def plan(self, counts, plan):
        ld, off = self.o.expert_load(counts.numpy())
        plan.update(self.o.plan(ld, N, R))

    def reroute(self, ids_local, plan, phys_local):
        n = T // self.G
        phys_local[:] = torch.from_numpy(self.o.reroute(self.ids_full.numpy(), E, plan)[self.g * n:(self.g + 1) * n])

    def sync(self, slot_bases, slot_bytes, plan, round):
        self._stamp(round + 1, 0)              # log row 0: the direct form, 1 + k: relay round k
        if self.g == 0:
            time.sleep(0.3)                    # a missing barrier would let the others run ahead
        self.o.sync_relay(self.W.numpy(), slot_bytes, E, N, R, plan["slot_expert"], self.G, round, self.g)
        self._stamp(round + 1, 1)

    def grad_reduce(self, master_local, grad_bases, grads_dtype, P_, plan):
        self._stamp(7, 0)
        full = self.master.numpy().copy()
        self.o.grad_reduce(full, self.grads.numpy(), P_, E, N, R, plan)
        EG = E // self.G
        master_local[:] = torch.from_numpy(full[self.g * EG:(self.g + 1) * EG])
        self._stamp(7, 1)


def _worker(rank, world, relay, port, ids_full, W, master, grads, W_new, log, t0, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    from moe_expert_load_ue_b200.shard import ShardedBalancer
    from moe_expert_load_ue_b200 import ue
    dist.init_process_group("gloo", rank=rank, world_size=world)
    cfg = ue.Config(E=E, N=N, R=R, K=K, T=T)
    ops = OracleOps(rank, world, ids_full, W, master, grads, log, t0)
    bal = ShardedBalancer(cfg, ops, device="cpu")
    n = T // world
    ids_local = ids_full[rank * n:(rank + 1) * n].clone()
    counts = torch.full((N, E), -1, dtype=torch.int32)
    bad = torch.full((N,), -1, dtype=torch.int32)
    plan, phys = {}, torch.empty_like(ids_local)
    bal.rebalance(ids_local, counts, bad, plan, phys)
    ops.write_home(W_new)
    bal.sync(None, NB, plan, relay=relay)
    EG = E // world
    bal.grad_reduce(master[rank * EG:(rank + 1) * EG], None, torch.float32, P, plan)
    dist.destroy_process_group()
    q.put((rank, counts.numpy(), bad.numpy(), plan["slot_expert"], phys.numpy(), bal.relay_rounds))


@pytest.mark.parametrize("world,relay", [(2, True), (4, True), (4, False)])
def test_sharded_balancer_on_gloo_ranks(world, relay):
    sys.path.insert(0, ROOT)
    import oracle
    ids, W0, m0, g0, Wn = _inputs()
    ids_t = torch.from_numpy(ids).share_memory_()
    W_new = torch.from_numpy(Wn).share_memory_()
    W = torch.from_numpy(W0.copy()).share_memory_()
    master = torch.from_numpy(m0.copy()).share_memory_()
    grads = torch.from_numpy(g0).share_memory_()
    log = torch.zeros((world, 8, 2), dtype=torch.int64).share_memory_()
    t0 = time.monotonic_ns()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, relay, port, ids_t, W, master, grads, W_new, log, t0, q))
             for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=180) for _ in procs], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    ref = oracle.rebalance(ids, E, N, R)
    rounds = out[0][5]
    assert rounds == oracle.relay_rounds(world)
    for rank, counts, bad, se, phys, _ in out:
        assert np.array_equal(counts, ref["counts"]) and np.array_equal(bad, ref["bad"])
        assert np.array_equal(se, ref["plan"]["slot_expert"])
    assert np.array_equal(np.concatenate([o[4] for o in out]), ref["phys"])
    Wref = W0.copy()
    home = (np.arange(Wref.shape[0]) % (E // N + R)) < E // N
    Wref[home] = Wn[home]
    oracle.sync(Wref, NB, E, N, R, ref["plan"]["slot_expert"])
    assert np.array_equal(W.numpy(), Wref)
    mref = m0.copy()
    oracle.grad_reduce(mref, g0, P, E, N, R, ref["plan"])
    assert np.array_equal(master.numpy(), mref)
    lg = log.numpy()
    rows = list(range(1, rounds + 1)) if relay else [0]
    assert lg[:, rows[0], 0].min() >= lg[:, 6, 1].max(), "a sync round started before every home slot was written"
    for a, b in zip(rows, rows[1:]):
        assert lg[:, b, 0].min() >= lg[:, a, 1].max(), f"log row {b} started before row {a} ended"
    assert lg[:, 7, 0].min() >= lg[:, rows[-1], 1].max()   # gradient reduction after the last sync round
