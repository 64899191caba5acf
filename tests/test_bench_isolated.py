"""bench.run_isolated: the across-GPU leg of a multi-GPU bench runs on a gloo
group of its own, so a failure on some ranks ends on every rank within the
group's timeout and the job's main group stays usable (two gloo ranks on CPU)."""
import datetime
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import time

    import torch
    import torch.distributed as dist

    import bench
    try:
        dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
        d = bench.Dist()
        d.world, d.rank, d.pg = 2, rank, dist

        def ok(grp):
            dist.barrier(group=grp)
            t = torch.tensor([float(rank)])
            dist.all_reduce(t, group=grp)
            return {"sum": t.item()}

        def one_rank_fails(grp):
            if rank == 1:
                raise RuntimeError("planted failure on rank 1")
            dist.barrier(group=grp)          # rank 1 never arrives: runs out after the group's timeout
            return {"unexpected": True}

        r1 = bench.run_isolated(d, ok, timeout_s=5)
        t0 = time.time()
        r2 = bench.run_isolated(d, one_rank_fails, timeout_s=3)
        waited = time.time() - t0
        # the main group still works, in the same order on both ranks
        t = torch.tensor([1.0 + rank])
        dist.all_reduce(t)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, r1, r2, waited, t.item()))
    except Exception as exc:
        q.put((rank, "worker failed", repr(exc), 0.0, 0.0))
        raise


def test_a_failure_on_one_rank_stays_inside_the_isolated_group():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    outs = sorted([q.get(timeout=120) for _ in procs], key=lambda o: o[0])
    for p in procs:
        p.join(timeout=60)
    for rank, r1, r2, waited, total in outs:
        assert r1 == {"sum": 1.0}, (rank, r1, r2)
        assert "error" in r2, (rank, r2)
        assert total == 3.0
        assert waited < 30
    assert "planted failure" in outs[1][2]["error"]
    assert all(p.exitcode == 0 for p in procs)
