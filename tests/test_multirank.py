"""Host logic of the multi-GPU bench on CPU: N independent replicas, joined only
by a barrier and the max over ranks of their timings (gloo, world size 2)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist().init("gloo")
    d.barrier()
    mx = d.max([10.0 * (rank + 1), -rank])
    sm = d.sum([1.0, rank])
    d.barrier()
    d.close()
    q.put((rank, mx, sm))


def test_max_and_sum_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm in out:
        assert mx == [20.0, 0.0]          # element-wise max over ranks
        assert sm == [2.0, 1.0]


def test_single_rank_dist_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    if d.world == 1:
        assert d.max([3.0, 1.0]) == [3.0, 1.0]
        d.barrier()


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "1", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    if rank == 0:
        rec = json.loads(lines[-1])
        assert rec["impl"] == "reference" and rec["n_gpus"] == 2
        assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0
        assert rec["value"] > 0 and rec["unit"] == "µs" and rec["higher_is_better"] is False
    else:
        assert lines == []
