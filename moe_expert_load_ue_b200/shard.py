"""The balancer across the GPUs of one NVLink domain: the order of the calls.

The N expert-parallel ranks are spread over G GPUs, one process per GPU
(torch.distributed); GPU g holds ranks [g*N/G, (g+1)*N/G) with their tokens,
slots, home experts and replica-gradient rows (include/ue.h, "across the GPUs
of one NVLink domain").  The path has two kinds of exchange between GPUs, and
this module issues them in order around the library's sharded calls:

- after the per-rank histograms (load computation), an all-gather of the
  counts rows, so that every GPU plans from the same [N][E] counts and
  computes the same plan (placement planning is deterministic) with its
  per-rank offsets for routing expansion;
- barriers across GPUs that order the relay rounds of the replica weight sync
  (no GPU pulls a home slot before its GPU has finished writing it, and a GPU
  pulls in the all-gather round only parts the scatter round brought to the
  other GPUs) and fence the
  replica gradient reduction (every replica gradient written before the home
  GPUs read them; all reads done before the buffers are reused).

The device steps go through `ops` (`DeviceOps`: the C ABI on this GPU); the
exchanges through the process group.  With the NCCL backend a barrier is an
all-reduce of one element on the current stream, so the kernels after it on
that stream start only once every GPU has reached it.  With a host-side group
(gloo; `host_staged=True`) each barrier first waits for this process's stream,
then meets the others on the host, and the counts rows travel through host
memory.  The peer tables of the sync and gradient calls come from
`peer.PeerBuffers` (CUDA IPC).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ue


class DeviceOps:
    """The sharded C-ABI calls for GPU g of G."""

    def __init__(self, ctx: ue.Context, cfg: ue.Config, G: int, g: int, variant: int = 0):
        self.ctx, self.cfg, self.G, self.g, self.variant = ctx, cfg, G, g, variant

    def load(self, ids_local, counts, bad):
        ue.ue_load_shard(self.ctx, self.cfg, self.G, self.g, ids_local, counts, bad)

    def plan(self, counts, plan):
        ue.ue_plan_ex(self.ctx, self.cfg, counts, plan, self.variant)

    def reroute(self, ids_local, plan, phys_local):
        ue.ue_reroute_shard(self.ctx, self.cfg, self.G, self.g, ids_local, plan, phys_local)

    def sync(self, slot_bases, slot_bytes, plan, round):
        ue.ue_sync_shard(self.ctx, self.cfg, self.G, self.g, slot_bases, slot_bytes, plan, round)

    def grad_reduce(self, master_local, grad_bases, grads_dtype, P, plan):
        ue.ue_grad_reduce_shard(self.ctx, self.cfg, self.G, self.g, master_local, grad_bases, grads_dtype, P, plan)


class ShardedBalancer:
    """Per-microbatch sequence of one GPU (g of G = the process group's size
    and rank unless given)."""

    def __init__(self, cfg: ue.Config, ops, G: int | None = None, g: int | None = None, group=None,
                 device: str | torch.device = "cuda", host_staged: bool = False):
        self.cfg, self.ops, self.group, self.host_staged = cfg, ops, group, host_staged
        self.G = G if G is not None else (dist.get_world_size(group) if dist.is_initialized() else 1)
        self.g = g if g is not None else (dist.get_rank(group) if dist.is_initialized() else 0)
        if cfg.N % self.G != 0:
            raise ValueError(f"N={cfg.N} is not a multiple of G={self.G}")
        self.NG = cfg.N // self.G
        self._token = torch.zeros(1, dtype=torch.int32, device=device)

    @property
    def relay_rounds(self) -> int:
        return ue.ue_relay_rounds(self.G)

    def barrier(self) -> None:
        if self.G > 1:
            if self.host_staged:
                if self._token.is_cuda:
                    torch.cuda.current_stream(self._token.device).synchronize()
                dist.barrier(group=self.group)
            else:
                dist.all_reduce(self._token, group=self.group)

    def rebalance(self, ids_local, counts, bad, plan, phys_local) -> None:
        """Load computation for this GPU's ranks, all-gather of the counts
        rows (and bad-id rows), placement planning on the full counts, routing
        expansion of this GPU's tokens."""
        self.ops.load(ids_local, counts, bad)
        if self.G > 1:
            lo, hi = self.g * self.NG, (self.g + 1) * self.NG
            for t in (counts, bad):
                if t is None:
                    continue
                if self.host_staged:
                    full = torch.empty(t.shape, dtype=t.dtype)
                    dist.all_gather_into_tensor(full, t[lo:hi].cpu(), group=self.group)
                    t.copy_(full)
                else:
                    dist.all_gather_into_tensor(t, t[lo:hi].clone(), group=self.group)
        self.ops.plan(counts, plan)
        self.ops.reroute(ids_local, plan, phys_local)

    def sync(self, slot_bases, slot_bytes: int, plan, relay: bool = True) -> None:
        """Replica weight sync: the relay rounds (or the direct form), with a
        barrier before every round and after the last.  The first barrier
        makes every GPU's home slots final (an optimizer step or any earlier
        write on another GPU's stream) before any GPU pulls from them."""
        rounds = range(self.relay_rounds) if relay else (-1,)
        for k in rounds:
            self.barrier()
            self.ops.sync(slot_bases, slot_bytes, plan, k)
        self.barrier()

    def grad_reduce(self, master_local, grad_bases, grads_dtype, P: int, plan) -> None:
        """Replica gradient reduction on the home GPUs, fenced by barriers."""
        self.barrier()
        self.ops.grad_reduce(master_local, grad_bases, grads_dtype, P, plan)
        self.barrier()
