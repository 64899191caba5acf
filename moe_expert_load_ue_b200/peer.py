"""Peer tables for the calls across GPUs: one buffer per process, mapped into every process.

The sharded weight sync and gradient reduction (include/ue.h, "across the GPUs
of one NVLink domain") read other GPUs' slots and replica-gradient rows through
a table of G device pointers, entry h being GPU h's buffer as mapped in the
calling process.  PeerBuffers builds that table with interprocess buffers (the
runtime's CUDA IPC buffers, csrc/utils/ipc_manager.cu in "How
dots-infra/ultraep works"): every process exports its buffer as a CUDA IPC
memory handle, the handles travel over the process group, and every process
opens the others' (with peer access enabled lazily when the buffers live on
other GPUs).  Only the library's own kernels read through the table, with plain
bulk or vector loads.

This module is plumbing (device-memory mapping with torch's IPC machinery); it
holds none of the balancer's arithmetic.
"""
from __future__ import annotations

import torch
import torch.distributed as dist
from torch.multiprocessing.reductions import reduce_tensor


class PeerBuffers:
    """`local` (a CUDA tensor of this process) as seen by every process of the
    group: `ptrs[h]` is process h's buffer mapped here (h = this rank: the local
    buffer itself).  Every process calls it collectively with its own buffer.
    Keep the object (and `local`) alive while kernels read through the table;
    call close() on every process, after a barrier, when done."""

    def __init__(self, local: torch.Tensor, group=None):
        if not local.is_cuda:
            raise ValueError("PeerBuffers maps CUDA tensors")
        self.G = dist.get_world_size(group)
        self.g = dist.get_rank(group)
        # The exported handle must see the buffer's pending writes complete.
        torch.cuda.current_stream(local.device).synchronize()
        rebuild, args = reduce_tensor(local)
        handles: list = [None] * self.G
        dist.all_gather_object(handles, (rebuild, args), group=group)
        self.tensors = [local if h == self.g else fn(*a) for h, (fn, a) in enumerate(handles)]
        self.ptrs = [t.data_ptr() for t in self.tensors]

    def close(self) -> None:
        self.tensors = []
        self.ptrs = []
