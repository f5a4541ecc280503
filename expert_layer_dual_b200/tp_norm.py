"""Tensor-parallel all-reduce + residual + RMSNorm across the ranks of a
process group (one process per GPU), low-latency Lamport P2P form.

"HPC-Ops - 騰訊混元開源的工業級高性能大模型推理算子庫", section HPC-Ops的技術原理,
"Fused AllReduce+Norm": out = RMSNorm(AllReduce(x) + residual, weight) as one
NVLink operation; the decode version stores the data straight into the peers'
memory and overlaps with the previous kernel by programmatic dependent
launch.  The kernel is moe_allreduce_rmsnorm; this module sets up the peer
memory it needs: each rank allocates its Lamport buffer, fills it with the
empty pattern, and shares a CUDA IPC handle of it with every other rank
through the process group; each rank maps the others' buffers.  After a
barrier (every buffer initialised before anyone stores into it) the layer is
ready; `call` advances by one per forward on every rank alike.
"""
from __future__ import annotations

from typing import Optional

import torch


class LamportAllReduceNorm:
    def __init__(self, T_max: int, d: int, group=None, device=None, lib=None):
        import torch.distributed as dist
        if lib is None:
            from . import moe as lib
        self.lib = lib
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.T_max, self.d = T_max, d
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.nbytes = lib.lamport_buffer_bytes(self.G, T_max, d)
        if self.nbytes == 0:
            raise ValueError(f"unsupported group size {self.G} or shape T_max={T_max}, d={d}")
        self.own, handle = lib.peer_buffer_alloc(self.nbytes)
        lib.lamport_init(self.own, self.nbytes)
        handles = [None] * self.G
        dist.all_gather_object(handles, handle, group=group)
        self.bufs = [self.own if r == self.rank else lib.peer_buffer_open(h)
                     for r, h in enumerate(handles)]
        self._sync()
        dist.barrier(group=group)           # every buffer is empty before any rank stores
        self.ws = torch.zeros(256, dtype=torch.uint8, device=self.device)
        self.call = 0

    def _sync(self):
        if torch.cuda.is_available():
            torch.cuda.synchronize()

    def __call__(self, x: torch.Tensor, residual: Optional[torch.Tensor], gamma: torch.Tensor,
                 eps: float, out: Optional[torch.Tensor] = None,
                 residual_out: Optional[torch.Tensor] = None, stream=None):
        """out (and residual_out when given) for this rank's partial x [T, d]
        bf16; every rank of the group must make the same sequence of calls."""
        if out is None:
            out = torch.empty_like(x)
        self.lib.allreduce_rmsnorm(self.bufs, self.rank, self.call, self.T_max,
                                   x.view(torch.uint16), None if residual is None else residual.view(torch.uint16),
                                   gamma.view(torch.uint16), eps, out.view(torch.uint16),
                                   None if residual_out is None else residual_out.view(torch.uint16),
                                   self.ws, stream)
        self.call += 1
        return out

    def status(self) -> int:
        return self.lib.read_device_status(self.ws)

    def close(self):
        import torch.distributed as dist
        self._sync()
        dist.barrier(group=self.group)      # no rank stores into a buffer being unmapped
        for r, p in enumerate(self.bufs):
            if r != self.rank:
                self.lib.peer_buffer_close(p)
        dist.barrier(group=self.group)
        self.lib.peer_buffer_free(self.own)
        self.bufs = []
