"""ZeRO-style sharded step over peer memory (front end of opt2s_shard_step).

Every rank holds the whole flat param buffer and its own whole flat grad
buffer; ``ShardedStep`` keeps the fp32 optimizer state of this rank's shard
only and, per step, launches ONE kernel that averages all ranks' gradients
for the shard (rank order, fp32), updates it, and writes the new values into
every rank's param buffer.  How the other ranks' buffers become addressable
from this device is the caller's choice (CUDA IPC handles, symmetric memory,
or peer access between devices driven by one process); the step only needs
their addresses.  ``PeerBuffers`` does it with CUDA IPC over a
torch.distributed process group, one process per GPU.  Order each step after
all ranks' gradients are complete and before any rank reads its params again
(a barrier on each side).
"""
from __future__ import annotations

import torch

from . import binding as B


def shard_range(numel: int, world: int, rank: int) -> tuple:
    """(start, length) of ``rank``'s shard; shards are disjoint, cover every
    element, differ in size by at most 8 and start at multiples of 8."""
    return B.opt2s_shard_range(numel, world, rank)


class PeerBuffers:
    """Every rank's flat param and grad buffers, addressable from this rank's
    device: this rank's own tensors, and the other ranks' allocations mapped
    through CUDA IPC (opt2s_ipc_export / opt2s_ipc_open; across GPUs the
    mapping enables peer access, so the step's loads and stores cross
    NVLink).  The handles travel with one all_gather_object over ``group``.
    Call close() once no kernel uses the mappings any more."""

    def __init__(self, param: torch.Tensor, grad: torch.Tensor, group=None):
        import torch.distributed as dist
        world = dist.get_world_size(group)
        rank = dist.get_rank(group)
        mine = (B.ipc_export(param), B.ipc_export(grad), param.numel(), str(param.dtype))
        every = [None] * world
        dist.all_gather_object(every, mine, group=group)
        for q, (_, _, n, dt) in enumerate(every):
            if n != param.numel() or dt != str(param.dtype):
                raise ValueError(f"rank {q} holds {n} elements of {dt}; every rank must match")
        self.params, self.grads = [], []
        self._bases = []
        opened = {}          # one mapping per exported allocation
        for q, (ph, gh, _, _) in enumerate(every):
            if q == rank:
                self.params.append(param)
                self.grads.append(grad)
                continue
            addr = []
            for handle, offset in (ph, gh):
                if handle not in opened:
                    base, _ = B.ipc_open(handle, 0)
                    opened[handle] = base
                    self._bases.append(base)
                addr.append(opened[handle] + offset)
            self.params.append(addr[0])
            self.grads.append(addr[1])
        self._keep = (param, grad)

    def close(self) -> None:
        for base in self._bases:
            B.ipc_close(base)
        self._bases = []


class ShardedStep:
    def __init__(self, params: list, grads: list, rank: int, algo: str = "adam",
                 device=None):
        """params[q], grads[q]: rank q's flat buffers (torch tensors or raw
        device addresses usable from this rank's device), equal length and
        dtype.  The state tensors for this rank's shard are allocated here."""
        if len(params) != len(grads) or not 1 <= len(params) <= B.MAX_WORLD:
            raise ValueError(f"1..{B.MAX_WORLD} ranks, one param and one grad buffer each")
        self.world = len(params)
        self.rank = rank
        self.algo = "ademamix" if algo == "ademamix" else "adam"
        ref = params[rank]
        self.numel = ref.numel()
        self.dtype = B._torch_dtype_code(ref)
        for p, g in zip(params, grads):
            if isinstance(p, torch.Tensor) and (p.numel() != self.numel or p.dtype != ref.dtype):
                raise ValueError("every rank's param buffer must match in length and dtype")
            if isinstance(g, torch.Tensor) and (g.numel() != self.numel or g.dtype != ref.dtype):
                raise ValueError("every rank's grad buffer must match the params")
        self.start, self.length = shard_range(self.numel, self.world, rank)
        dev = device if device is not None else ref.device
        k = self.length
        self.state1 = torch.zeros(2 * k if self.algo == "ademamix" else k, dtype=torch.float32, device=dev)
        self.state2 = torch.zeros(k, dtype=torch.float32, device=dev)
        self._keep = (params, grads)
        self.desc = B.make_shard_desc(self.world, rank, self.numel, self.dtype, params, grads,
                                      self.state1 if k else None, self.state2 if k else None)

    def step(self, hyper: B.Hyper, step: int, stream=None) -> None:
        B.opt2s_shard_step(self.desc, hyper, step, stream)
