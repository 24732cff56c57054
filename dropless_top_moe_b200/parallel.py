"""Deterministic gradient all-reduce for data-parallel replicas of the layer.

The layer itself has no exchange step: each GPU runs the whole forward and
backward on its own tokens.  A data-parallel trainer then sums the weight
gradients (dW_r, dW1, dW3, dW2) over the replicas.  This helper does that sum
so that the result is bitwise identical on every rank and from run to run,
whatever order the interconnect delivers data in:

  1. all-to-all: rank r receives every rank's copy of shard r (equal shards);
  2. local sum of those copies in rank order (moe_sum_rank_ordered on the GPU,
     an explicit ordered loop on CPU tensors);
  3. all-gather of the reduced shards.

Communication per rank is 2 * (world-1)/world of the tensor, like a ring
all-reduce.  torch.distributed only moves bytes; the arithmetic is the
library kernel on CUDA tensors.
"""
from __future__ import annotations

from typing import Iterable, Optional

import torch
import torch.distributed as dist

from ._lib import MOE_BF16, MOE_F32, call

_DT = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16}


def _ordered_sum(recv: torch.Tensor, world: int, scale: float, out: torch.Tensor) -> None:
    """out = scale * sum over rows of recv [world, shard], rows in rank order."""
    if recv.is_cuda:
        call("moe_sum_rank_ordered", recv.data_ptr(), world, out.numel(), _DT[recv.dtype], float(scale),
             out.data_ptr(), torch.cuda.current_stream(recv.device).cuda_stream)
        return
    acc = torch.zeros(out.shape, dtype=torch.float32)
    for r in range(world):
        acc += recv[r].to(torch.float32)
    out.copy_((acc * scale).to(out.dtype))


def allreduce_grads(tensors: Iterable[torch.Tensor], group: Optional[dist.ProcessGroup] = None,
                    average: bool = True, chunk_elems: int = 1 << 26) -> None:
    """Sum (or average) each tensor over the ranks of `group`, in place,
    deterministically.  Tensors must be contiguous float32 or bfloat16."""
    world = dist.get_world_size(group)
    if world == 1:
        return
    scale = 1.0 / world if average else 1.0
    for t in tensors:
        if t.dtype not in _DT or not t.is_contiguous():
            raise TypeError("gradients must be contiguous float32 or bfloat16 tensors")
        flat = t.view(-1)
        align = 8 * world
        for start in range(0, flat.numel(), chunk_elems):
            piece = flat[start:start + chunk_elems]
            n = piece.numel()
            padded = (n + align - 1) // align * align
            send = torch.zeros(padded, dtype=t.dtype, device=t.device)
            send[:n].copy_(piece)
            shard = padded // world
            recv = torch.empty(world, shard, dtype=t.dtype, device=t.device)
            dist.all_to_all_single(recv.view(-1), send, group=group)
            red = torch.empty(shard, dtype=t.dtype, device=t.device)
            _ordered_sum(recv, world, scale, red)
            gathered = torch.empty(padded, dtype=t.dtype, device=t.device)
            dist.all_gather_into_tensor(gathered, red, group=group)
            piece.copy_(gathered[:n])
