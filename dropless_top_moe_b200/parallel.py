"""Deterministic gradient all-reduce for data-parallel replicas of the layer.

The layer itself has no exchange step: each GPU runs the whole forward and
backward on its own tokens.  A data-parallel trainer then sums the weight
gradients (dW_r, dW1, dW3, dW2) over the replicas.  This helper does that sum
so that the result is bitwise identical on every rank and from run to run,
whatever order the interconnect delivers data in:

  1. all-to-all: rank r receives every rank's copy of shard r (equal shards);
  2. local sum of those copies in rank order (the moe_sum_rank_ordered
     kernel);
  3. all-gather of the reduced shards.

Communication per rank is 2 * (world-1)/world of the tensor, like a ring
all-reduce.  torch.distributed only moves bytes; the arithmetic is the
library kernel, so the tensors must live on the GPU.  (The exchange logic
alone can be exercised on CPU ranks by passing another `local_sum`.)
"""
from __future__ import annotations

from typing import Callable, Iterable, Optional

import torch
import torch.distributed as dist

from ._lib import MOE_BF16, MOE_F32, call

_DT = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16}


def ordered_sum(recv: torch.Tensor, world: int, scale: float, out: torch.Tensor) -> None:
    """out = scale * sum over rows of recv [world, shard], rows in rank order
    (the library's moe_sum_rank_ordered kernel; CUDA tensors only)."""
    if not (recv.is_cuda and out.is_cuda):
        raise RuntimeError("the rank-ordered sum runs in the library kernel: CUDA tensors only")
    call("moe_sum_rank_ordered", recv.data_ptr(), world, out.numel(), _DT[recv.dtype], float(scale),
         out.data_ptr(), torch.cuda.current_stream(recv.device).cuda_stream)


def allreduce_grads(tensors: Iterable[torch.Tensor], group: Optional[dist.ProcessGroup] = None,
                    average: bool = True, chunk_elems: int = 1 << 26,
                    local_sum: Callable[[torch.Tensor, int, float, torch.Tensor], None] = ordered_sum) -> None:
    """Sum (or average) each tensor over the ranks of `group`, in place,
    deterministically.  Tensors must be contiguous float32 or bfloat16.
    local_sum(recv [world, shard], world, scale, out) is step 2."""
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
            local_sum(recv, world, scale, red)
            gathered = torch.empty(padded, dtype=t.dtype, device=t.device)
            dist.all_gather_into_tensor(gathered, red, group=group)
            piece.copy_(gathered[:n])
