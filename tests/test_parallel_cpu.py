"""Data-parallel gradient reduction across replicas: gloo ranks on CPU.

Each rank holds gradients of its own tokens; after allreduce_grads every rank
must hold the rank-ordered average, bitwise equal across ranks and runs.  The
library's rank-ordered sum kernel needs a GPU, so these CPU ranks exercise
the exchange (all-to-all of shards, all-gather, chunking and padding) with a
rank-ordered sum written here; the kernel itself is checked on the GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dropless_top_moe_b200.parallel import allreduce_grads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cpu_ordered_sum(recv, world, scale, out):
    acc = torch.zeros(out.shape, dtype=torch.float32)
    for r in range(world):
        acc += recv[r].to(torch.float32)
    out.copy_((acc * scale).to(out.dtype))


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = []
        for dt in (torch.float32, torch.bfloat16):
            g = torch.Generator().manual_seed(100 + rank)
            ts = [torch.randn(3, 70, 33, generator=g).to(dt), torch.randn(1001, generator=g).to(dt)]
            allreduce_grads(ts, average=True, chunk_elems=512, local_sum=_cpu_ordered_sum)
            out.append([t.clone() for t in ts])
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_default_sum_refuses_cpu_tensors():
    from dropless_top_moe_b200.parallel import ordered_sum
    with pytest.raises(RuntimeError, match="CUDA"):
        ordered_sum(torch.zeros(2, 8), 2, 0.5, torch.zeros(8))


@pytest.mark.parametrize("world", [2, 3])
def test_allreduce_grads_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # expected: rank-ordered fp32 sum of every rank's tensors, times 1/world
    for di, dt in enumerate((torch.float32, torch.bfloat16)):
        gens = [torch.Generator().manual_seed(100 + r) for r in range(world)]
        inputs = [[torch.randn(3, 70, 33, generator=g).to(dt), torch.randn(1001, generator=g).to(dt)]
                  for g in gens]
        for ti in range(2):
            acc = torch.zeros(inputs[0][ti].shape, dtype=torch.float32)
            for r in range(world):
                acc += inputs[r][ti].float()
            exp = (acc * (1.0 / world)).to(dt)
            for r in range(world):
                assert torch.equal(res[r][di][ti], exp), (dt, ti, r)
