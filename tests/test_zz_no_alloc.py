"""The allocation-free dispatch-metadata entry point (GPU only).

moe_dispatch_meta_noalloc serves callers that cannot call cudaMalloc (code
inside another runtime that owns all device memory, or a hot path where an
allocation is not allowed): its scratch is a fixed device array inside the
library.  Its outputs must equal those of moe_dispatch_meta, which uses a
caller workspace, on consecutive calls that reuse the shared array.
This file is collected last so a failure here leaves every other test run.
"""
import numpy as np
import pytest
import torch

import dropless_top_moe_b200 as moe
from dropless_top_moe_b200._lib import MOE_ERR_WORKSPACE, call, load

pytestmark = pytest.mark.gpu


def _routing(N, K, E, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randperm(E, generator=g)[:K] for _ in range(N)]).to(torch.int32)


def _noalloc(te, E):
    N, K = te.shape
    dev = te.device
    out = {k: torch.full((N * K,), -7, dtype=torch.int32, device=dev) for k in ("indices", "bin_ids", "pos")}
    out["bins"] = torch.full((E,), -7, dtype=torch.int32, device=dev)
    out["padded_bins"] = torch.full((E,), -7, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    call("moe_dispatch_meta_noalloc", te.data_ptr(), N, K, E, out["indices"].data_ptr(),
         out["bin_ids"].data_ptr(), out["bins"].data_ptr(), out["padded_bins"].data_ptr(),
         out["pos"].data_ptr(), status.data_ptr(), s)
    torch.cuda.synchronize()
    return out, int(status.item())


def test_noalloc_meta_matches_workspace_entry_on_consecutive_calls():
    # a larger call first, then a smaller one: the second must not see
    # anything the first left in the shared array
    for N, K, E, seed in ((6000, 8, 256, 1), (1500, 2, 8, 2)):
        te = _routing(N, K, E, seed).cuda()
        ref = moe.moe_dispatch_meta(te, E)
        got, status = _noalloc(te, E)
        assert status == 0
        for k in ("indices", "bin_ids", "bins", "padded_bins", "pos"):
            assert torch.equal(got[k], ref[k]), k


def test_noalloc_meta_rejects_sizes_beyond_its_array():
    lib = load()
    fake = 0x10000   # never dereferenced: the size check returns first
    assert lib.moe_dispatch_meta_noalloc(fake, 300000, 8, 256, fake, fake, fake, fake, fake, None,
                                         None) == MOE_ERR_WORKSPACE
