"""Failure detection on the GPU without a fault (GPU only).

A stalled pipeline must end its kernel with a status bit the host can read,
not hang the GPU: every mbarrier wait of the tcgen05 pipelines is bounded.
The self-test entry point runs that same wait on a barrier nothing arrives
at.  Grouped rows beyond a caller's buffer are reported the same way.
"""
import numpy as np
import pytest
import torch

import dropless_top_moe_b200 as moe
from dropless_top_moe_b200._lib import MOE_DEVERR_MODE, MOE_DEVERR_ROWS, MOE_DEVERR_TIMEOUT
from oracle import moe_oracle as om
from tests._cases import assert_scaled, make_case, small_shape

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_into_the_status_word():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.selftest_wait_timeout(st, 20_000_000)       # 20 ms
    torch.cuda.synchronize()
    assert int(st.item()) & MOE_DEVERR_TIMEOUT
    # the context is still usable: a layer runs and matches the oracle
    shape = small_shape("after_timeout", N=300, H=256, E=8, K=2, F=256)
    c = make_case(shape, seed=41)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K)
    assert_scaled(y, ref["y"], "bf16", "y")


def test_padded_rows_beyond_the_buffer_are_reported():
    H, F, E = 256, 256, 2
    pb = torch.tensor([256, 640], dtype=torch.int32, device="cuda")   # 640 rows needed
    P = 512                                                            # buffer holds 512
    g = torch.Generator(device="cuda").manual_seed(5)
    x_perm = torch.randn(P, H, generator=g, device="cuda").to(torch.bfloat16)
    W1 = (torch.randn(E, H, F, generator=g, device="cuda") / 16).to(torch.bfloat16)
    W3 = (torch.randn(E, H, F, generator=g, device="cuda") / 16).to(torch.bfloat16)
    W2 = (torch.randn(E, F, H, generator=g, device="cuda") / 16).to(torch.bfloat16)
    ws = moe.workspace(moe.load().moe_grouped_workspace_size(), "cuda")
    moe.moe_grouped_swiglu(x_perm, W1, W3, W2, pb, ws=ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) & MOE_DEVERR_ROWS


def test_backward_flags_unlike_the_forward_are_reported():
    # The backward reads buffers the forward wrote at offsets that the
    # training flags decide.  Both mismatches below keep every access inside
    # the workspace (the token positions sit at the same offset in every
    # layout); the check turns what would be silent garbage into a status bit.
    shape = small_shape("flags_mismatch", N=300, H=256, E=8, K=2, F=256, training=True)
    c = make_case(shape, seed=43, with_dy=True)
    args = (c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    for fwd_mode, bwd_mode in ((1, 2), (1, 1 | moe.MOE_LAYER_GATHER_ROWS)):
        layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, training=fwd_mode)
        layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
        layer.backward(*args)
        torch.cuda.synchronize()
        assert layer.status() == 0
        layer.mode = bwd_mode        # workspace sized for fwd_mode: large enough for bwd_mode
        layer.backward(*args)
        torch.cuda.synchronize()
        assert layer.status() & MOE_DEVERR_MODE, (fwd_mode, bwd_mode)
