"""Row-gathered GEMM operands against the staged pipeline (GPU only).

With the MOE_LAYER_GATHER_ROWS flag the bf16 layer never writes the permuted
token copy: GEMM1 and the dW1/dW3 contraction fetch padded row r of expert e
straight from x as
token indices[bins[e-1] + r - padded_bins[e-1]] / K, with pad rows read as
zeros (the permute's job, "MegaBlocks - architecture", sec. 2.1 and the
dropless row layout of sec. 3).  The gathered tiles hold the same bf16 values
in the same order as the staged pipeline's x_perm, and every accumulation runs
in the same order, so the layer must agree with route -> dispatch metadata ->
permute -> grouped GEMMs -> combine (and the backward stages) bit for bit.
Every case is also held to the CPU oracle at the layer's tolerances, so an
error shared by both CUDA paths cannot pass.
"""
import numpy as np
import pytest
import torch

import dropless_top_moe_b200 as moe
from oracle import moe_oracle as om
from tests._cases import assert_scaled, make_case, small_shape

pytestmark = pytest.mark.gpu

CASES = [
    # one or two 128-row tiles per expert, CTA-pair weight gradient (H % 256 == 0)
    small_shape("g_ragged", N=300, H=256, E=8, K=2, F=256, training=True),
    # H % 256 != 0: single-CTA weight gradient with gathered rows
    small_shape("g_h384", N=515, H=384, E=16, K=4, F=384, training=True),
    # skewed: experts with no tokens and experts with many tiles
    small_shape("g_zipf", N=640, H=256, E=64, K=6, F=256, skew="zipf", skew_param=1.0, training=True),
    # several tiles per expert, odd and even tile counts
    small_shape("g_mid", N=3000, H=512, E=16, K=4, F=512, skew="normal", skew_param=0.75, training=True),
]


def _staged(c, shape, capacity=0):
    N, E, K = shape.N, shape.E, shape.K
    r = moe.moe_route(c["x"], c["W_r"], K)
    m = moe.moe_dispatch_meta(r["top_experts"], E, capacity=capacity)
    P = moe.padded_rows_max(N, E, K)
    xp = moe.moe_permute(c["x"], m["pos"], m["bins"], m["padded_bins"], K, P)
    act, out, gu = moe.moe_grouped_swiglu(xp, c["W1"], c["W3"], c["W2"], m["padded_bins"], save_gate_up=True)
    y = moe.moe_combine(out, r["weights"], m["pos"], N)
    dw, dlogit, d_out = moe.moe_combine_bwd(c["dy"], out, r["weights"], m["pos"], m["bins"], m["padded_bins"])
    gb = moe.moe_grouped_swiglu_bwd(d_out, xp, act, gu, c["W1"], c["W3"], c["W2"], m["padded_bins"])
    res = {"top": r["top_experts"], "y": y, "dW1": gb["dW1"], "dW3": gb["dW3"], "dW2": gb["dW2"]}
    if capacity == 0:
        dx, dW_r = moe.moe_unpermute_router_bwd(gb["dx_perm"], dlogit, c["x"], c["W_r"], r["top_experts"],
                                                m["pos"], m["indices"], m["bins"], m["padded_bins"])
        res.update(dx=dx, dW_r=dW_r)
    return res


def _check_oracle(c, shape, y, g, capacity=0):
    """y and every gradient against the float64 oracle (routing taken from
    the oracle's own logits; the inputs keep a 1e-3 logit gap)."""
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    W1, W3, W2 = c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu()
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], W1, W3, W2, shape.K, routing=ref, capacity=capacity)["y"]
    assert_scaled(y, yr, shape.dtype, "y vs oracle")
    if g is None:
        return
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], W1, W3, W2, shape.K, c["dy"].cpu(), routing=ref,
                         capacity=capacity)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert_scaled(g[k], gr[k], shape.dtype, f"{k} vs oracle")


def _layer(c, shape, mode=1, capacity=0):
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=mode, capacity=capacity, gather_rows=True)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"]).clone()
    g = layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    return layer, y, g


@pytest.mark.parametrize("shape", CASES, ids=lambda s: s.name)
def test_layer_gather_matches_staged_pipeline_bitwise(shape):
    c = make_case(shape, seed=31, with_dy=True)
    ref = _staged(c, shape)
    for mode in (1, 2):     # keep G, U / recompute them (the recompute gathers too)
        layer, y, g = _layer(c, shape, mode)
        assert layer.mode & moe.MOE_LAYER_GATHER_ROWS
        assert torch.equal(layer.top_experts, ref["top"])
        assert torch.equal(y, ref["y"]), "y"
        for k in ("dW1", "dW3", "dW2", "dx", "dW_r"):
            assert torch.equal(g[k], ref[k]), f"{k} mode={mode}"
        _check_oracle(c, shape, y, g)


def test_layer_gather_token_dropping_bitwise():
    shape = small_shape("g_cap", N=900, H=256, E=8, K=2, F=256, skew="zipf", skew_param=1.0, training=True)
    cap = om.capacity_from_factor(shape.N, shape.E, 1.0, shape.K)
    c = make_case(shape, seed=32, with_dy=True)
    ref = _staged(c, shape, capacity=cap)
    layer, y, g = _layer(c, shape, 1, capacity=cap)
    assert int(layer.bins[-1]) < shape.N * shape.K      # something was dropped
    assert torch.equal(y, ref["y"])
    for k in ("dW1", "dW3", "dW2"):
        assert torch.equal(g[k], ref[k]), k
    _check_oracle(c, shape, y, g, capacity=cap)



def test_gather_forward_only_layer():
    shape = small_shape("g_fwd", N=700, H=256, E=16, K=4, F=256)
    c = make_case(shape, seed=33)
    r = moe.moe_route(c["x"], c["W_r"], shape.K)
    m = moe.moe_dispatch_meta(r["top_experts"], shape.E)
    xp = moe.moe_permute(c["x"], m["pos"], m["bins"], m["padded_bins"], shape.K)
    _, out, _ = moe.moe_grouped_swiglu(xp, c["W1"], c["W3"], c["W2"], m["padded_bins"])
    y_ref = moe.moe_combine(out, r["weights"], m["pos"], shape.N)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, gather_rows=True)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert torch.equal(y, y_ref)
    _check_oracle(c, shape, y, None)
