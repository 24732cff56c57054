"""Whole-layer parity (forward and backward) of the CUDA path against the CPU
oracle, through moe_layer_fwd / moe_layer_bwd (GPU only)."""
import numpy as np
import pytest
import torch

import dropless_top_moe_b200 as moe
from gen import WORKLOADS
from oracle import moe_oracle as om
from tests._cases import TOL, assert_routing, assert_scaled, make_case, small_shape

pytestmark = pytest.mark.gpu


def run_fwd(shape, c, training=False):
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=training)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"]).clone()
    return layer, y


def check_routing_and_meta(layer, shape, ref):
    np.testing.assert_array_equal(layer.top_experts.cpu().numpy(), ref["top_experts"])
    assert_routing(layer.weights, ref["weights"], shape.H, ref["logits"], "routing weights")
    m = om.dispatch_meta(ref["top_experts"], shape.E)
    np.testing.assert_array_equal(layer.indices.cpu().numpy(), m["indices"])
    np.testing.assert_array_equal(layer.bins.cpu().numpy(), m["bins"])
    np.testing.assert_array_equal(layer.padded_bins.cpu().numpy(), m["padded_bins"])
    return m


FWD_SMALL = [
    small_shape("tiny_fp32_like", N=256, H=128, E=4, K=2, F=256, dtype="f32"),
    small_shape("f32_ragged", N=203, H=64, E=5, K=3, F=96, dtype="f32"),
    small_shape("bf16_e8", N=700, H=256, E=8, K=2, F=512),
    small_shape("bf16_e64_k6_zipf", N=900, H=256, E=64, K=6, F=384, skew="zipf", skew_param=1.0),
    small_shape("bf16_e256_k8", N=600, H=256, E=256, K=8, F=256, skew="normal", skew_param=1.0),
    small_shape("bf16_k1", N=333, H=128, E=16, K=1, F=128),
    small_shape("bf16_k_eq_e", N=250, H=128, E=16, K=16, F=128),
    small_shape("f32_single_expert", N=77, H=32, E=1, K=1, F=48, dtype="f32"),
    small_shape("megablocks_dmoe_test_dims", N=1024, H=512, E=8, K=2, F=1024),
]


@pytest.mark.parametrize("shape", FWD_SMALL, ids=lambda s: s.name)
def test_layer_forward_small(shape):
    c = make_case(shape, seed=3)
    layer, y = run_fwd(shape, c)
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    check_routing_and_meta(layer, shape, ref)
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(),
                        shape.K, routing=ref)["y"]
    assert_scaled(y, yr, shape.dtype, "y")


def test_layer_forward_tiny_fp32_workload():
    shape = WORKLOADS["tiny_fp32"]
    c = make_case(shape, seed=0)
    layer, y = run_fwd(shape, c)
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    check_routing_and_meta(layer, shape, ref)
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(),
                        shape.K, routing=ref)["y"]
    assert_scaled(y, yr, "f32", "y")


def test_one_expert_takes_every_token():
    shape = small_shape("hot", N=512, H=128, E=8, K=2, F=128, skew="zipf", skew_param=1.0)
    c = make_case(shape, seed=4, repair=False)
    c["W_r"][0, :] = 0
    c["W_r"][0, 5] = 60.0          # expert 5 first for every token
    c["W_r"][0, 2] = 30.0          # expert 2 second
    layer, y = run_fwd(shape, c)
    te = layer.top_experts.cpu().numpy()
    assert np.all(te[:, 0] == 5) and np.all(te[:, 1] == 2)
    bins = layer.bins.cpu().numpy()
    assert bins[-1] == 1024 and np.count_nonzero(np.diff(np.concatenate([[0], bins]))) == 2
    ref = om.route(c["x"].cpu(), c["W_r"].cpu(), 2)
    yr = om.moe_forward(c["x"].cpu(), c["W_r"].cpu(), c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), 2,
                        routing=ref)["y"]
    assert_scaled(y, yr, "bf16", "y")


def test_layer_forward_mixtral_full_size_sampled():
    shape = WORKLOADS["mixtral"]
    c = make_case(shape, seed=0)
    layer, y = run_fwd(shape, c)
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    m = check_routing_and_meta(layer, shape, ref)
    assert om.maxvio(m["hist"], shape.N, shape.K, shape.E) < 0.3
    tok = np.sort(np.random.default_rng(0).choice(shape.N, 1024, replace=False))
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"], c["W3"], c["W2"], shape.K, routing=ref,
                        tokens=tok)["y"]
    assert_scaled(y[torch.as_tensor(tok, device="cuda")], yr, "bf16", "y sampled")


BWD_SMALL = [
    small_shape("f32_bwd", N=256, H=64, E=4, K=2, F=96, dtype="f32", training=True),
    small_shape("f32_bwd_k3", N=190, H=32, E=6, K=3, F=64, dtype="f32", training=True),
    small_shape("bf16_bwd", N=640, H=256, E=8, K=2, F=256, training=True),
    small_shape("bf16_bwd_e64", N=900, H=256, E=64, K=4, F=384, training=True),
    small_shape("bf16_bwd_h128", N=400, H=128, E=16, K=4, F=128, training=True),
    # every token to both experts, so each expert holds N rows: more than 8
    # row units, and the grouped GEMMs' raster cuts an expert into several
    # groups (H=384: 128-row units in GEMM2 and the dgrad to x)
    small_shape("bf16_bwd_big_experts", N=2500, H=256, E=2, K=2, F=256, training=True),
    small_shape("bf16_bwd_big_h384", N=1500, H=384, E=2, K=2, F=256, training=True),
]


def _bwd_case(shape, seed):
    c = make_case(shape, seed=seed, with_dy=True)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=True)
    layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    g = layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    return c, layer, g


# The bf16 router's H split (S = 8, 4, 2 for these shapes) gives the dispatch
# metadata chunks of 16, 32 and 64 tokens, counted in the router's epilogue;
# N is not a multiple of the chunk, so the last chunk is ragged.
SPLIT = [small_shape("split8", N=1000, H=2048, E=64, K=4, F=256, training=True),
         small_shape("split4_zipf", N=700, H=1024, E=16, K=2, F=128, skew="zipf", skew_param=1.0,
                     training=True),
         small_shape("split2_e256", N=6000, H=1024, E=256, K=8, F=128, skew="normal", skew_param=0.75,
                     training=True)]


@pytest.mark.parametrize("shape", SPLIT, ids=lambda s: s.name)
def test_layer_with_split_router_matches_oracle(shape):
    c, layer, g = _bwd_case(shape, seed=16)
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    check_routing_and_meta(layer, shape, ref)
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                        routing=ref)["y"]
    assert_scaled(layer.y, yr, shape.dtype, "y")
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                         c["dy"].cpu(), routing=ref)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert_scaled(g[k], gr[k], shape.dtype, k)


@pytest.mark.parametrize("shape", BWD_SMALL, ids=lambda s: s.name)
def test_layer_backward_small(shape):
    c, layer, g = _bwd_case(shape, seed=5)
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    check_routing_and_meta(layer, shape, ref)
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(),
                         shape.K, c["dy"].cpu(), routing=ref)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert_scaled(g[k], gr[k], shape.dtype, k)


def test_layer_is_bitwise_deterministic():
    shape = small_shape("det", N=1500, H=256, E=64, K=4, F=256, training=True)
    outs = []
    for _ in range(2):
        c, layer, g = _bwd_case(shape, seed=6)
        outs.append([layer.y.clone(), layer.top_experts.clone(), layer.weights.clone()] +
                    [g[k].clone() for k in ("dx", "dW_r", "dW1", "dW3", "dW2")])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


# bf16 with E % 64 == 0 and H % 256 == 0 runs the dense router backward on
# tensor cores (D rounded to bf16); the other shapes on CUDA cores in fp32
AUX = [small_shape("aux_f32", N=256, H=64, E=8, K=2, F=96, dtype="f32", training=True),
       small_shape("aux_bf16", N=700, H=256, E=64, K=4, F=256, training=True),
       small_shape("aux_bf16_e128", N=1500, H=512, E=128, K=6, F=256, skew="zipf", skew_param=1.0,
                   training=True),
       small_shape("aux_bf16_e8", N=333, H=128, E=8, K=2, F=128, training=True),
       small_shape("aux_bf16_n3", N=3, H=256, E=64, K=2, F=256, training=True)]


@pytest.mark.parametrize("shape", AUX, ids=lambda s: s.name)
def test_layer_with_load_balancing_loss(shape):
    alpha, g = 0.01, 1.7
    c = make_case(shape, seed=8, with_dy=True)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=True, aux_alpha=alpha)
    layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    grads = layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"], aux_grad=g)
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    check_routing_and_meta(layer, shape, ref)
    la = om.aux_loss(ref["probs"], ref["top_experts"], alpha)
    assert abs(layer.aux_loss.item() - la) <= 1e-4 * abs(la)
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                         c["dy"].cpu(), routing=ref, aux_alpha=alpha, aux_grad=g)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert_scaled(grads[k], gr[k], shape.dtype, k)


def test_aux_loss_stage_matches_oracle():
    shape = small_shape("aux_stage", N=1000, H=256, E=64, K=6, skew="zipf", skew_param=1.0)
    c = make_case(shape, seed=9)
    r = moe.moe_route(c["x"], c["W_r"], shape.K, want_probs=True)
    m = moe.moe_dispatch_meta(r["top_experts"], shape.E)
    loss, P = moe.moe_aux_loss(r["probs"], m["bins"], shape.K, 0.05)
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    la = om.aux_loss(ref["probs"], ref["top_experts"], 0.05)
    assert abs(loss.item() - la) <= 1e-4 * abs(la)
    assert_scaled(P, ref["probs"].mean(axis=0), "f32", "P")


CAP = [small_shape("cap_f32", N=256, H=64, E=8, K=2, F=96, dtype="f32", training=True),
       small_shape("cap_bf16_zipf", N=900, H=256, E=16, K=4, F=256, skew="zipf", skew_param=1.0,
                   training=True),
       small_shape("cap_bf16_e64", N=1000, H=256, E=64, K=4, F=256, skew="zipf", skew_param=1.0,
                   training=True)]


@pytest.mark.parametrize("shape", CAP, ids=lambda s: s.name)
def test_layer_token_dropping_variant(shape):
    cap = om.capacity_from_factor(shape.N, shape.E, 1.0, shape.K)   # icman sec. 3.4, factor 1
    c = make_case(shape, seed=12, with_dy=True)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=True, capacity=cap)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"]).clone()
    g = layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    np.testing.assert_array_equal(layer.top_experts.cpu().numpy(), ref["top_experts"])
    m = om.dispatch_meta(ref["top_experts"], shape.E, capacity=cap)
    assert m["hist"].sum() < shape.N * shape.K          # something was dropped
    np.testing.assert_array_equal(layer.bins.cpu().numpy(), m["bins"])
    np.testing.assert_array_equal(layer.padded_bins.cpu().numpy(), m["padded_bins"])
    np.testing.assert_array_equal(layer.indices.cpu().numpy()[:m["indices"].size], m["indices"])
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                        routing=ref, capacity=cap)["y"]
    assert_scaled(y, yr, shape.dtype, "y")
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                         c["dy"].cpu(), routing=ref, capacity=cap)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert_scaled(g[k], gr[k], shape.dtype, k)


def test_dispatch_meta_capacity_bit_exact():
    g = torch.Generator().manual_seed(21)
    te = torch.stack([torch.randperm(16, generator=g)[:3] for _ in range(3000)]).to(torch.int32)
    te[:1500, 0] = 5                                    # overflow expert 5
    for cap in (1, 100, 600, 10 ** 6):
        m = moe.moe_dispatch_meta(te.cuda(), 16, capacity=cap)
        ref = om.dispatch_meta(te.numpy(), 16, capacity=cap)
        n = ref["indices"].size
        for k in ("bins", "padded_bins", "pos"):
            np.testing.assert_array_equal(m[k].cpu().numpy(), ref[k], err_msg=f"{k} cap={cap}")
        for k in ("indices", "bin_ids"):
            np.testing.assert_array_equal(m[k].cpu().numpy()[:n], ref[k], err_msg=f"{k} cap={cap}")


@pytest.mark.parametrize("shape", [small_shape("memopt_bf16", N=800, H=256, E=16, K=4, F=384, training=True),
                                   small_shape("memopt_f32", N=200, H=64, E=4, K=2, F=96, dtype="f32",
                                               training=True)], ids=lambda s: s.name)
def test_memory_optimised_backward_is_bit_identical(shape):
    """training=2 keeps no gate/up projections and recomputes them in the
    backward with the forward's own kernel: same bits as training=1, less
    workspace, and both within tolerance of the oracle."""
    c = make_case(shape, seed=13, with_dy=True)
    outs = {}
    for mode in (1, 2):
        layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                             training=mode)
        y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"]).clone()
        g = {k: v.clone() for k, v in layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"]).items()}
        torch.cuda.synchronize()
        assert layer.status() == 0
        outs[mode] = (y, g, layer.ws.numel())
    assert outs[2][2] < outs[1][2]
    assert torch.equal(outs[1][0], outs[2][0])
    for k in outs[1][1]:
        assert torch.equal(outs[1][1][k], outs[2][1][k]), k
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    W1, W3, W2 = c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu()
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], W1, W3, W2, shape.K, routing=ref)["y"]
    assert_scaled(outs[2][0], yr, shape.dtype, "y")
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], W1, W3, W2, shape.K, c["dy"].cpu(), routing=ref)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert_scaled(outs[2][1][k], gr[k], shape.dtype, k)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_empty_batch(dtype):
    """N = 0: the forward writes all-zero bins and nothing else; the backward
    gives zero weight gradients (sums over no tokens).  Token-sized buffers
    are empty tensors (NULL pointers)."""
    H, F = (256, 256) if dtype == "bf16" else (64, 96)
    shape = small_shape("empty", N=0, H=H, E=8, K=2, F=F, dtype=dtype, training=True)
    c = make_case(shape, seed=3, with_dy=True)
    layer = moe.MoELayer(0, H, shape.E, shape.K, F, dtype=shape.torch_dtype, training=True)
    layer.bins.fill_(-1)
    layer.padded_bins.fill_(-1)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    g = layer.grad_buffers()
    for v in g.values():
        v.fill_(1.0)
    layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert tuple(y.shape) == (0, H)
    assert int(layer.bins.abs().sum()) == 0 and int(layer.padded_bins.abs().sum()) == 0
    for k in ("dW_r", "dW1", "dW3", "dW2"):
        assert int(torch.count_nonzero(g[k])) == 0, k


# Load-balancing loss and token dropping together: the loss's f_i count every
# routed assignment, dropped ones included (icman sec. 4.2 defines f_i as the
# share of tokens the router assigns to expert i; capacity, sec. 3.4, acts
# after that assignment).  bf16 E % 64 == 0 takes the tensor-core dense router
# backward, the others the fp32 CUDA-core one.
AUX_CAP = [small_shape("auxcap_f32", N=256, H=64, E=8, K=2, F=96, dtype="f32", skew="zipf", skew_param=1.0,
                       training=True),
           small_shape("auxcap_bf16_e64", N=1000, H=256, E=64, K=4, F=256, skew="zipf", skew_param=1.0,
                       training=True),
           small_shape("auxcap_bf16_e16", N=700, H=128, E=16, K=2, F=128, skew="zipf", skew_param=1.0,
                       training=True)]


@pytest.mark.parametrize("shape", AUX_CAP, ids=lambda s: s.name)
def test_layer_aux_loss_with_token_dropping(shape):
    alpha, g = 0.02, 0.9
    cap = om.capacity_from_factor(shape.N, shape.E, 1.0, shape.K)
    c = make_case(shape, seed=14, with_dy=True)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=True, aux_alpha=alpha, capacity=cap)
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"]).clone()
    grads = layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"], aux_grad=g)
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    np.testing.assert_array_equal(layer.top_experts.cpu().numpy(), ref["top_experts"])
    m = om.dispatch_meta(ref["top_experts"], shape.E, capacity=cap)
    assert m["hist"].sum() < shape.N * shape.K          # something was dropped
    np.testing.assert_array_equal(layer.bins.cpu().numpy(), m["bins"])
    la = om.aux_loss(ref["probs"], ref["top_experts"], alpha)
    assert abs(layer.aux_loss.item() - la) <= 1e-4 * abs(la)
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                        routing=ref, capacity=cap)["y"]
    assert_scaled(y, yr, shape.dtype, "y")
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                         c["dy"].cpu(), routing=ref, aux_alpha=alpha, aux_grad=g, capacity=cap)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert_scaled(grads[k], gr[k], shape.dtype, k)


# Every layer variant on a workspace whose bytes past the status region hold
# 0xFF (a NaN bit pattern for fp32 and bf16), with NaN-filled outputs: a read
# of anything the forward did not write, or an output left unwritten, shows
# up as NaN against the oracle.
POISON = [("dropless", dict()), ("capacity", dict(capacity_factor=1.0)), ("aux", dict(aux_alpha=0.01)),
          ("aux_capacity", dict(aux_alpha=0.01, capacity_factor=1.0)), ("memopt", dict(mode=2)),
          ("gather", dict(gather_rows=True)), ("gather_memopt_capacity", dict(gather_rows=True, mode=2,
                                                                              capacity_factor=1.0))]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("name,opts", POISON, ids=[p[0] for p in POISON])
def test_layer_on_poisoned_workspace_matches_oracle(dtype, name, opts):
    if dtype == "f32" and opts.get("gather_rows"):
        pytest.skip("row gathers are a bf16 option")
    if dtype == "bf16":
        shape = small_shape("poison", N=777, H=256, E=64, K=4, F=256, skew="zipf", skew_param=1.0,
                            training=True)
    else:
        shape = small_shape("poison_f32", N=200, H=64, E=8, K=2, F=96, dtype="f32", skew="zipf",
                            skew_param=1.0, training=True)
    cap = (om.capacity_from_factor(shape.N, shape.E, opts["capacity_factor"], shape.K)
           if "capacity_factor" in opts else 0)
    alpha, g = opts.get("aux_alpha", 0.0), 1.3
    c = make_case(shape, seed=15, with_dy=True)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype,
                         training=opts.get("mode", 1), aux_alpha=alpha, capacity=cap,
                         gather_rows=opts.get("gather_rows", False))
    layer.ws[256:].fill_(0xFF)
    grads = layer.grad_buffers()
    for v in grads.values():
        v.fill_(float("nan"))
    layer.y.fill_(float("nan"))
    y = layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"]).clone()
    layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"], aux_grad=g)
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    np.testing.assert_array_equal(layer.top_experts.cpu().numpy(), ref["top_experts"])
    if alpha:
        la = om.aux_loss(ref["probs"], ref["top_experts"], alpha)
        assert abs(layer.aux_loss.item() - la) <= 1e-4 * abs(la)
    yr = om.moe_forward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                        routing=ref, capacity=cap)["y"]
    assert_scaled(y, yr, shape.dtype, "y")
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), shape.K,
                         c["dy"].cpu(), routing=ref, aux_alpha=alpha, aux_grad=g, capacity=cap)
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        assert not torch.isnan(grads[k]).any(), k
        assert_scaled(grads[k], gr[k], shape.dtype, k)
