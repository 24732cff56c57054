"""The Python binding refuses tensors whose shape or dtype disagrees with the
sizes a call derives from its other arguments (CPU only: the checks run
before any workspace allocation or library call).  The library reads and
writes through raw pointers with those sizes, so each of these mistakes
would otherwise touch memory outside a tensor."""
import pytest
import torch

import dropless_top_moe_b200 as moe

N, H, E, K, F = 32, 128, 4, 2, 256
P = 640
bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def z(*shape, dtype=bf):
    return torch.zeros(*shape, dtype=dtype)


def test_route_checks_router_weights():
    with pytest.raises(ValueError, match="W_r"):
        moe.moe_route(z(N, H), z(H + 128, E), K)
    with pytest.raises(TypeError, match="W_r"):
        moe.moe_route(z(N, H), z(H, E, dtype=f32), K)


def test_dispatch_meta_wants_int32_ids():
    with pytest.raises(TypeError, match="top_experts"):
        moe.moe_dispatch_meta(z(N, K, dtype=torch.int64), E)


def test_permute_checks_index_arrays_and_output():
    x, bins = z(N, H), z(E, dtype=i32)
    with pytest.raises(ValueError, match="pos"):
        moe.moe_permute(x, z(N * K - 1, dtype=i32), bins, bins, K)
    with pytest.raises(ValueError, match="padded_bins"):
        moe.moe_permute(x, z(N * K, dtype=i32), bins, z(E + 1, dtype=i32), K)
    with pytest.raises(ValueError, match="out"):
        moe.moe_permute(x, z(N * K, dtype=i32), bins, bins, K, P=P, out=z(P, H - 128))


def test_grouped_swiglu_checks_every_expert_weight():
    xp, pb = z(P, H), z(E, dtype=i32)
    W1, W3, W2 = z(E, H, F), z(E, H, F), z(E, F, H)
    with pytest.raises(ValueError, match="W3"):
        moe.moe_grouped_swiglu(xp, W1, z(E, H, F + 128), W2, pb)
    with pytest.raises(ValueError, match="W2"):
        moe.moe_grouped_swiglu(xp, W1, W3, z(E, H, F), pb)          # transposed W2
    with pytest.raises(ValueError, match="W1"):
        moe.moe_grouped_swiglu(z(P, H + 128), W1, W3, W2, pb)      # x_perm width != W1's H
    with pytest.raises(ValueError, match="padded_bins"):
        moe.moe_grouped_swiglu(xp, W1, W3, W2, z(E - 1, dtype=i32))
    with pytest.raises(TypeError, match="W1"):
        moe.moe_grouped_swiglu(xp, z(E, H, F, dtype=f32), W3, W2, pb)
    with pytest.raises(ValueError, match="gate_up"):
        moe.moe_grouped_swiglu_bwd(z(P, H), xp, z(P, F), z(P, F), W1, W3, W2, pb)


def test_combine_and_its_backward_check_routing_arrays():
    out, pos = z(P, H), z(N * K, dtype=i32)
    with pytest.raises(TypeError, match="weights"):
        moe.moe_combine(out, z(N, K), pos, N)                       # bf16 weights
    with pytest.raises(ValueError, match="pos"):
        moe.moe_combine(out, z(N, K, dtype=f32), z(N, dtype=i32), N)
    with pytest.raises(ValueError, match="y"):
        moe.moe_combine(out, z(N, K, dtype=f32), pos, N, y=z(N + 1, H))
    with pytest.raises(ValueError, match="out"):
        moe.moe_combine_bwd(z(N, H), z(P, H + 128), z(N, K, dtype=f32), pos, z(E, dtype=i32), z(E, dtype=i32))


def test_router_backward_and_aux_loss_check_their_inputs():
    args = dict(dx_perm=z(P, H), dlogit=z(N, K, dtype=f32), x=z(N, H), W_r=z(H, E), top_experts=z(N, K, dtype=i32),
                pos=z(N * K, dtype=i32), indices=z(N * K, dtype=i32), bins=z(E, dtype=i32),
                padded_bins=z(E, dtype=i32))
    bad = dict(args, W_r=z(E, H))
    with pytest.raises(ValueError, match="W_r"):
        moe.moe_unpermute_router_bwd(**bad)
    with pytest.raises(ValueError, match="probs"):
        moe.moe_unpermute_router_bwd(**args, probs=z(N, E + 1, dtype=f32), aux_alpha=0.01)
    with pytest.raises(ValueError, match="bins"):
        moe.moe_aux_loss(z(N, E, dtype=f32), z(E + 2, dtype=i32), K, 0.01)
    with pytest.raises(TypeError, match="probs"):
        moe.moe_aux_loss(z(N, E), z(E, dtype=i32), K, 0.01)


def test_layer_checks_parameters_and_gradient_buffers():
    layer = moe.MoELayer.__new__(moe.MoELayer)       # no device workspace: the checks come first
    layer.N, layer.H, layer.E, layer.K, layer.F = N, H, E, K, F
    layer.dtype, layer.training = bf, True
    params = [z(N, H), z(H, E), z(E, H, F), z(E, H, F), z(E, F, H)]
    with pytest.raises(ValueError, match="x"):
        layer.forward(z(N - 1, H), *params[1:])
    with pytest.raises(TypeError, match="W1"):
        layer.forward(params[0], params[1], z(E, H, F, dtype=f32), *params[3:])
    with pytest.raises(ValueError, match="y"):
        layer.forward(*params, y=z(N, H + 128))
    grads = {"dx": z(N, H), "dW_r": z(H, E), "dW1": z(E, H, F), "dW3": z(E, H, F), "dW2": z(E, H, F)}
    with pytest.raises(ValueError, match="dW2"):
        layer.backward(z(N, H), *params, grads=grads)
    with pytest.raises(ValueError, match="dy"):
        layer.backward(z(N, H + 128), *params, grads=dict(grads, dW2=z(E, F, H)))
