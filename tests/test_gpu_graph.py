"""The layer step inside a CUDA graph (GPU only).

Every entry point is asynchronous on its stream, allocates nothing and never
synchronises the host, so a training step (forward + backward) can be
captured once and replayed.  Kernel attributes are set on the first (eager)
call; the captured calls only launch.  Replays must reproduce the eager step
bit for bit.
"""
import pytest
import torch

import dropless_top_moe_b200 as moe
from tests._cases import make_case, small_shape

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [small_shape("graph_bf16", N=1000, H=256, E=16, K=4, F=256, training=True),
                                   small_shape("graph_f32", N=300, H=64, E=4, K=2, F=96, dtype="f32",
                                               training=True)], ids=lambda s: s.name)
def test_layer_step_replays_from_a_cuda_graph(shape):
    c = make_case(shape, seed=61, with_dy=True)
    layer = moe.MoELayer(shape.N, shape.H, shape.E, shape.K, shape.F, dtype=shape.torch_dtype, training=True)
    grads = layer.grad_buffers()

    def step():
        layer.forward(c["x"], c["W_r"], c["W1"], c["W3"], c["W2"])
        layer.backward(c["dy"], c["x"], c["W_r"], c["W1"], c["W3"], c["W2"], grads)

    step()                                  # eager: first-call set-up happens here
    torch.cuda.synchronize()
    assert layer.status() == 0
    y0 = layer.y.clone()
    g0 = {k: v.clone() for k, v in grads.items()}

    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        layer.y.zero_()
        for v in grads.values():
            v.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert layer.status() == 0
        assert torch.equal(layer.y, y0)
        for k in grads:
            assert torch.equal(grads[k], g0[k]), k
