"""The forward recorded into a CUDA graph (stream capture) and replayed
gives the same output as the eager call, bit for bit: the library's host
side allocates nothing and synchronises nothing on the stream, so a caller
can capture it (after one eager call, which configures the kernels)."""
import pytest
import torch

import sparse_moe_layer_mean_b200 as M
import workloads as W
from helpers import device_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name,T", [("c0_tiny", 64), ("c0_fp8", 200), ("c2_prefill", 256)])
def test_forward_in_cuda_graph_matches_eager(name, T):
    s = W.CONFIGS[name].with_T(T)
    w = device_weights(name)
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 2, 920, "cuda")
    layer = M.MRLMoELayer(s, w)
    y_eager = layer(x, bias)
    torch.cuda.synchronize()
    y = torch.empty_like(y_eager)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        layer(x, bias, y=y, stream=torch.cuda.current_stream())
    for _ in range(2):
        y.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))


@pytest.mark.parametrize("name,T", [("c0_tiny", 300), ("c2_prefill", 256)])
def test_training_step_in_cuda_graph_matches_eager(name, T):
    # forward_train + backward recorded together (the backward's status and
    # hold-byte writes are memsets, its tensor maps are built on the host)
    s = W.CONFIGS[name].with_T(T)
    w = device_weights(name)
    x = W.make_x(s, "cuda")
    dy = W.make_dy(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 2, 920, "cuda")
    layer = M.MRLMoELayer(s, w, train=True)
    layer.forward_train(x, bias)
    ref = {k: v.clone() for k, v in layer.backward(x, dy).items()}
    torch.cuda.synchronize()
    grads = M.grad_buffers(layer.cfg)
    y = torch.empty(T, s.d_model, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        cur = torch.cuda.current_stream()
        layer.forward_train(x, bias, y=y, stream=cur)
        layer.backward(x, dy, grads=grads, stream=cur)
    for _ in range(2):
        for t in grads.values():
            t.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    for k in ref:
        assert torch.equal(grads[k], ref[k]), k
