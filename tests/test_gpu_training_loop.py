"""A training loop through the C ABI: forward_train, the loss gradient, the
backward, an SGD step on fp32 master weights (their bf16 copies are what the
layer reads) and the balancing-bias update from the step's expert counts.
The loss falls at every step and follows the oracle's loop
(helpers.train_loop_oracle, same teacher target, learning rate and
bias step) to within the drift that bf16 gradients accumulate."""
import pytest
import torch

import sparse_moe_layer_mean_b200 as M
import workloads as W
from oracle import mrlmoe_backward as B
from helpers import train_loop_oracle

pytestmark = pytest.mark.gpu

LR, GAMMA, STEPS = 7.8125e-4, 1e-3, 12


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_training_loop_lowers_the_loss_and_follows_the_oracle():
    s = W.CONFIGS["c0_tiny"]
    master = {k: v.float() for k, v in W.make_weights(s, "cuda").items()}
    w = {k: (v.to(torch.bfloat16) if v.dim() > 1 else v.clone()) for k, v in master.items()}
    teacher = {k: v.to(torch.bfloat16) if v.dim() > 1 else v.float()
               for k, v in W.make_weights(s, "cpu", seed=5).items()}
    x = W.make_x(s, "cuda")
    bias = torch.zeros(s.n_experts, device="cuda")
    target = B.forward_for_grad(x.cpu(), teacher, bias.cpu(), s.top_k).y.to("cuda")
    layer = M.MRLMoELayer(s, w, train=True)
    r = layer.routing_buffers()
    losses = []
    for _ in range(STEPS):
        y = layer.forward_train(x, bias, routing=r)
        d = y.double() - target
        losses.append(0.5 * float((d * d).mean()))
        g = layer.backward(x, d.to(torch.bfloat16))
        M.mrlmoe_bias_update(layer.cfg, r["counts"], bias, GAMMA)
        for k in master:
            master[k] -= LR * g["d_" + k]
            w[k].copy_(master[k])          # in place: the layer keeps its pointers
        assert layer.device_status() == 0
    ref = train_loop_oracle(STEPS, LR, GAMMA)
    print([f"{a:.4f}/{b:.4f}" for a, b in zip(losses, ref)])
    assert all(b < a for a, b in zip(losses, losses[1:])), losses
    assert losses[-1] < 0.2 * losses[0], losses
    for a, b in zip(losses, ref):
        assert abs(a - b) <= 0.05 * b, (losses, ref)
