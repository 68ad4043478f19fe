"""GPU parity of the backward pass (mrlmoe_forward_train + mrlmoe_backward)
against the oracle's fp64 backward on the same seeded inputs.

The oracle differentiates the forward with its rounding points applied (the
readings in its header); the CUDA path rounds the gradients it hands from
one GEMM to the next to bf16 (dc, dg, du, dzx) and keeps g, u as bf16, with
fp32 accumulation everywhere.  Each of those roundings perturbs an element
by at most 2^-9 of itself, and the few of them in series leave the
gradients within a few parts in a thousand of the oracle (measured on B200:
at most 4e-3 in norm, 6e-3 in the largest element, over the cases below);
the bounds BWD_FRO, BWD_MAX allow a factor of about four over that.
"""
import dataclasses

import pytest
import torch

import sparse_moe_layer_mean_b200 as M
import workloads as W
from oracle import mrlmoe_backward as B

pytestmark = pytest.mark.gpu

# ||g - g_ref|| / ||g_ref|| and max|g - g_ref| / max|g_ref| per gradient
BWD_FRO = 1.5e-2
BWD_MAX = 2.5e-2

NAMES = {"dx": "x", "d_w_down": "w_down", "d_w_router": "w_router", "d_w_gate": "w_gate",
         "d_w_up_e": "w_up_e", "d_w_down_e": "w_down_e", "d_w_sh_gate": "w_sh_gate",
         "d_w_sh_up": "w_sh_up", "d_w_sh_down": "w_sh_down", "d_rms_gain": "rms_gain",
         "d_w_up": "w_up", "d_expert_scale": "expert_scale"}


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _weights(s):
    w = dict(W.make_weights(s, "cuda"))
    w["rms_gain"] = W.make_train_gain(s, "cuda")
    return w


def _run(s, seed_bias=7):
    w = _weights(s)
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, 900 + seed_bias, "cuda")
    dy = W.make_dy(s, "cuda")
    layer = M.MRLMoELayer(s, w, train=True)
    r = layer.routing_buffers()
    y = layer.forward_train(x, bias, routing=r)
    grads = layer.backward(x, dy)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return layer, w, x, bias, dy, r, y, grads


def _oracle(s, w, x, bias, dy, experts=None):
    wh = {k: v.cpu() for k, v in w.items()}
    fc = B.forward_for_grad(x.cpu(), wh, bias.cpu(), s.top_k, rms_eps=s.rms_eps, aggregation=s.aggregation,
                            round_points=True)
    return fc, B.backward(fc, wh, dy.cpu(), s.top_k, aggregation=s.aggregation, experts=experts)


EXPERT_GRADS = ("d_w_gate", "d_w_up_e", "d_w_down_e")


def _errors(g, ref):
    g = g.cpu().double()
    d = g - ref
    fro = (d.norm() / ref.norm().clamp_min(1e-300)).item()
    mx = (d.abs().max() / ref.abs().max().clamp_min(1e-300)).item()
    return fro, mx


def _compare(s, grads, ref, fro_tol=BWD_FRO, max_tol=BWD_MAX, experts=None):
    worst = {}
    for name, oname in NAMES.items():
        g = grads[name]
        if experts is not None and name in EXPERT_GRADS:
            g = g[torch.tensor(experts, device=g.device)]
        fro, mx = _errors(g, ref[oname])
        worst[name] = (fro, mx)
    print({k: (f"{a:.2e}", f"{b:.2e}") for k, (a, b) in worst.items()})
    for name, (fro, mx) in worst.items():
        assert fro <= fro_tol and mx <= max_tol, (name, fro, mx)


CASES = [
    ("c0_tiny", 64, "mean"),
    ("c0_tiny", 37, "mean"),    # ragged token tile
    ("c0_tiny", 1, "mean"),     # one token
    ("c0_tiny", 300, "mean"),   # several token tiles; several ragged K blocks per expert
    ("c0_tiny", 64, "sum"),
    ("c0_tiny", 64, "max"),
    ("c2_prefill", 64, "mean"),  # full width: most experts without rows (zero tiles)
]


@pytest.mark.parametrize("config,T,agg", CASES)
def test_backward_matches_oracle(config, T, agg):
    s = dataclasses.replace(W.CONFIGS[config], T=T, aggregation=agg)
    layer, w, x, bias, dy, r, y, grads = _run(s)
    experts = None
    if s.n_experts * s.d_ff * s.d_lat > 1 << 24:
        # full width: the routed experts' weight gradients on a sample of
        # experts with rows and two without (zero gradients)
        idx = r["topk_idx"].cpu().long()
        used = torch.unique(idx).tolist()
        unused = sorted(set(range(s.n_experts)) - set(used))
        experts = used[:6] + unused[:2]
    fc, ref = _oracle(s, w, x, bias, dy, experts)
    # the same experts were selected (the gradient depends on the selection)
    assert torch.equal(r["topk_idx"].cpu().long().view(T, s.top_k), fc.idx)
    _compare(s, grads, ref, experts=experts)


EDGE = [  # (overrides of c0_tiny, T)
    (dict(n_routers=1), 64),                  # one router
    (dict(n_routers=8), 64),                  # eight routers
    (dict(top_k=1), 64),                      # k = 1: w = 1, no router gradient
    (dict(top_k=16), 40),                     # k = E: every expert selected
    (dict(n_experts=64, top_k=17), 50),       # the wide (32-entry) top-k lists
    (dict(n_experts=1024, top_k=4), 200),     # most experts without rows (zero gradient tiles)
]


@pytest.mark.parametrize("over,T", EDGE)
def test_backward_edge_cases(over, T):
    s = dataclasses.replace(W.CONFIGS["c0_tiny"], T=T, **over)
    layer, w, x, bias, dy, r, y, grads = _run(s)
    fc, ref = _oracle(s, w, x, bias, dy)
    assert torch.equal(r["topk_idx"].cpu().long().view(T, s.top_k), fc.idx)
    _compare(s, grads, ref)
    if s.top_k == 1:
        assert float(grads["d_w_router"].abs().max()) < 1e-6 * float(grads["d_w_gate"].abs().max())


def test_training_forward_output_equals_forward():
    s = W.CONFIGS["c0_tiny"].with_T(300)
    w = _weights(s)
    x = W.make_x(s, "cuda")
    bias = torch.zeros(s.n_experts, device="cuda")
    y0 = M.MRLMoELayer(s, w)(x, bias)
    y1 = M.MRLMoELayer(s, w, train=True).forward_train(x, bias)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)


def test_backward_is_deterministic():
    s = W.CONFIGS["c0_tiny"].with_T(300)
    layer, w, x, bias, dy, r, y, g1 = _run(s)
    g1 = {k: v.clone() for k, v in g1.items()}
    layer.forward_train(x, bias)
    g2 = layer.backward(x, dy)
    torch.cuda.synchronize()
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def test_full_width_sampled_rows():
    # full-width prefill-sized tokens: every gradient's shape and finiteness,
    # and the dense input gradient against the oracle on a sample of tokens
    # whose routing the oracle reproduces (dx_t depends on token t only)
    s = W.CONFIGS["c2_prefill"].with_T(1024)
    layer, w, x, bias, dy, r, y, grads = _run(s)
    for name, t in grads.items():
        assert torch.isfinite(t.float()).all(), name
    sample = torch.tensor([0, 1, 2, 511, 777, 1023])
    xs = x[sample].contiguous()
    dys = dy[sample].contiguous()
    ss = s.with_T(len(sample))
    fc, ref = _oracle(ss, w, xs, bias, dys, experts=[])
    assert torch.equal(r["topk_idx"].cpu().long().view(s.T, s.top_k)[sample], fc.idx)
    fro, mx = _errors(grads["dx"][sample.cuda()], ref["x"])
    assert fro <= BWD_FRO and mx <= BWD_MAX, (fro, mx)


def test_backward_rejects_fp8_and_small_workspace():
    s = W.CONFIGS["c0_fp8"]
    cfg = M.make_config(s)
    assert M.mrlmoe_train_workspace_size(cfg) == 0
    s = W.CONFIGS["c0_tiny"]
    layer = M.MRLMoELayer(s, _weights(s))  # sized for the forward only
    x = W.make_x(s, "cuda")
    with pytest.raises(M.MrlmoeError):
        M.mrlmoe_backward(layer.cfg, layer.cw, x, W.make_dy(s, "cuda"), M.make_grads(M.grad_buffers(layer.cfg)),
                          layer.workspace, layer.ws_bytes)


@pytest.mark.parametrize("config,T", [("c0_tiny", 300), ("c2_prefill", 64)])
def test_accumulated_gradients_add_up(config, T):
    # zeroed buffers, two accumulating calls = twice the written gradients,
    # bit for bit (g + g is exact in fp32); dx is overwritten each time
    s = W.CONFIGS[config].with_T(T)
    layer, w, x, bias, dy, r, y, g1 = _run(s)
    g1 = {k: v.clone() for k, v in g1.items()}
    acc = M.grad_buffers(layer.cfg)
    for t in acc.values():
        t.zero_()
    for _ in range(2):
        layer.forward_train(x, bias)
        layer.backward(x, dy, grads=acc, accumulate=True)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(acc["dx"], g1["dx"])
    for k in g1:
        if k != "dx":
            assert torch.equal(acc[k], 2 * g1[k]), k
