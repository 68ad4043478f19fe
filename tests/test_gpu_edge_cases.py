"""Edge cases of the layer on the GPU against the oracle: the largest expert
count, top-k and router count the library accepts, degenerate routing (every
token on the same experts: one group holds all rows, the rest are empty), a
single token at full width, and an all-zero input (every score ties, so the
lower-index rule decides the whole selection)."""
import dataclasses

import pytest
import torch

import oracle as O
import sparse_moe_layer_mean_b200 as M
import workloads as W
from helpers import (BF16_MAX_REL, BF16_MEAN_REL, GAP_TOL, check_dispatch_properties, host_weights,
                     device_weights, rel_errors, routing_audit)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _forward(s, w, x, bias):
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers()
    y = layer(x, bias, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return y, r


def _check(s, x, bias, y, r, wh, tokens=None):
    xs = x.cpu() if tokens is None else x.cpu()[tokens]
    ref = O.forward(xs, wh, bias.cpu(), s.top_k, s.rms_eps, aggregation=s.aggregation)
    gidx = r["topk_idx"].view(-1, s.top_k)
    if tokens is not None:
        gidx = gidx[tokens.to(gidx.device)]
    bad, gaps, _ = routing_audit(gidx, ref.s, bias, s.top_k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    keep = torch.ones(xs.shape[0], dtype=torch.bool)
    keep[bad] = False
    yg = y.cpu() if tokens is None else y.cpu()[tokens]
    mx, mean = rel_errors(yg[keep], ref.y[keep])
    assert mx <= BF16_MAX_REL and mean <= BF16_MEAN_REL, (mx, mean)
    return ref


def test_largest_expert_count_topk_and_router_count():
    # E = 1024 (the group tables' limit), k = 16, R = 8; narrow hidden sizes
    # keep the oracle cheap; d_lat 256 takes the CTA-pair down GEMM
    s = W.LayerShape("edge_max", T=300, d_model=256, d_lat=256, n_experts=1024, top_k=16, d_ff=128,
                     n_routers=8)
    w = W.make_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, 910, "cuda")
    y, r = _forward(s, w, x, bias)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    assert int((r["counts"] == 0).sum()) > 0          # some of the 1024 groups are empty
    _check(s, x, bias, y, r, {k: v.cpu() for k, v in w.items()})


@pytest.mark.parametrize("T", [1000, 17])
def test_every_token_on_the_same_experts(T):
    # a bias that dwarfs the scores sends every token to experts 3 and 11:
    # two groups of T rows (several token tiles), fourteen empty groups
    s = W.CONFIGS["c0_tiny"].with_T(T)
    w = device_weights("c0_tiny")
    x = W.make_x(s, "cuda")
    bias = torch.zeros(s.n_experts, dtype=torch.float32, device="cuda")
    bias[3] = 10.0
    bias[11] = 10.0
    y, r = _forward(s, w, x, bias)
    counts = r["counts"].cpu()
    assert int(counts[3]) == T and int(counts[11]) == T and int(counts.sum()) == 2 * T
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    _check(s, x, bias, y, r, host_weights("c0_tiny"))


def test_full_width_all_tokens_on_ten_experts():
    s = W.CONFIGS["c2_prefill"].with_T(300)
    w = device_weights("c2_prefill")
    x = W.make_x(s, "cuda")
    bias = torch.zeros(s.n_experts, dtype=torch.float32, device="cuda")
    hot = torch.tensor([0, 5, 77, 128, 255, 256, 300, 401, 510, 511])
    bias[hot.cuda()] = 10.0
    y, r = _forward(s, w, x, bias)
    counts = r["counts"].cpu()
    assert torch.all(counts[hot] == s.T) and int(counts.sum()) == s.T * s.top_k
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    _check(s, x, bias, y, r, host_weights("c2_prefill"), tokens=torch.tensor([0, 1, 150, 299]))


def test_single_token_full_width():
    s = W.CONFIGS["c2_prefill"].with_T(1)
    w = device_weights("c2_prefill")
    x = W.make_x(s, "cuda")
    bias = torch.zeros(s.n_experts, dtype=torch.float32, device="cuda")
    y, r = _forward(s, w, x, bias)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    _check(s, x, bias, y, r, host_weights("c2_prefill"))


def test_all_zero_input():
    # x = 0: every logit is 0, every score 1/2, so the selection is experts
    # 0..k-1 by the lower-index rule, the weights are 1/k, h = SiLU(0) * 0 = 0
    # and y = 0 exactly
    s = W.CONFIGS["c0_tiny"]
    w = device_weights("c0_tiny")
    x = torch.zeros(s.T, s.d_model, dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(s.n_experts, dtype=torch.float32, device="cuda")
    y, r = _forward(s, w, x, bias)
    idx = r["topk_idx"].view(s.T, s.top_k).cpu()
    assert torch.equal(idx, torch.arange(s.top_k, dtype=torch.int32).expand(s.T, s.top_k))
    assert torch.all(r["topk_w"].cpu() == 1.0 / s.top_k)
    assert torch.all(y.cpu().float() == 0)
    ref = O.forward(x.cpu(), host_weights("c0_tiny"), bias.cpu(), s.top_k, s.rms_eps)
    assert torch.equal(ref.topk_idx, idx.long()) and torch.all(ref.y == 0)
