"""Router score aggregation (mean / sum / max) and the number of routers R,
on the GPU against the oracle.

The pages say several independently initialised sigmoid routers are
aggregated, without the rule or R (aitest123, "模型结构"; derekhsu,
"多路由潛在 MoE"); the layer reads the mean with R = 4.  These tests sweep the
alternatives through the same kernels: the whole tiny layer, and routing from
x alone at full width (512 experts, top-10, where the router splits the
expert range over CTAs and merges partial top-k lists).
"""
import dataclasses

import pytest
import torch

import oracle as O
import sparse_moe_layer_mean_b200 as M
import workloads as W
from helpers import (BF16_MAX_REL, BF16_MEAN_REL, GAP_TOL, check_dispatch_properties, rel_errors,
                     routing_audit)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _score_tol(agg: str, R: int) -> float:
    # the routers read the fp32 latent, so one router's score differs from the
    # oracle's only by the tensor core's accumulation of 2*L products in its
    # logit, times the sigmoid's slope (<= 1/4): bounded by 1e-5 per router,
    # the same bound as the routing-gap rule.  The mean and the max of R
    # scores keep that bound; the sum carries R of them.
    return 1e-5 * (R if agg == "sum" else 1)


@pytest.mark.parametrize("agg", ["mean", "sum", "max"])
@pytest.mark.parametrize("R", [1, 3, 8])
def test_forward_c0_aggregation_and_router_count(agg, R):
    s = dataclasses.replace(W.CONFIGS["c0_tiny"], n_routers=R, aggregation=agg)
    w = W.make_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = torch.zeros(s.n_experts, dtype=torch.float32, device="cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=True)
    y = layer(x, bias, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    wh = {k: v.cpu() for k, v in w.items()}
    ref = O.forward(x.cpu(), wh, bias.cpu(), s.top_k, s.rms_eps, aggregation=agg)
    sg = r["scores"].view(s.T, s.n_experts).cpu().double()
    assert (sg - ref.s.double()).abs().max().item() < _score_tol(agg, R)
    bad, gaps, _ = routing_audit(r["topk_idx"].view(-1, s.top_k), ref.s, bias, s.top_k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    keep = torch.ones(s.T, dtype=torch.bool)
    keep[bad] = False
    mx, mean = rel_errors(y.cpu()[keep], ref.y[keep])
    assert mx <= BF16_MAX_REL and mean <= BF16_MEAN_REL, (mx, mean)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)


@pytest.mark.parametrize("agg,R", [("mean", 4), ("sum", 4), ("max", 4), ("mean", 1), ("max", 8), ("sum", 3)])
def test_route_full_width_aggregation_and_router_count(agg, R):
    s = dataclasses.replace(W.CONFIGS["c2_prefill"], T=256, n_routers=R, aggregation=agg)
    w = W.make_routing_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.02, 0.02, 3, 900, "cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=True)
    layer.route(bias, x=x, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    zx = x.cpu().double() @ w["w_down"].cpu().double().T      # the routers read the unrounded latent
    s_ref = O.router_scores(zx, w["w_router"].cpu(), agg)
    sg = r["scores"].view(s.T, s.n_experts).cpu().double()
    assert (sg - s_ref.double()).abs().max().item() < _score_tol(agg, R)
    bad, gaps, ref_idx = routing_audit(r["topk_idx"].view(-1, s.top_k), s_ref, bias, s.top_k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    # weights: renormalised unbiased scores of the selected experts (before alpha)
    good = torch.ones(s.T, dtype=torch.bool)
    good[bad] = False
    wg = r["topk_w"].view(s.T, s.top_k).cpu().double()[good]
    assert (wg.sum(1) - 1).abs().max().item() < 1e-5
