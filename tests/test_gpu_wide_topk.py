"""Top-k beyond 16 experts per token (16 < k <= 32, the longer running lists)
on the GPU against the oracle: routing from x through the router GEMM with
the expert range split over CTAs and merged (T large enough that the K range
is not split), routing from x through the K-split router (small T), and the
whole tiny layer at k = 32.  Scores-in routing at k = 17, 24, 32 is bit-exact
in test_gpu_parity."""
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


@pytest.mark.parametrize("T,k", [(1280, 24), (1280, 32), (200, 32), (200, 20)])
def test_route_from_x_wide_k(T, k):
    # E = 512, R = 4: 8 expert chunks; T = 1280 gives 10 token tiles (router
    # over expert chunks + merge), T = 200 two tiles (K-split router)
    s = W.LayerShape("wide", T=T, d_model=256, d_lat=128, n_experts=512, top_k=k, d_ff=128, n_routers=4)
    w = W.make_routing_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.02, 0.02, 3, 930, "cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=True)
    layer.route(bias, x=x, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    zx = x.cpu().double() @ w["w_down"].cpu().double().T
    s_ref = O.router_scores(zx, w["w_router"].cpu())
    sg = r["scores"].view(T, s.n_experts).cpu().double()
    assert (sg - s_ref.double()).abs().max().item() < 1e-5
    bad, gaps, _ = routing_audit(r["topk_idx"].view(-1, k), s_ref, bias, k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    check_dispatch_properties(r, T, s.n_experts, k)
    good = torch.ones(T, dtype=torch.bool)
    good[bad] = False
    wg = r["topk_w"].view(T, k).cpu().double()[good]
    assert (wg.sum(1) - 1).abs().max().item() < 1e-5
    layer.check_routing(r, clear=True)
    assert layer.device_detail() == (0, 0)


def test_forward_tiny_layer_k32():
    s = W.LayerShape("k32", T=96, d_model=256, d_lat=128, n_experts=48, top_k=32, d_ff=128, n_routers=2)
    w = W.make_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, 931, "cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers()
    y = layer(x, bias, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    ref = O.forward(x.cpu(), {n: v.cpu() for n, v in w.items()}, bias.cpu(), s.top_k, s.rms_eps)
    bad, gaps, _ = routing_audit(r["topk_idx"].view(-1, s.top_k), ref.s, bias, s.top_k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    keep = torch.ones(s.T, dtype=torch.bool)
    keep[bad] = False
    mx, mean = rel_errors(y.cpu()[keep], ref.y[keep])
    assert mx <= BF16_MAX_REL and mean <= BF16_MEAN_REL, (mx, mean)


@pytest.mark.parametrize("T,R,k,agg", [(2500, 4, 10, "mean"), (2600, 4, 24, "mean"), (2401, 3, 10, "sum"),
                                       (9300, 1, 10, "mean"), (1300, 8, 10, "max"), (1300, 8, 32, "sum")])
def test_route_from_x_larger_T(T, R, k, agg):
    # token counts above the K-split router's range: the router walks its
    # expert chunks per token tile and the partial lists are merged; ragged
    # last tiles, odd R, R = 1 (two chunks of 256 experts), R = 8, wide k
    import dataclasses
    s = dataclasses.replace(W.LayerShape("pair", T=T, d_model=256, d_lat=256, n_experts=512, top_k=k, d_ff=128,
                                         n_routers=R), aggregation=agg)
    w = W.make_routing_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.02, 0.02, 3, 960, "cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=True)
    layer.route(bias, x=x, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    zx = x.cpu().double() @ w["w_down"].cpu().double().T
    s_ref = O.router_scores(zx, w["w_router"].cpu(), agg)
    sg = r["scores"].view(T, s.n_experts).cpu().double()
    assert (sg - s_ref.double()).abs().max().item() < 1e-5 * (R if agg == "sum" else 1)
    bad, gaps, _ = routing_audit(r["topk_idx"].view(-1, k), s_ref, bias, k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    check_dispatch_properties(r, T, s.n_experts, k)
    good = torch.ones(T, dtype=torch.bool)
    good[bad] = False
    wg = r["topk_w"].view(T, k).cpu().double()[good]
    assert (wg.sum(1) - 1).abs().max().item() < 1e-5
