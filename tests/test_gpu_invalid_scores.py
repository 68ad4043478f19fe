"""Routing inputs that break the precondition of the routing entry points:
NaN scores (given, or from a NaN token in x) and -inf biases that leave a
token fewer than k selectable experts.

Every such call ends with MRLMOE_ERR_CHECK in the device status word.  The
empty slots read expert -1 and weight 0.  The call's later kernels do nothing
(y is left untouched), no index outside [0, E) is ever used, and the next clean
call on the same workspace equals the oracle.  A -inf bias that still leaves
exactly k selectable experts is valid input and is bit-exact against the
oracle.  None of these cases can fault: each expert index is range-checked
before any kernel uses it.
"""
import pytest
import torch

import oracle as O
import sparse_moe_layer_mean_b200 as M
import workloads as W
from helpers import device_weights

pytestmark = pytest.mark.gpu

OK, CHECK = 0, 6
NAN = float("nan")


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _scores_layer(T, E, k):
    shape = W.LayerShape("t", T=T, d_model=256, d_lat=128, n_experts=E, top_k=k, d_ff=128, n_routers=1)
    alpha = W.uniform((E,), 0.5, 1.5, 3, 300, "cuda")
    w = {"w_router": torch.zeros(1, E, 128, dtype=torch.bfloat16, device="cuda"), "expert_scale": alpha}
    return M.MRLMoELayer(shape, w), alpha


def _route_scores(layer, s, b):
    r = layer.routing_buffers()
    r["scores"] = s.cuda().flatten()
    layer.route(b.cuda(), routing=r, scores_in=True)
    return r


def _assert_matches_oracle(r, s, b, alpha, T, k, rows=None):
    ref = O.forward(None, {"expert_scale": alpha.cpu()}, b.cpu(), k, scores=s.cpu())
    idx = r["topk_idx"].cpu().long().view(T, k)
    w = r["topk_w"].cpu().view(T, k)
    rows = torch.arange(T) if rows is None else rows
    assert torch.equal(idx[rows], ref.topk_idx[rows])
    assert torch.equal(w[rows].view(torch.int32), ref.topk_w[rows].view(torch.int32))
    return ref


@pytest.mark.parametrize("T,E,k", [(64, 16, 2), (1000, 512, 10), (300, 64, 24)])
def test_nan_scores_end_in_check_with_empty_slots(T, E, k):
    layer, alpha = _scores_layer(T, E, k)
    s = W.uniform((T, E), 0.0, 1.0, 41, 200, "cpu")
    b = W.uniform((E,), -0.05, 0.05, 41, 201, "cpu")
    bad = s.clone()
    bad[5] = NAN                               # nothing selectable
    bad[9] = NAN
    bad[9, 3] = 0.5                            # one selectable expert of k
    r = _route_scores(layer, bad, b)
    assert layer.device_status() == CHECK
    idx = r["topk_idx"].cpu().view(T, k)
    w = r["topk_w"].cpu().view(T, k)
    assert idx[5].tolist() == [-1] * k and w[5].tolist() == [0.0] * k
    assert idx[9].tolist() == [3] + [-1] * (k - 1)
    assert w[9].tolist() == [1.0] + [0.0] * (k - 1)
    good = torch.tensor([t for t in range(T) if t not in (5, 9)])
    _assert_matches_oracle(r, bad, b, alpha, T, k, rows=good)   # the top-k kernel still wrote every token
    # the next call on the same workspace is clean and exact
    r = _route_scores(layer, s, b)
    assert layer.device_status() == OK
    ref = _assert_matches_oracle(r, s, b, alpha, T, k)
    assert torch.equal(r["perm"].cpu().long(), ref.perm)


def test_neg_inf_bias_on_too_many_experts_ends_in_check():
    T, E, k = 200, 64, 8
    layer, alpha = _scores_layer(T, E, k)
    s = W.uniform((T, E), 0.0, 1.0, 42, 200, "cpu")
    b = torch.zeros(E)
    b[: E - k + 1] = float("-inf")             # k - 1 selectable experts per token
    r = _route_scores(layer, s, b)
    assert layer.device_status() == CHECK
    idx = r["topk_idx"].cpu().view(T, k)
    assert torch.all(idx[:, -1] == -1) and torch.all(idx[:, :-1] >= E - k + 1)


def test_neg_inf_bias_leaving_exactly_k_experts_is_exact():
    T, E, k = 200, 64, 8
    layer, alpha = _scores_layer(T, E, k)
    s = W.uniform((T, E), 0.0, 1.0, 43, 200, "cpu")
    b = W.uniform((E,), -0.05, 0.05, 43, 201, "cpu")
    b[torch.arange(0, E, 2)[: E - k]] = float("-inf")
    r = _route_scores(layer, s, b)
    assert layer.device_status() == OK
    ref = _assert_matches_oracle(r, s, b, alpha, T, k)
    assert torch.equal(r["counts"].cpu().long(), ref.counts)
    assert torch.equal(r["perm"].cpu().long(), ref.perm)


def test_nan_token_in_x_fails_the_forward_and_writes_nothing():
    s = W.CONFIGS["c0_tiny"]
    x = W.make_x(s, "cuda")
    bias = torch.zeros(s.n_experts, device="cuda")
    layer = M.MRLMoELayer(s, device_weights("c0_tiny"))
    y_ok = layer(x, bias)
    assert layer.device_status() == OK
    xb = x.clone()
    xb[3] = NAN
    y_bad = torch.zeros_like(y_ok)
    layer(xb, bias, y=y_bad)
    assert layer.device_status() == CHECK
    assert torch.all(y_bad == 0)               # the kernels after the router did nothing
    y_again = layer(x, bias)
    assert layer.device_status() == OK
    assert torch.equal(y_again, y_ok)


@pytest.mark.parametrize("T", [1152, 1153])
def test_nan_token_through_both_router_forms(T):
    # full-width routing: T = 1152 takes the K-split router and the top-k
    # kernel, T = 1153 the router GEMM's top-k epilogue and the merge
    s = W.LayerShape("split", T=T, d_model=256, d_lat=128, n_experts=512, top_k=10, d_ff=128, n_routers=4)
    w = W.make_routing_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.02, 0.02, 3, 940, "cuda")
    layer = M.MRLMoELayer(s, w)
    xb = x.clone()
    xb[7] = NAN
    r = layer.route(bias, x=xb)
    assert layer.device_status() == CHECK
    assert r["topk_idx"].view(T, s.top_k)[7].tolist() == [-1] * s.top_k
    r = layer.route(bias, x=x)
    assert layer.device_status() == OK
    assert bool(((r["topk_idx"] >= 0) & (r["topk_idx"] < s.n_experts)).all())


def test_static_entry_point_nan_scores_reported_by_the_checker():
    T, E, k = 64, 16, 2
    shape = W.LayerShape("t", T=T, d_model=256, d_lat=128, n_experts=E, top_k=k, d_ff=128, n_routers=1)
    cfg = M.make_config(shape)
    s = W.uniform((T, E), 0.0, 1.0, 44, 200, "cuda")
    b = W.uniform((E,), -0.05, 0.05, 44, 201, "cuda")
    alpha = W.uniform((E,), 0.5, 1.5, 44, 202, "cuda")
    i32 = dict(dtype=torch.int32, device="cuda")

    def call(scores):
        r = {"topk_idx": torch.empty(T * k, **i32), "topk_w": torch.empty(T * k, dtype=torch.float32, device="cuda"),
             "counts": torch.zeros(E, **i32), "offsets": torch.zeros(E + 1, **i32),
             "perm": torch.zeros(T * k, **i32), "inv_perm": torch.zeros(T * k, **i32),
             "scores": scores.flatten()}
        M.mrlmoe_route_scores_static(cfg, b, alpha, M.make_routing(r))
        ws = torch.empty(256, dtype=torch.uint8, device="cuda")
        M.mrlmoe_check_routing(cfg, M.make_routing(r), ws, 256, True)
        return r, M.mrlmoe_get_device_detail(ws)

    bad = s.clone()
    bad[11] = NAN
    r, (status, bits) = call(bad)
    assert status == CHECK and bits & 1       # MRLMOE_CHECK_INDEX: the -1 slots
    assert r["topk_idx"].view(T, k)[11].tolist() == [-1, -1]
    r, (status, bits) = call(s)
    assert (status, bits) == (OK, 0)
    ref = O.forward(None, {"expert_scale": alpha.cpu()}, b.cpu(), k, scores=s.cpu())
    assert torch.equal(r["perm"].cpu().long(), ref.perm)
