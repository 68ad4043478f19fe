"""mrlmoe_route_scores_static: routing without a caller workspace.

Some callers cannot call cudaMalloc at all: code embedded in a host framework
that owns every device allocation, or work recorded into a pre-planned graph
whose buffers are fixed up front.  For them the library offers one entry
point whose scratch is a static device array inside the library.  These tests
call it through the C ABI and compare it with the workspace entry point
(mrlmoe_route with caller-given scores) on the same inputs, two calls in a
row; the routing record is integer and index data plus the same fp32
arithmetic, so the comparison is bit-exact.

The file name sorts last so a run that stops at the first failure has
already run every other test.
"""
import pytest
import torch

import sparse_moe_layer_mean_b200 as M
import workloads as W

pytestmark = pytest.mark.gpu


def _case(T, E, k, seed):
    s = W.uniform((T, E), 0.0, 1.0, seed, 700, "cuda")
    b = W.uniform((E,), -0.05, 0.05, seed, 701, "cuda")
    alpha = W.uniform((E,), 0.5, 1.5, seed, 702, "cuda")
    return s.contiguous(), b, alpha


def _shape(T, E, k):
    return W.LayerShape("t", T=T, d_model=256, d_lat=128, n_experts=E, top_k=k, d_ff=128, n_routers=1)


def _with_workspace(shape, s, b, alpha):
    w = {"w_router": torch.zeros(1, shape.n_experts, 128, dtype=torch.bfloat16, device="cuda"),
         "expert_scale": alpha}
    layer = M.MRLMoELayer(shape, w)
    r = layer.routing_buffers()
    r["scores"] = s.flatten()
    layer.route(b, routing=r, scores_in=True)
    return r


def _record(T, E, k):
    i32 = dict(dtype=torch.int32, device="cuda")
    return {"topk_idx": torch.empty(T * k, **i32),
            "topk_w": torch.empty(T * k, dtype=torch.float32, device="cuda"),
            "counts": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
            "perm": torch.empty(T * k, **i32), "inv_perm": torch.empty(T * k, **i32)}


def _static(shape, s, b, alpha):
    cfg = M.make_config(shape)
    r = _record(shape.T, shape.n_experts, shape.top_k)
    r["scores"] = s.flatten()
    M.mrlmoe_route_scores_static(cfg, b, alpha, M.make_routing(r))
    return r


FIELDS = ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm")


def _same(a, b):
    for f in FIELDS:
        assert torch.equal(a[f].view(torch.int32), b[f].view(torch.int32)), f


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_static_scratch_matches_workspace_route_two_calls():
    # first call (sets the array up), second call on other inputs and shapes:
    # the array keeps the first call's contents, which must not leak
    for (T, E, k, seed) in [(1000, 512, 10, 1), (64, 16, 2, 2), (1000, 512, 10, 3)]:
        shape = _shape(T, E, k)
        s, b, alpha = _case(T, E, k, seed)
        ref = _with_workspace(shape, s, b, alpha)
        got = _static(shape, s, b, alpha)
        torch.cuda.synchronize()
        _same(got, ref)


def test_static_scratch_repeated_on_one_stream():
    shape = _shape(2048, 512, 10)
    s, b, alpha = _case(2048, 512, 10, 4)
    ref = _with_workspace(shape, s, b, alpha)
    first = _static(shape, s, b, alpha)
    second = _static(shape, s, b, alpha)
    torch.cuda.synchronize()
    _same(first, ref)
    _same(second, ref)


def test_static_scratch_rejects_oversized_problem():
    shape = _shape(65536, 1024, 16)          # needs far more than the built-in scratch
    cfg = M.make_config(shape)
    s = torch.zeros(16, device="cuda")
    r = {f: s for f in FIELDS}
    r["scores"] = s
    with pytest.raises(M.MrlmoeError) as ei:
        M.mrlmoe_route_scores_static(cfg, s, s, M.make_routing(r))
    assert ei.value.code == 7
