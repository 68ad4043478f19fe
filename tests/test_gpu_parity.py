"""Parity of the CUDA path (through the C ABI) with the CPU oracle."""
import pytest
import torch

import oracle as O
import workloads as W
import sparse_moe_layer_mean_b200 as M
from helpers import (BF16_MAX_REL, BF16_MEAN_REL, FP8_MAX_REL, FP8_MEAN_REL, GAP_TOL,
                     check_dispatch_properties, hard_tokens,
                     device_weights, host_weights, rel_errors, routing_audit)

pytestmark = pytest.mark.gpu


def _require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.fixture(autouse=True)
def _gpu():
    _require_gpu()
    yield


# ------------------------------------------------------------------ linear
@pytest.mark.parametrize("M_,N_,K_", [(1, 128, 128), (127, 256, 256), (129, 384, 640),
                                      (300, 2048, 4096), (1000, 4096, 2048),
                                      # CTA-pair tiles: a ragged 256-row M tile, a 128-wide last N tile
                                      (8229, 384, 256), (2100, 2048, 4096)])
def test_linear_matches_oracle(M_, N_, K_):
    a = W.normal((M_, K_), 7, 100, "cuda")
    w = W.normal((N_, K_), 7, 101, "cuda", std=K_ ** -0.5)
    out = torch.empty(M_, N_, dtype=torch.bfloat16, device="cuda")
    M.mrlmoe_linear(a, w, out, M_, N_, K_)
    torch.cuda.synchronize()
    ref = O.linear_bf16(a.cpu(), w.cpu())
    d = (out.cpu().double() - ref).abs()
    # bf16 output rounding (one step) plus fp32 accumulation error, which is
    # bounded by the sum of |products|, not by |result|
    acc = (a.cpu().double().abs() @ w.cpu().double().abs().T) * 2 ** -16
    bad = d > ref.abs() * 2 ** -7 + acc
    assert not bool(bad.any()), (int(bad.sum()), d[bad][:5], ref[bad][:5])
    assert (d.sum() / ref.abs().sum()).item() < 1e-3


# ------------------------------------------------- routing: scores given
def _scores_case(name, T, E, k):
    if name == "uniform":
        s = W.uniform((T, E), 0.0, 1.0, 11, 200, "cpu")
        b = W.uniform((E,), -0.05, 0.05, 11, 201, "cpu")
    elif name == "dyadic_ties":
        s = (W.uniform((T, E), 0.0, 8.0, 12, 200, "cpu").floor() / 8).float()
        b = (W.uniform((E,), -2.0, 2.0, 12, 201, "cpu").floor() / 16).float()
    elif name == "all_equal":
        s = torch.full((T, E), 0.5)
        b = torch.zeros(E)
    elif name == "signed_zeros":
        u = W.uniform((T, E), 0.0, 3.0, 13, 200, "cpu").floor()
        s = torch.where(u == 0, torch.tensor(0.0), torch.where(u == 1, torch.tensor(-0.0), torch.tensor(-1.0)))
        s[:, E // 2] = 0.75          # a positive selected score keeps the weights finite
        b = torch.zeros(E)
    elif name == "all_zero":
        # every selected score 0: the weights are the uniform fp32(1/k)
        s = torch.zeros(T, E)
        b = W.uniform((E,), -0.05, 0.05, 14, 201, "cpu")
    elif name == "zipf_skew":
        # the skewed workload's Zipf(1.1) selection bias on uniform scores
        s = W.uniform((T, E), 0.0, 1.0, 15, 200, "cpu")
        b = W.make_bias(W.CONFIGS["c3_skew"], "cpu")
    return s.float().contiguous(), b.float().contiguous()


def _route_scores_in_and_compare(T, E, k, s, b):
    shape = W.LayerShape("t", T=T, d_model=256, d_lat=128, n_experts=E, top_k=k, d_ff=128, n_routers=1)
    alpha = W.uniform((E,), 0.5, 1.5, 3, 300, "cpu")
    dev = "cuda"
    w = {"w_router": torch.zeros(1, E, 128, dtype=torch.bfloat16, device=dev),
         "expert_scale": alpha.to(dev)}
    layer = M.MRLMoELayer(shape, w)
    r = layer.routing_buffers(scores=False)
    r["scores"] = s.to(dev).flatten()
    layer.route(b.to(dev), routing=r, scores_in=True)
    torch.cuda.synchronize()
    ref = O.forward(None, {"expert_scale": alpha}, b, k, scores=s)
    assert torch.equal(r["topk_idx"].cpu().long().view(T, k), ref.topk_idx)
    assert torch.equal(r["topk_w"].cpu().view(T, k).view(torch.int32), ref.topk_w.view(torch.int32))
    assert torch.equal(r["counts"].cpu().long(), ref.counts)
    assert torch.equal(r["offsets"].cpu().long(), ref.offsets)
    assert torch.equal(r["perm"].cpu().long(), ref.perm)
    assert torch.equal(r["inv_perm"].cpu().long(), ref.inv_perm)
    assert layer.device_status() == 0
    return ref


@pytest.mark.parametrize("case", ["uniform", "dyadic_ties", "all_equal", "signed_zeros", "all_zero"])
@pytest.mark.parametrize("T,E,k", [(64, 16, 2), (1, 16, 2), (33, 512, 10), (1000, 512, 10),
                                   (257, 1024, 16), (513, 512, 17), (300, 64, 24), (77, 32, 32)])
def test_route_scores_in_bit_exact(case, T, E, k):
    s, b = _scores_case(case, T, E, k)
    _route_scores_in_and_compare(T, E, k, s, b)


@pytest.mark.parametrize("case,T", [("uniform", 8192), ("dyadic_ties", 8192), ("uniform", 16384),
                                    ("zipf_skew", 32768), ("dyadic_ties", 32768)])
def test_route_scores_in_bit_exact_full_size(case, T):
    # the workloads' token counts with 512 experts, top-10: 256 to 1024 token
    # chunks per expert column, so the column scan runs 8 to 32 chunks per warp
    s, b = _scores_case(case, T, 512, 10)
    ref = _route_scores_in_and_compare(T, 512, 10, s, b)
    if case == "zipf_skew":
        counts = ref.counts.double()
        assert counts.max() / counts.mean() > 10.0       # skewed loads really reached the scan


# ------------------------------------------------------- full layer, tiny
def _run_layer(name, T=None, x=None, bias=None, seed=0, scores=True):
    s = W.CONFIGS[name] if T is None else W.CONFIGS[name].with_T(T)
    w = device_weights(name, seed)
    if x is None:
        x = W.make_x(s, "cuda", seed=seed)
    if bias is None:
        bias = torch.zeros(s.n_experts, dtype=torch.float32, device="cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=scores)
    y = layer(x, bias, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return s, x, bias, y, r, layer


def _compare_layer(s, x, bias, y, r, wh, tokens=None):
    """Oracle on the given tokens; output parity on tokens routed alike."""
    xs = x.cpu() if tokens is None else x.cpu()[tokens]
    ref = O.forward(xs, wh, bias.cpu(), s.top_k, s.rms_eps)
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
    if "scores" in r:
        sg = r["scores"].view(-1, s.n_experts).cpu()
        if tokens is not None:
            sg = sg[tokens]
        # routers read the fp32 latent (bf16 hi + lo): only accumulation-order noise remains
        assert (sg.double() - ref.s.double()).abs().max().item() < 5e-6
    return ref, bad


def test_forward_c0_tiny():
    s, x, bias, y, r, _ = _run_layer("c0_tiny")
    ref, bad = _compare_layer(s, x, bias, y, r, host_weights("c0_tiny"))
    assert bad.numel() == 0
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    assert torch.equal(r["counts"].cpu().long(), ref.counts)
    assert torch.equal(r["perm"].cpu().long(), ref.perm)
    g = r["topk_w"].view(-1, s.top_k).cpu().double()
    assert (g - ref.topk_w.double()).abs().max().item() < 1e-6


@pytest.mark.parametrize("T", [1, 31, 200])
def test_forward_c0_ragged_T(T):
    s, x, bias, y, r, _ = _run_layer("c0_tiny", T=T)
    _compare_layer(s, x, bias, y, r, host_weights("c0_tiny"))


def test_forward_c0_with_bias():
    s = W.CONFIGS["c0_tiny"]
    bias = W.uniform((s.n_experts,), -0.1, 0.1, 5, 400, "cuda")
    s, x, bias, y, r, _ = _run_layer("c0_tiny", bias=bias)
    _compare_layer(s, x, bias, y, r, host_weights("c0_tiny"))


def test_forward_deterministic():
    s, x, bias, y1, r1, layer = _run_layer("c0_tiny", T=200)
    y2 = layer(x, bias)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


# -------------------------------------------------- full layer, full width
def test_forward_full_width_ragged():
    s, x, bias, y, r, _ = _run_layer("c2_prefill", T=300)
    _compare_layer(s, x, bias, y, r, host_weights("c2_prefill"))
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)


def test_forward_c2_sampled_tokens():
    s, x, bias, y, r, _ = _run_layer("c2_prefill")
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    tokens = hard_tokens(r, s.T, s.n_experts, s.top_k, want=64, seed=2)
    assert tokens.numel() >= 64
    _compare_layer(s, x, bias, y, r, host_weights("c2_prefill"), tokens=tokens)


def test_forward_c1_decode():
    s, x, bias, y, r, _ = _run_layer("c1_decode")
    _compare_layer(s, x, bias, y, r, host_weights("c2_prefill"))


# ---------------------------------------------------------------- bias
def test_bias_update_bit_exact():
    shape = W.CONFIGS["c3_skew"]
    E, T, k = shape.n_experts, shape.T, shape.top_k
    counts = (W.uniform((E,), 0, 1300, 9, 500, "cpu").floor()).to(torch.int32)
    counts[:5] = T * k // E                                                   # exact mean load
    bias = W.uniform((E,), -0.3, 0.3, 9, 501, "cpu")
    bias[5] = -0.0
    cfg = M.make_config(shape)
    b_dev = bias.cuda()
    M.mrlmoe_bias_update(cfg, counts.cuda(), b_dev, 1e-3)
    torch.cuda.synchronize()
    ref = O.bias_update(bias, counts, T, k, 1e-3)
    assert torch.equal(b_dev.cpu().view(torch.int32), ref.view(torch.int32))


def test_forward_c3_skew_sampled_tokens_and_bias_update():
    s = W.CONFIGS["c3_skew"]
    bias = W.make_bias(s, "cuda")
    s, x, bias, y, r, layer = _run_layer("c3_skew", bias=bias, scores=False)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    counts = r["counts"].cpu().long()
    ratio = (counts.max().double() / counts.double().mean()).item()
    assert 20.0 < ratio < 45.0, ratio          # Zipf(1.1) skew, fitted to ~30x on the oracle
    # the busiest expert (~30x the mean load) spans many token tiles: its first,
    # middle and ragged last tile, both halves of a pair's tile, and the cold
    # experts' small groups (groups of 1-16 rows at full width are also the
    # bulk of the T = 300 case, compared on every token)
    tokens = hard_tokens(r, s.T, s.n_experts, s.top_k, want=80, seed=3)
    assert tokens.numel() >= 64
    _compare_layer(s, x, bias, y, r, host_weights("c3_skew"), tokens=tokens)
    # one balancing step: every bias moves by exactly +-gamma or 0, against the load
    gamma = 1e-3
    b0 = bias.clone()
    M.mrlmoe_bias_update(layer.cfg, r["counts"], bias, gamma)
    torch.cuda.synchronize()
    d = (bias - b0).cpu()
    sgn = torch.sign(torch.tensor(s.T * s.top_k) - s.n_experts * counts)
    want = (b0.cpu() + torch.tensor(gamma, dtype=torch.float32) * sgn.float()) - b0.cpu()
    assert torch.equal(d, want)
    assert int((sgn < 0).sum()) > 0 and int((sgn > 0).sum()) > 0


# ------------------------------------------------------------------- FP8
@pytest.mark.parametrize("rows,K", [(300, 512), (37, 384)])   # even and odd block counts per row
def test_quantize_e4m3_bit_exact(rows, K):
    g = torch.Generator().manual_seed(21)
    v = (torch.randn(rows, K, generator=g) * torch.exp(torch.randn(rows, 1, generator=g) * 2))
    v[3, :128] = 0.0                                   # an all-zero block
    v[5, 130] = 1e4                                    # an outlier
    v[7, 256:384] = -0.0
    xb = v.to(torch.bfloat16)
    xd = xb.cuda()
    q = torch.empty(rows, K, dtype=torch.uint8, device="cuda")
    sc = torch.empty(rows, K // 128, dtype=torch.float32, device="cuda")
    M.mrlmoe_quantize_e4m3(xd, rows, K, q, sc)
    torch.cuda.synchronize()
    deq = O.e4m3_decode(q.cpu()) * sc.cpu().double().repeat_interleave(128, 1)
    ref = O.quantize_act_1x128(xb.double())
    assert torch.equal(deq, ref)
    amax = xb.float().abs().reshape(rows, K // 128, 128).amax(-1)
    want = torch.where(amax == 0, torch.ones_like(amax), amax / torch.tensor(448.0))
    assert torch.equal(sc.cpu(), want)


def _compare_fp8(s, x, bias, y, r, wh, tokens=None):
    xs = x.cpu() if tokens is None else x.cpu()[tokens]
    ref = O.forward(xs, wh, bias.cpu(), s.top_k, s.rms_eps, fp8=True, fp4=s.fp4)
    gidx = r["topk_idx"].view(-1, s.top_k)
    if tokens is not None:
        gidx = gidx[tokens.to(gidx.device)]
    bad, gaps, _ = routing_audit(gidx, ref.s, bias, s.top_k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    keep = torch.ones(xs.shape[0], dtype=torch.bool)
    keep[bad] = False
    yg = y.cpu() if tokens is None else y.cpu()[tokens]
    mx, mean = rel_errors(yg[keep], ref.y[keep])
    assert mx <= FP8_MAX_REL and mean <= FP8_MEAN_REL, (mx, mean)
    return ref


def test_forward_fp8_tiny():
    s, x, bias, y, r, _ = _run_layer("c0_fp8")
    ref = _compare_fp8(s, x, bias, y, r, host_weights("c0_fp8"))
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)


@pytest.mark.parametrize("T", [1, 200])
def test_forward_fp8_tiny_ragged(T):
    s, x, bias, y, r, _ = _run_layer("c0_fp8", T=T)
    _compare_fp8(s, x, bias, y, r, host_weights("c0_fp8"))


@pytest.mark.parametrize("T", [1024, 1100, 10100])
def test_forward_fp8_tiny_larger_T(T):
    # the tiny FP8 layer at token counts whose experts average >= 128 rows
    # (several 128-token e4m3 units per expert, ragged last units); at
    # T = 10100 the projections run ~80 token tiles
    s, x, bias, y, r, _ = _run_layer("c0_fp8", T=T, scores=False)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    tokens = None if T <= 1100 else hard_tokens(r, s.T, s.n_experts, s.top_k, bn=256, want=300, seed=5)
    if tokens is not None:
        tokens = torch.unique(torch.cat([tokens, torch.arange(T - 140, T)]))
    _compare_fp8(s, x, bias, y, r, host_weights("c0_fp8"), tokens=tokens)


def test_forward_fp8_groups_of_every_size_larger_T():
    # expert 0 takes every token (1100 rows: eight full 128-token units and a
    # ragged one), the others 1 to a few hundred rows
    bias = torch.linspace(0.0, 0.05, 16, dtype=torch.float32)
    bias[0] = 10.0
    bias[5] += 0.2
    s, x, bias, y, r, _ = _run_layer("c0_fp8", T=1100, bias=bias.cuda(), scores=False)
    counts = r["counts"].cpu()
    assert int(counts[0]) == 1100 and int(counts.min()) < 128
    _compare_fp8(s, x, bias, y, r, host_weights("c0_fp8"))
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)


def _fp8_mid_width(T, fp4=False):
    # d_lat 512 (two 256-wide slices in the expert-down units), d_ff 384
    # (three 128-wide gate/up slices), d_model 384 (the up-projection's last
    # 256-column unit half outside N); at T = 10100 both projections run on
    # 256-column units (79 token tiles x 2 column tiles).  With fp4 the six
    # expert matrices are e2m1 codes, which the same units read through the
    # 4-bit unpacking TMA type.
    return W.LayerShape("fp4_mid" if fp4 else "fp8_mid", T=T, d_model=384, d_lat=512, n_experts=16, top_k=2,
                        d_ff=384, n_routers=2, fp8=True, fp4=fp4, outlier_frac=0.01)


@pytest.mark.parametrize("T,fp4", [(300, False), (10100, False), (300, True), (10100, True), (64, False),
                                   (64, True), (1, False), (1, True)])
def test_forward_fp8_mid_width(T, fp4):
    # T = 64: 8 rows per expert on average (groups of 0 to ~20 rows, one
    # 16- or 32-row token box each); T = 1: three groups of one row, most
    # CTAs without a unit
    s = _fp8_mid_width(T, fp4)
    w = W.make_layer_weights(s, "cuda", seed=0)
    x = W.make_x(s, "cuda", seed=0)
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, 901, "cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=False)
    y = layer(x, bias, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    tokens = None
    if T > 300:
        tokens = hard_tokens(r, s.T, s.n_experts, s.top_k, bn=128, want=300, seed=6)
        tokens = torch.unique(torch.cat([tokens, torch.arange(T - 140, T)]))
    _compare_fp8(s, x, bias, y, r, {k: v.cpu() for k, v in w.items()}, tokens=tokens)


@pytest.mark.parametrize("fp4", [False, True])
def test_forward_fp8_small_batch_hot_expert(fp4):
    # T = 64 with expert 0 taking every token (64 rows in one unit), expert 5
    # favoured and the rest holding 0 to a few rows
    s = _fp8_mid_width(64, fp4)
    w = W.make_layer_weights(s, "cuda", seed=1)
    x = W.make_x(s, "cuda", seed=1)
    bias = torch.linspace(0.0, 0.05, s.n_experts, dtype=torch.float32)
    bias[0] = 10.0
    bias[5] += 0.2
    bias = bias.cuda()
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=False)
    y = layer(x, bias, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    counts = r["counts"].cpu()
    assert int(counts[0]) == 64 and int(counts.min()) < 8
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    _compare_fp8(s, x, bias, y, r, {k: v.cpu() for k, v in w.items()})


def test_forward_c4_fp8_sampled_tokens():
    s, x, bias, y, r, _ = _run_layer("c4_fp8", scores=False)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    # e4m3 token tiles are 128 rows (boxes of 128/64/32/16): the same hard rows
    tokens = hard_tokens(r, s.T, s.n_experts, s.top_k, bn=128, want=40, seed=4)
    _compare_fp8(s, x, bias, y, r, host_weights("c4_fp8"), tokens=tokens)


def test_forward_fp8_groups_of_every_size():
    # every token on expert 0 (300 rows: two full 128-row tiles and a ragged
    # one), expert 5 favoured, a small ramp over the rest: groups of 1 to ~100
    # rows, so the token tiles load 16, 32, 32+16, 64 and 64+32+16-row boxes
    s = W.CONFIGS["c0_fp8"].with_T(300)
    bias = torch.linspace(0.0, 0.05, s.n_experts, dtype=torch.float32)
    bias[0] = 10.0
    bias[5] += 0.2
    s, x, bias, y, r, _ = _run_layer("c0_fp8", T=300, bias=bias.cuda())
    counts = r["counts"].cpu()
    assert int(counts.min()) < 16 and int(counts[0]) == 300
    assert len(set((int(c) + 15) // 16 for c in counts)) >= 5
    _compare_fp8(s, x, bias, y, r, host_weights("c0_fp8"))
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)


def test_forward_fp8_decode_size_sampled_tokens():
    s, x, bias, y, r, _ = _run_layer("c4_fp8", T=128, scores=False)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    _compare_fp8(s, x, bias, y, r, host_weights("c4_fp8"), tokens=torch.tensor([0, 63, 127]))


@pytest.mark.parametrize("T", [1152, 1153])
def test_route_either_side_of_the_router_k_split(T):
    # E = 512, R = 4: 8 expert chunks; 9 token tiles (T = 1152) take the
    # K-split router, 10 (T = 1153) the one that splits the expert range
    s = W.LayerShape("split", T=T, d_model=256, d_lat=128, n_experts=512, top_k=10, d_ff=128, n_routers=4)
    w = W.make_routing_weights(s, "cuda")
    x = W.make_x(s, "cuda")
    bias = W.uniform((s.n_experts,), -0.02, 0.02, 3, 940, "cuda")
    layer = M.MRLMoELayer(s, w)
    r = layer.routing_buffers(scores=True)
    layer.route(bias, x=x, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    zx = x.cpu().double() @ w["w_down"].cpu().double().T
    s_ref = O.router_scores(zx, w["w_router"].cpu())
    sg = r["scores"].view(T, s.n_experts).cpu().double()
    assert (sg - s_ref.double()).abs().max().item() < 1e-5
    bad, gaps, _ = routing_audit(r["topk_idx"].view(-1, s.top_k), s_ref, bias, s.top_k)
    assert torch.all(gaps < GAP_TOL), (bad, gaps)
    check_dispatch_properties(r, T, s.n_experts, s.top_k)


# ------------------------------------------------ FP4 expert weights (e2m1)
def test_forward_fp4_tiny():
    s, x, bias, y, r, _ = _run_layer("c0_fp4")
    _compare_fp8(s, x, bias, y, r, host_weights("c0_fp4"))
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)


@pytest.mark.parametrize("T", [1, 200])
def test_forward_fp4_tiny_ragged(T):
    s, x, bias, y, r, _ = _run_layer("c0_fp4", T=T)
    _compare_fp8(s, x, bias, y, r, host_weights("c0_fp4"))


def test_forward_fp4_groups_of_every_size():
    # as the FP8 case: expert 0 takes all 300 tokens (five 64-row token
    # tiles, the last ragged), the other groups hold 1 to ~100 rows
    bias = torch.linspace(0.0, 0.05, 16, dtype=torch.float32)
    bias[0] = 10.0
    bias[5] += 0.2
    s, x, bias, y, r, _ = _run_layer("c0_fp4", T=300, bias=bias.cuda())
    assert int(r["counts"][0]) == 300
    _compare_fp8(s, x, bias, y, r, host_weights("c0_fp4"))
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)


def test_forward_c1_fp4_sampled_tokens():
    s, x, bias, y, r, _ = _run_layer("c1_fp4", scores=False)
    check_dispatch_properties(r, s.T, s.n_experts, s.top_k)
    _compare_fp8(s, x, bias, y, r, host_weights("c1_fp4"), tokens=torch.tensor([0, 64, 127]))
