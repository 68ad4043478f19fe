"""The expert-parallel form of the layer on one GPU: N ranks emulated in one
process through the C ABI's three phases (mrlmoe_ep_dispatch,
mrlmoe_ep_experts, mrlmoe_ep_combine).  The exchanges are device copies of
the slices; no rank reads another's buffers.

Every rank's y is compared with two things.  The first is the single-GPU
forward of that rank's own tokens, bit for bit: the combine adds in the
single-GPU order and precision, and each expert row goes through the same
GEMM arithmetic.  The second is the expert-parallel oracle
(oracle/mrlmoe_ep.py), within the layer's bf16 bounds, for N = 2, 4 and 8."""
import pytest
import torch

import oracle as O
import sparse_moe_layer_mean_b200 as M
import workloads as W
from oracle import mrlmoe_ep as OEP
from sparse_moe_layer_mean_b200 import ep as EP
from helpers import BF16_MAX_REL, BF16_MEAN_REL, GAP_TOL, device_weights, host_weights, rel_errors, routing_audit

pytestmark = pytest.mark.gpu

TOKENS = [64, 37, 1, 50, 64, 20, 3, 64]


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _ranks(name, n, Ts, seed_bias=900):
    s = W.CONFIGS[name]
    w = device_weights(name)
    shape = s.with_T(max(Ts))
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, seed_bias, "cuda")
    xs = [W.make_x(s, "cuda", seed=11 + r, T=T) for r, T in enumerate(Ts)]
    ranks = [EP.ExpertParallelRank(shape, w, r, n) for r in range(n)]
    return s, w, bias, xs, ranks


def _single_gpu(s, w, x, bias):
    layer = M.MRLMoELayer(s.with_T(x.shape[0]), w)
    r = layer.routing_buffers()
    y = layer(x, bias, routing=r)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return y, r


@pytest.mark.parametrize("n", [2, 4, 8])
def test_expert_parallel_tiny_equals_single_gpu_and_oracle(n):
    Ts = TOKENS[:n]
    s, w, bias, xs, ranks = _ranks("c0_tiny", n, Ts)
    ys = EP.emulate_forward(ranks, xs, bias)
    torch.cuda.synchronize()
    routes = []
    for r in range(n):
        assert ranks[r].status() == 0, r
        y1, rt = _single_gpu(s, w, xs[r], bias)
        assert torch.equal(ys[r], y1), r
        routes.append(rt)
    wh = host_weights("c0_tiny")
    outs, recs = OEP.ep_forward([x.cpu() for x in xs], wh, bias.cpu(), s.top_k, s.rms_eps)
    for r in range(n):
        ref = O.forward(xs[r].cpu(), wh, bias.cpu(), s.top_k, s.rms_eps)
        bad, gaps, _ = routing_audit(routes[r]["topk_idx"], ref.s, bias, s.top_k)
        assert torch.all(gaps < GAP_TOL), (bad, gaps)
        keep = torch.ones(Ts[r], dtype=torch.bool)
        keep[bad] = False
        mx, mean = rel_errors(ys[r].cpu()[keep], outs[r]["y"][keep])
        assert mx <= BF16_MAX_REL and mean <= BF16_MEAN_REL, (r, mx, mean)


@pytest.mark.parametrize("n,Ts", [(8, [128, 64, 1, 200, 33, 96, 128, 17]), (4, [300, 1, 64, 129])])
def test_expert_parallel_full_width_equals_single_gpu(n, Ts):
    s, w, bias, xs, ranks = _ranks("c2_prefill", n, Ts)
    ys = EP.emulate_forward(ranks, xs, bias)
    torch.cuda.synchronize()
    for r in range(n):
        assert ranks[r].status() == 0, r
        assert torch.equal(ys[r], _single_gpu(s, w, xs[r], bias)[0]), r


def test_expert_parallel_full_width_against_the_oracle():
    # four ranks, the oracle on a few tokens of two of them (the single-GPU
    # oracle per rank equals the expert-parallel oracle: its own CPU test)
    Ts = [96, 7, 64, 33]
    s, w, bias, xs, ranks = _ranks("c2_prefill", 4, Ts)
    ys = EP.emulate_forward(ranks, xs, bias)
    torch.cuda.synchronize()
    wh = host_weights("c2_prefill")
    for r, toks in ((0, [0, 5, 95]), (1, [0, 3, 6])):
        t = torch.tensor(toks)
        _, rt = _single_gpu(s, w, xs[r], bias)
        ref = O.forward(xs[r].cpu()[t], wh, bias.cpu(), s.top_k, s.rms_eps)
        bad, gaps, _ = routing_audit(rt["topk_idx"].view(-1, s.top_k)[t.cuda()], ref.s, bias, s.top_k)
        assert torch.all(gaps < GAP_TOL), (bad, gaps)
        keep = torch.ones(len(toks), dtype=torch.bool)
        keep[bad] = False
        mx, mean = rel_errors(ys[r].cpu()[t][keep], ref.y[keep])
        assert mx <= BF16_MAX_REL and mean <= BF16_MEAN_REL, (r, mx, mean)


def test_expert_parallel_bad_counts_end_in_check():
    # counts that do not add up to the rows received: the owner records
    # MRLMOE_ERR_CHECK and reads nothing through them
    s, w, bias, xs, ranks = _ranks("c0_tiny", 2, [64, 37])
    d = ranks[0].dispatch(xs[0], bias)
    rc = torch.stack([EP.counts_by_destination(d.counts, 2)[0]] * 2).contiguous()
    n_in = int(rc.sum())
    recv = torch.zeros(n_in + 5, s.d_lat, dtype=torch.bfloat16, device="cuda")
    out = torch.full((n_in + 5, s.d_lat), 7.0, device="cuda")
    M._native.mrlmoe_ep_experts(M.make_config(s.with_T(64)), ranks[0].cw_local, 2, recv, rc, n_in + 5, out,
                                ranks[0].workspace, ranks[0].ws_bytes)
    assert ranks[0].status() == 6
    assert torch.all(out == 7.0)
