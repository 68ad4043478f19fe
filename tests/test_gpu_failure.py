"""Failure detection on the GPU, with no fault, trap or endless wait:

* a call whose GEMM family has its tile loads held (mrlmoe_config.hold: a
  flag that makes the loads never arrive) ends with MRLMOE_ERR_TIMEOUT after
  the bounded waits run out; the call's later kernels do nothing (y is left
  untouched), and the next call on the same workspace is clean and
  bit-identical to one made before;
* the device checker of the routing record passes every record the layer
  writes and reports each host-side corruption with exactly the invariant
  bits that the CPU reading of the invariants gives;
* outputs and the workspace stay inside their buffers (canary padding).
"""
import time

import pytest
import torch

import routing_checks as RC
import sparse_moe_layer_mean_b200 as M
import workloads as W
from helpers import device_weights
from sparse_moe_layer_mean_b200 import _native as N

pytestmark = pytest.mark.gpu

OK, TIMEOUT, CHECK = 0, 5, 6


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _bias(E):
    return W.uniform((E,), -0.01, 0.01, 4, 920, "cuda")


@pytest.mark.parametrize("family,config,T", [("gemm", "c0_tiny", None), ("gemm_pair", "c0_tiny", None),
                                             ("gemm_fp8", "c0_fp8", None), ("gemm_fp8", "c0_fp4", None),
                                             ("gemm_fp8", "c0_fp8", 1100),
                                             # full width at T = 4096: the first e4m3 GEMM (the
                                             # down-projection) runs on 256-column units
                                             ("gemm_fp8", "c4_fp8", 4096)])
def test_held_loads_run_out_the_bounded_waits(family, config, T):
    s = W.CONFIGS[config] if T is None else W.CONFIGS[config].with_T(T)
    x = W.make_x(s, "cuda")
    bias = _bias(s.n_experts)
    layer = M.MRLMoELayer(s, device_weights(config))
    y_ok = layer(x, bias)
    assert layer.device_status() == OK
    layer.cfg.hold = M.HOLD[family]
    y_bad = torch.zeros_like(y_ok)
    t0 = time.monotonic()
    layer(x, bias, y=y_bad)
    status = layer.device_status()
    dt = time.monotonic() - t0
    assert status == TIMEOUT, M.status_string(status)
    assert 1.5 < dt < 60.0, dt                 # the waits give up after about 2 s
    assert torch.all(y_bad == 0)               # the up-projection after the failure did nothing
    layer.cfg.hold = 0
    y_again = layer(x, bias)
    assert layer.device_status() == OK
    assert torch.equal(y_again, y_ok)


@pytest.mark.parametrize("config,T", [("c0_tiny", None), ("c0_tiny", 1), ("c0_tiny", 17),
                                      ("c2_prefill", 300), ("c0_fp8", None), ("c0_fp4", None)])
def test_checker_passes_the_layers_records(config, T):
    s = W.CONFIGS[config] if T is None else W.CONFIGS[config].with_T(T)
    x = W.make_x(s, "cuda")
    bias = _bias(s.n_experts)
    layer = M.MRLMoELayer(s, device_weights(config), checks=True)
    r = layer.routing_buffers()
    layer(x, bias, routing=r)                  # record in the caller's buffers
    assert layer.device_detail() == (OK, 0)
    layer(x, bias)                             # record kept in the workspace only
    assert layer.device_detail() == (OK, 0)
    layer.route(bias, x=x, routing=r)
    assert layer.device_detail() == (OK, 0)


def _check_on_device(rec, T, E, k):
    cfg = N.Config(T=T, d_model=128, d_lat=128, n_experts=E, top_k=k, d_ff=128, n_routers=1,
                   rms_eps=1e-6, dtype=0)
    dev = {n: v.cuda() for n, v in rec.items()}
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")       # the status header only
    M.mrlmoe_check_routing(cfg, M.make_routing(dev), ws, 256, True)
    return M.mrlmoe_get_device_detail(ws)


@pytest.mark.parametrize("T,E,k,hot", [(1, 16, 1, 0), (300, 64, 8, 0), (200, 64, 8, 8), (64, 1024, 16, 0),
                                       (5000, 512, 10, 0)])
def test_checker_passes_oracle_records(T, E, k, hot):
    rec = RC.oracle_record(T, E, k, seed=21 + T, hot=hot)
    assert RC.record_faults(rec, T, E, k) == 0
    assert _check_on_device(rec, T, E, k) == (OK, 0)


@pytest.mark.parametrize("kind", RC.KINDS)
@pytest.mark.parametrize("T,E,k,hot", [(300, 64, 8, 0), (200, 64, 8, 8)])
def test_checker_reports_host_corruptions(kind, T, E, k, hot):
    rec = RC.oracle_record(T, E, k, seed=5 + T, hot=hot)
    bad, want = RC.corrupt(rec, kind, T, E, k)
    assert RC.record_faults(bad, T, E, k) == want
    assert _check_on_device(bad, T, E, k) == (CHECK, want), kind


def test_checker_keeps_an_earlier_failure():
    # clear = 0 after a timed-out call: the status stays TIMEOUT (the first
    # failure of the call), while the check bits still accumulate
    s = W.CONFIGS["c0_tiny"]
    x = W.make_x(s, "cuda")
    layer = M.MRLMoELayer(s, device_weights("c0_tiny"))
    layer.cfg.hold = M.HOLD["gemm"]
    layer(x, _bias(s.n_experts))
    layer.check_routing()
    status, _ = layer.device_detail()
    assert status == TIMEOUT
    layer.cfg.hold = 0


CANARY16 = 0x7FA5            # a bf16 NaN pattern no kernel writes
CANARY32 = 0x5A5A5A5A


def _padded(n, dtype, pad, canary):
    it = torch.int16 if dtype == torch.bfloat16 else torch.int32
    buf = torch.full((n + 2 * pad,), canary, dtype=it, device="cuda")
    return buf, buf[pad:pad + n].view(dtype)


@pytest.mark.parametrize("config,T", [("c0_tiny", 37), ("c0_fp8", 37), ("c0_fp4", 37)])
def test_outputs_and_workspace_stay_inside_their_buffers(config, T):
    s = W.CONFIGS[config].with_T(T)
    x = W.make_x(s, "cuda")
    bias = _bias(s.n_experts)
    layer = M.MRLMoELayer(s, device_weights(config))
    ref_r = layer.routing_buffers(scores=True)
    y_ref = layer(x, bias, routing=ref_r)
    assert layer.device_status() == OK
    # the same call into canary-padded buffers: y, each routing array, the workspace
    pad = 64                                   # 128 or 256 bytes: keeps 16-byte alignment
    ybuf, y = _padded(T * s.d_model, torch.bfloat16, pad, CANARY16)
    bufs, r = {}, {}
    for name, t in ref_r.items():
        dt = torch.float32 if t.dtype == torch.float32 else torch.int32
        bufs[name], r[name] = _padded(t.numel(), dt, pad, CANARY32)
    wsbuf = torch.full((layer.ws_bytes + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    layer.workspace = wsbuf[:layer.ws_bytes]
    layer(x, bias, y=y.view(T, s.d_model), routing=r)
    assert layer.device_status() == OK
    torch.cuda.synchronize()
    assert torch.all(ybuf[:pad] == CANARY16) and torch.all(ybuf[-pad:] == CANARY16)
    for name, b in bufs.items():
        assert torch.all(b[:pad] == CANARY32) and torch.all(b[-pad:] == CANARY32), name
        assert torch.equal(r[name].cpu(), ref_r[name].cpu()), name
    assert torch.all(wsbuf[layer.ws_bytes:] == 0xA5)
    assert torch.equal(y.view(T, s.d_model), y_ref)


def _train_setup(config="c0_tiny", T=96):
    s = W.CONFIGS[config].with_T(T)
    x = W.make_x(s, "cuda")
    dy = W.make_dy(s, "cuda")
    bias = _bias(s.n_experts)
    layer = M.MRLMoELayer(s, device_weights(config), train=True)
    return s, x, dy, bias, layer


def _sentinel_grads(cfg):
    g = M.grad_buffers(cfg)
    for t in g.values():
        t.fill_(7.0)
    return g


def test_backward_with_held_loads_times_out_and_writes_nothing():
    s, x, dy, bias, layer = _train_setup()
    layer.forward_train(x, bias)
    ref = {k: v.clone() for k, v in layer.backward(x, dy).items()}
    assert layer.device_status() == OK
    layer.forward_train(x, bias)
    layer.cfg.hold = M.HOLD["gemm"]             # the backward's GEMMs issue no loads
    g = _sentinel_grads(layer.cfg)
    t0 = time.monotonic()
    layer.backward(x, dy, grads=g)
    status = layer.device_status()
    dt = time.monotonic() - t0
    assert status == TIMEOUT, M.status_string(status)
    assert 1.5 < dt < 60.0, dt
    for k, t in g.items():                      # the first GEMM timed out; no later kernel wrote
        assert torch.all(t == 7.0), k
    layer.cfg.hold = 0
    layer.forward_train(x, bias)
    again = layer.backward(x, dy)
    assert layer.device_status() == OK
    for k in ref:
        assert torch.equal(again[k], ref[k]), k


def test_backward_after_a_failed_training_forward_does_nothing():
    # the backward continues the forward's status word: a forward whose
    # gate/up GEMM timed out leaves the kept activations unwritten, and
    # every backward kernel then returns without reading them
    s, x, dy, bias, layer = _train_setup()
    layer.cfg.hold = M.HOLD["gemm_pair"]
    layer.forward_train(x, bias)
    layer.cfg.hold = 0
    g = _sentinel_grads(layer.cfg)
    layer.backward(x, dy, grads=g)
    assert layer.device_status() == TIMEOUT
    for k, t in g.items():
        assert torch.all(t == 7.0), k


def test_backward_buffers_stay_inside_their_bounds():
    s, x, dy, bias, layer = _train_setup(T=37)
    layer.forward_train(x, bias)
    ref = layer.backward(x, dy)
    torch.cuda.synchronize()
    assert layer.device_status() == OK
    pad = 64
    bufs, g = {}, {}
    for name, t in ref.items():
        it = torch.int16 if t.dtype == torch.bfloat16 else torch.int32
        canary = CANARY16 if it == torch.int16 else CANARY32
        buf = torch.full((t.numel() + 2 * pad,), canary, dtype=it, device="cuda")
        bufs[name] = (buf, canary)
        g[name] = buf[pad:pad + t.numel()].view(t.dtype).view(t.shape)
    wsbuf = torch.full((layer.ws_bytes + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    wsbuf[:layer.ws_bytes].copy_(layer.workspace)
    layer.workspace = wsbuf[:layer.ws_bytes]
    layer.forward_train(x, bias)
    layer.backward(x, dy, grads=g)
    assert layer.device_status() == OK
    torch.cuda.synchronize()
    for name, (buf, canary) in bufs.items():
        assert torch.all(buf[:pad] == canary) and torch.all(buf[-pad:] == canary), name
        assert torch.equal(g[name], ref[name]), name
    assert torch.all(wsbuf[layer.ws_bytes:] == 0xA5)
