"""The C ABI on the host (no GPU): the library loads, exports every entry
point include/mrlmoe.h declares, and rejects bad arguments with the
documented status before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_moe_layer_mean_b200 as M
from sparse_moe_layer_mean_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mrlmoe.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mrlmoe_[a-z0-9_]+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = N.lib()
    names = _declared()
    assert set(names) == set(N.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}\b", out), n


def test_status_strings():
    for code in range(8):
        assert M.status_string(code)
    assert M.status_string(99) == "unknown status"


def _cfg(**kw):
    d = dict(T=64, d_model=256, d_lat=128, n_experts=16, top_k=2, d_ff=128, n_routers=2,
             rms_eps=1e-6, dtype=0)
    d.update(kw)
    return N.Config(**d)


def test_workspace_size_valid_and_invalid():
    assert M.mrlmoe_workspace_size(_cfg()) > 0
    for bad in (dict(T=0), dict(d_model=200), dict(d_lat=0), dict(d_ff=100), dict(n_experts=8),
                dict(n_experts=24 + 1), dict(top_k=0), dict(top_k=17), dict(top_k=17, n_experts=16),
                dict(n_routers=0), dict(n_routers=9), dict(rms_eps=-1.0), dict(dtype=7),
                dict(aggregation=3), dict(aggregation=-1), dict(hold=8), dict(hold=0x100)):
        assert M.mrlmoe_workspace_size(_cfg(**bad)) == 0, bad
    for hold in (1, 2, 4, 7):                                    # the GEMM families of mrlmoe_hold
        assert M.mrlmoe_workspace_size(_cfg(hold=hold)) > 0
    # k up to min(E, 32)
    assert M.mrlmoe_workspace_size(_cfg(top_k=32, n_experts=32)) > 0
    assert M.mrlmoe_workspace_size(_cfg(top_k=17, n_experts=64)) > 0
    assert M.mrlmoe_workspace_size(_cfg(top_k=33, n_experts=64)) == 0
    for agg in (0, 1, 2):                                       # mean, sum, max
        assert M.mrlmoe_workspace_size(_cfg(aggregation=agg)) > 0
    # the FP8 variant stages at most 32 K-block scales per GEMM unit: K <= 4096
    for big in (dict(d_model=4224), dict(d_lat=4224), dict(d_ff=4224)):
        assert M.mrlmoe_workspace_size(_cfg(dtype=1, **big)) == 0, big
        assert M.mrlmoe_workspace_size(_cfg(dtype=0, **big)) > 0, big
    assert M.mrlmoe_workspace_size(_cfg(dtype=1, d_model=4096, d_lat=4096, d_ff=4096)) > 0
    # grows with T
    assert M.mrlmoe_workspace_size(_cfg(T=128)) > M.mrlmoe_workspace_size(_cfg(T=64))


def _raw_forward(cfg, w, bias, x, y, ws, nbytes):
    return N.lib().mrlmoe_forward(ctypes.byref(cfg) if cfg is not None else None,
                                  ctypes.byref(w) if w is not None else None,
                                  bias, x, y, None, ws, nbytes, None)


def test_forward_rejects_bad_arguments_before_cuda():
    cfg = _cfg()
    full = N.Weights(*([4096] * 11 + [None] * 8))   # fake, 16-byte aligned "pointers"
    need = M.mrlmoe_workspace_size(cfg)
    assert _raw_forward(None, full, 4096, 4096, 4096, 4096, need) == 1
    assert _raw_forward(_cfg(T=0), full, 4096, 4096, 4096, 4096, need) == 1
    assert _raw_forward(cfg, None, 4096, 4096, 4096, 4096, need) == 1
    assert _raw_forward(cfg, full, None, 4096, 4096, 4096, need) == 1      # bias
    assert _raw_forward(cfg, full, 4096, None, 4096, 4096, need) == 1      # x
    assert _raw_forward(cfg, full, 4096, 4104, 4096, 4096, need) == 1      # x misaligned
    partial = N.Weights(*([4096] * 2 + [None] + [4096] * 8 + [None] * 8))
    assert _raw_forward(cfg, partial, 4096, 4096, 4096, 4096, need) == 1   # w_gate missing
    assert _raw_forward(cfg, full, 4096, 4096, 4096, None, need) == 3      # no workspace
    assert _raw_forward(cfg, full, 4096, 4096, 4096, 4096 + 16, need) == 3  # misaligned
    assert _raw_forward(cfg, full, 4096, 4096, 4096, 4096, need - 1) == 3  # too small
    # the FP8 variant needs the block-scale arrays too
    cfg8 = _cfg(dtype=1)
    need8 = M.mrlmoe_workspace_size(cfg8)
    assert need8 > need                                                    # e4m3 copies of the GEMM inputs
    assert _raw_forward(cfg8, full, 4096, 4096, 4096, 4096, need8) == 1
    full8 = N.Weights(*([4096] * 11 + [8192] * 8))
    assert _raw_forward(cfg8, full8, 4096, 4096, 4096, 4096, need8 - 1) == 3
    # FP4 experts: the six expert code matrices must be 32-byte aligned (the
    # 4-bit unpacking TMA type); 16 bytes is enough for the FP8 variant
    cfg4 = _cfg(dtype=2)
    need4 = M.mrlmoe_workspace_size(cfg4)
    for i in range(2, 8):                                                 # w_gate .. w_sh_down
        ptrs = [4096] * 11 + [8192] * 8
        ptrs[i] = 4096 + 16
        assert _raw_forward(cfg4, N.Weights(*ptrs), 4096, 4096, 4096, 4096, need4) == 1, N.WEIGHT_FIELDS[i]
        assert _raw_forward(cfg8, N.Weights(*ptrs), 4096, 4096, 4096, 4096, need8 - 1) == 3


def test_route_rejects_bad_arguments_before_cuda():
    cfg = _cfg()
    w = N.Weights(*([4096] * 11 + [None] * 8))
    r = N.Routing(*([None] * 7))
    need = M.mrlmoe_workspace_size(cfg)
    L = N.lib()
    # scores_in without scores
    assert L.mrlmoe_route(ctypes.byref(cfg), ctypes.byref(w), 4096, None, 1, ctypes.byref(r), 4096,
                          need, None) == 1
    # routing from x without x
    assert L.mrlmoe_route(ctypes.byref(cfg), ctypes.byref(w), 4096, None, 0, ctypes.byref(r), 4096,
                          need, None) == 1
    # no routing struct
    assert L.mrlmoe_route(ctypes.byref(cfg), ctypes.byref(w), 4096, 4096, 0, None, 4096, need, None) == 1
    r2 = N.Routing(*([None] * 6 + [4096]))
    assert L.mrlmoe_route(ctypes.byref(cfg), ctypes.byref(w), 4096, None, 1, ctypes.byref(r2), 4096,
                          need - 256, None) == 3


def test_bias_update_and_linear_reject_bad_arguments():
    L = N.lib()
    cfg = _cfg()
    assert L.mrlmoe_bias_update(ctypes.byref(cfg), None, 4096, 1e-3, None) == 1
    assert L.mrlmoe_bias_update(ctypes.byref(cfg), 4096, None, 1e-3, None) == 1
    assert L.mrlmoe_bias_update(None, 4096, 4096, 1e-3, None) == 1
    assert L.mrlmoe_linear(4096, 4096, 4096, 0, 128, 128, None) == 1
    assert L.mrlmoe_linear(4096, 4096, 4096, 8, 100, 128, None) == 1
    assert L.mrlmoe_linear(4096, 4096, 4096, 8, 128, 64, None) == 1
    assert L.mrlmoe_linear(None, 4096, 4096, 8, 128, 128, None) == 1
    assert L.mrlmoe_linear(4096 + 2, 4096, 4096, 8, 128, 128, None) == 1


def test_quantize_rejects_bad_arguments():
    L = N.lib()
    assert L.mrlmoe_quantize_e4m3(None, 4, 128, 4096, 4096, None) == 1
    assert L.mrlmoe_quantize_e4m3(4096, 0, 128, 4096, 4096, None) == 1
    assert L.mrlmoe_quantize_e4m3(4096, 4, 100, 4096, 4096, None) == 1
    assert L.mrlmoe_quantize_e4m3(4096 + 2, 4, 128, 4096, 4096, None) == 1
    assert L.mrlmoe_quantize_e4m3(4096 + 8, 4, 128, 4096, 4096, None) == 1   # in: 16-byte aligned
    assert L.mrlmoe_quantize_e4m3(4096, 4, 128, 4096 + 4, 4096, None) == 1   # q: 8-byte aligned


def test_check_routing_and_detail_reject_bad_arguments():
    L = N.lib()
    cfg = _cfg()
    need = M.mrlmoe_workspace_size(cfg)
    whole = N.Routing(*([4096] * 6 + [None]))
    part = N.Routing(*([4096] * 3 + [None] * 4))
    chk = lambda c, r, ws, n: L.mrlmoe_check_routing(ctypes.byref(c) if c is not None else None,
                                                     ctypes.byref(r) if r is not None else None, ws, n, 1, None)
    assert chk(None, whole, 4096, 256) == 1
    assert chk(_cfg(hold=16), whole, 4096, 256) == 1
    assert chk(cfg, whole, None, 256) == 3          # no workspace
    assert chk(cfg, whole, 4096 + 16, 256) == 3     # misaligned
    assert chk(cfg, whole, 4096, 255) == 3          # smaller than the status header
    assert chk(cfg, part, 4096, 256) == 3           # a field read from the workspace: full size needed
    assert chk(cfg, None, 4096, need - 1) == 3
    det = ctypes.c_uint32(0)
    assert L.mrlmoe_get_device_detail(None, ctypes.byref(det), None) == 3
    assert L.mrlmoe_get_device_detail(4096, None, None) == 1


def test_python_binding_raises_on_error():
    with pytest.raises(M.MrlmoeError) as ei:
        M.mrlmoe_linear(0, 0, 0, 8, 128, 128, stream=0)
    assert ei.value.code == 1


def test_training_entry_points_reject_bad_arguments_before_cuda():
    L = N.lib()
    cfg = _cfg()
    fwd = M.mrlmoe_workspace_size(cfg)
    train = M.mrlmoe_train_workspace_size(cfg)
    assert train > fwd                                  # + kept pre-activations and backward buffers
    assert M.mrlmoe_train_workspace_size(_cfg(T=128)) > train
    assert M.mrlmoe_train_workspace_size(_cfg(dtype=1)) == 0   # bf16 only
    assert M.mrlmoe_train_workspace_size(_cfg(dtype=2)) == 0
    assert M.mrlmoe_train_workspace_size(_cfg(T=0)) == 0
    assert M.mrlmoe_train_workspace_size(_cfg(d_ff=8320)) == 0  # d_ff <= 8192
    w = N.Weights(*([4096] * 11 + [None] * 8))
    g = N.Grads(*([4096] * 12))
    bwd = lambda c, w_, x, dy, g_, ws, n: L.mrlmoe_backward(
        ctypes.byref(c) if c is not None else None, ctypes.byref(w_) if w_ is not None else None, x, dy,
        ctypes.byref(g_) if g_ is not None else None, ws, n, None)
    assert bwd(None, w, 4096, 4096, g, 4096, train) == 1
    assert bwd(_cfg(dtype=1), w, 4096, 4096, g, 4096, train) == 2       # unsupported: FP8
    assert bwd(cfg, w, None, 4096, g, 4096, train) == 1                 # x
    assert bwd(cfg, w, 4096, None, g, 4096, train) == 1                 # dy
    assert bwd(cfg, w, 4096, 4096 + 2, g, 4096, train) == 1             # dy misaligned
    assert bwd(cfg, w, 4096, 4096, None, 4096, train) == 1              # no grads struct
    for i in range(12):                                                 # every gradient is required
        gi = N.Grads(*([4096] * i + [None] + [4096] * (11 - i)))
        assert bwd(cfg, w, 4096, 4096, gi, 4096, train) == 1, N.GRAD_FIELDS[i]
    partial = N.Weights(*([4096] * 2 + [None] + [4096] * 8 + [None] * 8))
    assert bwd(cfg, partial, 4096, 4096, g, 4096, train) == 1          # w_gate missing
    assert bwd(cfg, w, 4096, 4096, g, None, train) == 3                 # no workspace
    assert bwd(cfg, w, 4096, 4096, g, 4096 + 16, train) == 3            # misaligned
    assert bwd(cfg, w, 4096, 4096, g, 4096, train - 1) == 3             # forward-sized is too small
    ft = lambda c, ws, n: L.mrlmoe_forward_train(ctypes.byref(c), ctypes.byref(w), 4096, 4096, 4096, None,
                                                 ws, n, None)
    assert ft(_cfg(dtype=1), 4096, train) == 2
    assert ft(cfg, 4096, train - 1) == 3
    ev = (ctypes.c_void_p * N.NUM_BACKWARD_EVENTS)(*([4096] * N.NUM_BACKWARD_EVENTS))
    assert L.mrlmoe_backward_timed(ctypes.byref(cfg), ctypes.byref(w), 4096, 4096, ctypes.byref(g), 4096, train,
                                   None, ev, N.NUM_BACKWARD_EVENTS - 1) == 1
    assert L.mrlmoe_backward_timed(ctypes.byref(cfg), ctypes.byref(w), 4096, 4096, ctypes.byref(g), 4096, train,
                                   None, None, N.NUM_BACKWARD_EVENTS) == 1


def test_expert_parallel_entry_points_reject_bad_arguments_before_cuda():
    L = N.lib()
    cfg = _cfg()
    base = M.mrlmoe_workspace_size(cfg)
    ws4 = N.mrlmoe_ep_workspace_size(cfg, 4)
    assert ws4 > base                                          # + received rows and their h
    assert N.mrlmoe_ep_workspace_size(cfg, 8) > ws4            # more sources, more rows
    assert N.mrlmoe_ep_workspace_size(cfg, 3) == 0             # E = 16 does not divide by 3
    assert N.mrlmoe_ep_workspace_size(cfg, 0) == 0
    assert N.mrlmoe_ep_workspace_size(cfg, 65) == 0
    assert N.mrlmoe_ep_workspace_size(_cfg(dtype=1), 2) == 0   # bf16 only
    w = N.Weights(*([4096] * 11 + [None] * 8))
    r = N.Routing(*([4096] * 7))
    disp = lambda c, n, x, r_, send, ws, nb: L.mrlmoe_ep_dispatch(
        ctypes.byref(c), ctypes.byref(w), 4096, x, n, ctypes.byref(r_) if r_ is not None else None, send, ws, nb, None)
    assert disp(cfg, 3, 4096, r, 4096, 4096, ws4) == 1               # ranks do not divide E
    assert disp(_cfg(dtype=1), 2, 4096, r, 4096, 4096, ws4) == 2     # FP8: unsupported
    assert disp(cfg, 4, None, r, 4096, 4096, ws4) == 1               # x
    assert disp(cfg, 4, 4096, None, 4096, 4096, ws4) == 1            # record
    no_counts = N.Routing(4096, 4096, None, 4096, 4096, 4096, 4096)
    assert disp(cfg, 4, 4096, no_counts, 4096, 4096, ws4) == 1       # counts are required
    assert disp(cfg, 4, 4096, r, 4096 + 8, 4096, ws4) == 1           # send rows misaligned
    assert disp(cfg, 4, 4096, r, 4096, 4096, base - 1) == 3          # workspace too small
    exp = lambda n, rows, counts, n_recv, out, ws, nb: L.mrlmoe_ep_experts(
        ctypes.byref(cfg), ctypes.byref(w), n, rows, counts, n_recv, out, ws, nb, None)
    assert exp(4, 4096, 4096, -1, 4096, 4096, ws4) == 1              # negative row count
    assert exp(4, 4096, None, 10, 4096, 4096, ws4) == 1              # counts
    assert exp(4, None, 4096, 10, 4096, 4096, ws4) == 1              # rows
    assert exp(4, 4096, 4096, 10, 4096 + 4, 4096, ws4) == 1          # out misaligned
    assert exp(4, 4096, 4096, 10 ** 6, 4096, 4096, ws4) == 3         # more rows than the workspace holds
    assert exp(4, None, 4096, 0, None, 4096, ws4) == 0               # nothing arrived: nothing to do
    comb = lambda ret, y, ws, nb: L.mrlmoe_ep_combine(ctypes.byref(cfg), ctypes.byref(w), ret, y, ws, nb, None)
    assert comb(None, 4096, 4096, ws4) == 1
    assert comb(4096, 4096 + 2, 4096, ws4) == 1
    assert comb(4096, 4096, 4096, base) == 3                         # needs the expert-parallel tables


def test_gradient_fields_cover_every_learnable_tensor():
    from oracle import mrlmoe_backward as OB
    # dx -> x, d_<name> -> <name>: the same twelve tensors as the oracle's backward
    assert sorted("x" if f == "dx" else f[2:] for f in N.GRAD_FIELDS) == sorted(OB.GRAD_NAMES)
    # and the C struct: twelve pointers then the accumulate flag
    assert [n for n, _ in N.Grads._fields_] == list(N.GRAD_FIELDS) + ["accumulate"]


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "mrlmoe.h"
int main(void) {
  mrlmoe_config c;
  memset(&c, 0, sizeof c);
  c.T = 64; c.d_model = 256; c.d_lat = 128; c.n_experts = 16; c.top_k = 2; c.d_ff = 128; c.n_routers = 2;
  c.rms_eps = 1e-6f; c.dtype = MRLMOE_BF16; c.aggregation = MRLMOE_AGG_MEAN;
  size_t f = mrlmoe_workspace_size(&c), t = mrlmoe_train_workspace_size(&c);
  mrlmoe_grads g;
  memset(&g, 0, sizeof g);
  /* host-side rejection before any CUDA work: a null x */
  mrlmoe_status s = mrlmoe_backward(&c, NULL, NULL, NULL, &g, NULL, t, NULL);
  printf("%zu %zu %d %s\n", f, t, (int)s, mrlmoe_status_string(s));
  return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    # the ABI from C itself: the header compiles as strict C99, a C program
    # links against the library and calls its host-only entry points
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    lib_dir = os.path.dirname(N.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(ROOT, "include"), str(src), "-L", lib_dir, "-lmrlmoe",
                        f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    f, t, code, *msg = out.stdout.split()
    assert int(f) == M.mrlmoe_workspace_size(_cfg())
    assert int(t) == M.mrlmoe_train_workspace_size(_cfg()) > int(f)
    assert int(code) == 1 and " ".join(msg) == M.status_string(1)
