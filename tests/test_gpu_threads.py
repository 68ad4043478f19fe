"""Host-side manners of the library under concurrency.

A fresh process makes its first calls from several host threads at once,
each thread with its own workspace and stream.  The library's first-use
state (the SM count per device, the shared-memory limit of each GEMM kernel
per device) is then set up concurrently.  Every thread's output must equal a
later single-threaded call bit for bit, and the caller's current device must
be unchanged after each call.  The first calls of a process happen only
once, so the check runs in a child process.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, threading
sys.path.insert(0, sys.argv[1])
import torch
import sparse_moe_layer_mean_b200 as M
import workloads as W

torch.cuda.set_device(0)
n = 4
cases = [("c0_tiny", None), ("c0_fp8", None), ("c0_tiny", 37), ("c0_fp4", None)]
jobs = []
for name, T in cases:
    s = W.CONFIGS[name] if T is None else W.CONFIGS[name].with_T(T)
    w = {k: v.cuda() for k, v in W.make_layer_weights(s, "cpu").items()}
    x = W.make_x(s, "cpu").cuda()
    bias = torch.zeros(s.n_experts, device="cuda")
    jobs.append((s, w, x, bias, M.MRLMoELayer(s, w), torch.cuda.Stream()))
torch.cuda.synchronize()
outs = [None] * n
devs = [None] * n
gate = threading.Barrier(n)

def run(i):
    s, w, x, bias, layer, st = jobs[i]
    torch.cuda.set_device(0)
    y = torch.empty(s.T, s.d_model, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    gate.wait()                                   # every thread's first call at once
    layer(x, bias, y=y, stream=st)
    devs[i] = torch.cuda.current_device()
    outs[i] = y

ts = [threading.Thread(target=run, args=(i,)) for i in range(n)]
for t in ts:
    t.start()
for t in ts:
    t.join()
torch.cuda.synchronize()
for i, (s, w, x, bias, layer, st) in enumerate(jobs):
    assert layer.device_status() == 0, (i, layer.device_status())
    assert devs[i] == 0
    again = layer(x, bias)                        # single-threaded, default stream
    torch.cuda.synchronize()
    assert torch.equal(again, outs[i]), i
print("threads ok")
"""


def test_concurrent_first_calls_from_host_threads():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "threads ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
