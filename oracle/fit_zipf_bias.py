"""Fit the scale of the skewed workload's selection bias on the oracle.

TEST INFRASTRUCTURE: writes tests/golden/<config>_zipf_lambda.json, an input
parameter of the skewed workload.  It calls only the oracle and the seeded
input generator.

The workload's bias is b_e = lambda * ln(p_rank(e) / p_1) with p_i ∝ i^-1.1
over a seeded random ranking of the experts; lambda > 0 is chosen by
bisection so that, under the oracle's routing of this config's x, the busiest
expert receives max(count) / mean(count) in [28, 32] (about 30x the mean
load), mean = T*k/E.

    python -m oracle.fit_zipf_bias [config]        # default c3_skew
"""
from __future__ import annotations

import json
import os
import sys
import time

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402
from oracle.mrlmoe_oracle import router_scores, select_topk  # noqa: E402

TARGET = (28.0, 32.0)


def skew_ratio(s: torch.Tensor, lnr: torch.Tensor, lam: float, k: int) -> float:
    b = torch.tensor(lam, dtype=torch.float32) * lnr
    idx = select_topk(s, b, k)
    counts = torch.bincount(idx.flatten(), minlength=lnr.numel()).double()
    return (counts.max() / counts.mean()).item()


def fit(name: str = "c3_skew", chunk: int = 4096):
    shape = W.CONFIGS[name]
    t0 = time.time()
    wdn = W.normal((shape.d_lat, shape.d_model), shape.seed, W._S_WDN, "cpu", std=shape.d_model ** -0.5)
    wr = W.normal((shape.n_routers, shape.n_experts, shape.d_lat), shape.seed, W._S_WR, "cpu",
                  std=shape.d_lat ** -0.5)
    x = W.make_x(shape, "cpu")
    parts = []
    for i in range(0, shape.T, chunk):
        zx = x[i:i + chunk].double() @ wdn.double().T       # the routers read the unrounded latent
        parts.append(router_scores(zx, wr))
    s = torch.cat(parts)
    lnr = W.zipf_ln_ratio(shape, "cpu")
    lo, hi = 0.0, 1.0
    while skew_ratio(s, lnr, hi, shape.top_k) < TARGET[0]:
        lo, hi = hi, hi * 2
    lam, ratio = hi, None
    for _ in range(40):
        lam = 0.5 * (lo + hi)
        ratio = skew_ratio(s, lnr, lam, shape.top_k)
        if ratio < TARGET[0]:
            lo = lam
        elif ratio > TARGET[1]:
            hi = lam
        else:
            break
    out = {"config": name, "lambda": lam, "max_over_mean_load": ratio, "target": list(TARGET),
           "T": shape.T, "n_experts": shape.n_experts, "top_k": shape.top_k, "seed": shape.seed,
           "zipf_s": 1.1, "made_by": "oracle/fit_zipf_bias.py (oracle routing of the config's x)",
           "seconds": round(time.time() - t0, 1)}
    path = os.path.join(ROOT, "tests", "golden", f"{name}_zipf_lambda.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    return out


if __name__ == "__main__":
    print(fit(sys.argv[1] if len(sys.argv) > 1 else "c3_skew"))
