"""Shared helpers for the GPU parity tests: seeded inputs on the device, host
copies for the oracle, and the parity metrics."""
from __future__ import annotations

import functools

import torch

import oracle as O
import workloads as W

# Output bounds for the bf16 layer: max|dy| / max|y_ref| and sum|dy| / sum|y_ref|.
BF16_MAX_REL = 1e-2
BF16_MEAN_REL = 2e-3
# ... and for the FP8 variant
FP8_MAX_REL = 3e-2
FP8_MEAN_REL = 6e-3
# A routing mismatch is legitimate only where the oracle's k-th vs (k+1)-th
# biased-score gap is below this.
GAP_TOL = 1e-5


def _wkey(name: str) -> str:
    """Configs with the same layer shape and weight type share one set of weights."""
    s = W.CONFIGS[name]
    if s.d_model == 256:
        return "c0_fp4" if s.fp4 else "c0_fp8" if s.fp8 else "c0_tiny"
    return "c1_fp4" if s.fp4 else "c4_fp8" if s.fp8 else "c2_prefill"


@functools.lru_cache(maxsize=2)
def _device_weights(key: str, seed: int):
    return W.make_layer_weights(W.CONFIGS[key], "cuda", seed=seed)


@functools.lru_cache(maxsize=2)
def _host_weights(key: str, seed: int):
    return {k: v.cpu() for k, v in _device_weights(key, seed).items()}


def device_weights(name: str, seed: int = 0):
    return _device_weights(_wkey(name), seed)


def host_weights(name: str, seed: int = 0):
    return _host_weights(_wkey(name), seed)


def rel_errors(y: torch.Tensor, ref: torch.Tensor):
    d = (y.double() - ref.double()).abs()
    r = ref.double().abs()
    return (d.max() / r.max()).item(), (d.sum() / r.sum()).item()


def routing_audit(gpu_idx: torch.Tensor, s_ref: torch.Tensor, bias: torch.Tensor, k: int):
    """Tokens whose GPU top-k set differs from the oracle's, and the oracle's
    boundary gap at each of them."""
    ref_idx = O.select_topk(s_ref, bias.cpu(), k)
    g = torch.sort(gpu_idx.cpu().long().view(-1, k), dim=1).values
    r = torch.sort(ref_idx, dim=1).values
    bad = (g != r).any(dim=1).nonzero().flatten()
    gaps = O.topk_boundary_gap(s_ref[bad], bias.cpu(), k) if bad.numel() else torch.zeros(0)
    return bad, gaps, ref_idx


def check_dispatch_properties(r, T: int, E: int, k: int):
    """Invariants of the dispatch record at any size."""
    idx = r["topk_idx"].cpu().long().view(T, k)
    counts = r["counts"].cpu().long()
    offsets = r["offsets"].cpu().long()
    perm = r["perm"].cpu().long()
    inv = r["inv_perm"].cpu().long()
    assert torch.all((idx >= 0) & (idx < E))
    assert torch.all(torch.sort(idx, dim=1).values[:, 1:] != torch.sort(idx, dim=1).values[:, :-1])
    assert torch.equal(counts, torch.bincount(idx.flatten(), minlength=E))
    assert int(counts.sum()) == T * k
    assert int(offsets[0]) == 0 and torch.equal(offsets[1:], torch.cumsum(counts, 0))
    assert torch.equal(torch.sort(perm).values, torch.arange(T * k))
    assert torch.equal(inv[perm], torch.arange(T * k))
    e_of_row = idx.flatten()[perm]
    rows_e = torch.repeat_interleave(torch.arange(E), counts)
    assert torch.equal(e_of_row, rows_e)
    tok = perm // k
    same = e_of_row[1:] == e_of_row[:-1]
    assert torch.all(tok[1:][same] > tok[:-1][same])


def hard_tokens(r, T: int, E: int, k: int, bn: int = 256, want: int = 64, seed: int = 0):
    """Tokens whose dispatch rows sit where the grouped GEMMs are hardest,
    read from the routing record: the first, last and ragged token tile of
    the busiest expert, rows on both sides of the CTA-pair split of a tile
    (half = round32(rows) / 2), groups of 1 to 16 rows, groups whose size
    straddles the 64/32/16-row box sizes, and the shared expert's first and
    last tiles; topped up with seeded random tokens to ``want``."""
    counts = r["counts"].cpu().long()
    offsets = r["offsets"].cpu().long()
    perm = r["perm"].cpu().long()
    rows = []

    def tile_rows(e, t0, nv):
        base = int(offsets[e]) + t0
        half = ((nv + 31) // 32 * 32) // 2
        for q in (0, 1, half - 1, half, nv - 1):
            if 0 <= q < nv:
                rows.append(base + q)

    hot = int(torch.argmax(counts))
    c = int(counts[hot])
    nt = (c + bn - 1) // bn
    tile_rows(hot, 0, min(bn, c))                                 # first tile
    if nt > 1:
        tile_rows(hot, (nt - 1) * bn, c - (nt - 1) * bn)          # last (ragged) tile
        tile_rows(hot, (nt // 2) * bn, min(bn, c - (nt // 2) * bn))
    small = [e for e in range(E) if 1 <= int(counts[e]) <= 16][:8]
    for e in small:
        tile_rows(e, 0, int(counts[e]))
    for m in (16, 17, 31, 32, 33, 63, 64, 65, 96, 127, 128, 129):
        hit = (counts % bn == m).nonzero().flatten()
        if hit.numel():
            e = int(hit[0])
            t0 = (int(counts[e]) // bn) * bn
            tile_rows(e, t0, m)
    tok = set(int(perm[q]) // k for q in rows)
    tok |= {0, 1, T - 1, min(255, T - 1), min(256, T - 1), max(T - 256, 0)}   # shared expert tiles
    g = torch.Generator().manual_seed(seed)
    extra = torch.randperm(T, generator=g).tolist()
    for t in extra:
        if len(tok) >= want:
            break
        tok.add(t)
    return torch.tensor(sorted(tok))


def train_loop_oracle(steps, lr=7.8125e-4, gamma=1e-3):
    """SGD on fp32 master weights (bf16 copies in the forward, as the layer
    stores them) towards a teacher layer's output, with the balancing-bias
    update after every step; returns the loss of each step."""
    from oracle import mrlmoe_backward as B
    s = W.CONFIGS["c0_tiny"]
    bf = lambda w: {k: v.to(torch.bfloat16) if v.dim() > 1 else v.float() for k, v in w.items()}
    master = {k: v.double() for k, v in W.make_weights(s, "cpu").items()}
    teacher = bf({k: v.double() for k, v in W.make_weights(s, "cpu", seed=5).items()})
    x = W.make_x(s, "cpu")
    bias = torch.zeros(s.n_experts)
    target = B.forward_for_grad(x, teacher, bias, s.top_k).y
    losses = []
    for _ in range(steps):
        w = bf(master)
        fc = B.forward_for_grad(x, w, bias, s.top_k)
        d = fc.y - target
        losses.append(0.5 * float((d * d).mean()))
        g = B.backward(fc, w, d.to(torch.bfloat16), s.top_k)
        for k in master:
            master[k] -= lr * g[k]
        bias = O.bias_update(bias, torch.bincount(fc.idx.flatten(), minlength=s.n_experts), s.T, s.top_k, gamma)
    return losses
