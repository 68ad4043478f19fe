"""Expert-parallel form of the layer forward, plain CPU reference.

TEST INFRASTRUCTURE ONLY, like the rest of this package.

The pages motivate the latent design by what crosses between GPUs when the
experts are spread over them: tokens travel to the ranks that own their
experts in the 2048-d latent instead of the 4096-d hidden state, so the
dispatch and combine traffic is halved (derekhsu, "多路由潛在 MoE
(Multi-Router Latent MoE)"; aitest123, "模型结构").  They give no layout; the
readings taken here:

  * N ranks; rank d owns the routed experts [d E/N, (d+1) E/N) (E divisible
    by N).  The down-projection, the routers, the shared expert, RMSNorm and
    the up-projection are replicated; every rank runs them on its own tokens.
  * Each rank routes its own tokens and builds the single-GPU dispatch record
    (rows expert-major, tokens ascending).  The rows bound for rank d are then
    the contiguous slice offsets[dE/N] .. offsets[(d+1)E/N] of its dispatched
    latent rows, sent with the counts of d's experts: no packing step.
  * Rank d runs each of its experts on that expert's rows from every source
    (sources in rank order, rows in each source's order) and returns the
    unweighted outputs o, row for row, to their source.
  * The source scales each returned row by its weight w' and combines as the
    single-GPU layer does (the same order of additions), then applies the
    shared expert, RMSNorm and the up-projection.

Every expert sees the same row values as on one GPU, so the result equals
the single-GPU oracle up to the rounding of the expert products over a
different batch of rows (fp64).  The phases are separate functions so that a
test can run them as separate processes with a real all-to-all between them.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Sequence, Tuple

import torch

from .mrlmoe_oracle import (_as_f64, bf16_round, expert_glu, permutation, rmsnorm, route_weights, router_scores,
                            select_topk)

F64 = torch.float64

__all__ = ["owned_range", "RankRecord", "route_and_dispatch", "send_buffers", "run_local_experts", "combine",
           "ep_forward", "exchange_bytes"]


def owned_range(E: int, n_ranks: int, d: int) -> Tuple[int, int]:
    """Routed experts [lo, hi) of rank d: E / N consecutive experts."""
    if E % n_ranks:
        raise ValueError("the expert count must divide by the number of ranks")
    per = E // n_ranks
    return d * per, (d + 1) * per


@dataclass
class RankRecord:
    z: torch.Tensor        # [T, L] bf16 values (fp64)
    idx: torch.Tensor      # [T, k]
    wsc: torch.Tensor      # [T, k] w' (fp32)
    counts: torch.Tensor   # [E]
    offsets: torch.Tensor  # [E + 1]
    perm: torch.Tensor     # [T k] dispatch row -> t k + j
    rows: torch.Tensor     # [T k, L] dispatched latent rows (fp64 holding bf16 values)


def route_and_dispatch(x: torch.Tensor, weights: Dict[str, torch.Tensor], bias: torch.Tensor, top_k: int,
                       aggregation: str = "mean") -> RankRecord:
    """Steps 1-6 of the single-GPU layer on one rank's tokens."""
    zx = _as_f64(x) @ _as_f64(weights["w_down"]).T
    z = bf16_round(zx)
    s = router_scores(zx, weights["w_router"], aggregation)
    idx = select_topk(s, bias, top_k)
    _, wsc = route_weights(s, idx, weights["expert_scale"])
    counts, offsets, perm, _ = permutation(idx, weights["expert_scale"].numel())
    return RankRecord(z, idx, wsc, counts, offsets, perm, z[perm // top_k])


def send_buffers(rec: RankRecord, n_ranks: int) -> List[Tuple[torch.Tensor, torch.Tensor]]:
    """Per destination rank d: (its slice of the dispatched rows, the row
    counts of d's experts)."""
    E = rec.counts.numel()
    out = []
    for d in range(n_ranks):
        lo, hi = owned_range(E, n_ranks, d)
        a, b = int(rec.offsets[lo]), int(rec.offsets[hi])
        out.append((rec.rows[a:b], rec.counts[lo:hi].clone()))
    return out


def run_local_experts(d: int, n_ranks: int, recv: Sequence[Tuple[torch.Tensor, torch.Tensor]],
                      weights: Dict[str, torch.Tensor]) -> List[torch.Tensor]:
    """Rank d: recv[s] = (rows, per-local-expert counts) from source s.  Each
    local expert runs once on its rows from all sources; the outputs go back
    per source, in the order the rows came."""
    E = weights["expert_scale"].numel()
    lo, hi = owned_range(E, n_ranks, d)
    L = weights["w_down_e"].shape[1]
    outs = [torch.zeros(r.shape[0], L, dtype=F64) for r, _ in recv]
    starts = [torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(c, 0)]) for _, c in recv]
    for e in range(lo, hi):
        pieces, where = [], []
        for s, (rows, cnt) in enumerate(recv):
            a, n = int(starts[s][e - lo]), int(cnt[e - lo])
            if n:
                pieces.append(rows[a:a + n])
                where.append((s, a, n))
        if not pieces:
            continue
        o = expert_glu(torch.cat(pieces), weights["w_gate"][e], weights["w_up_e"][e], weights["w_down_e"][e])
        i = 0
        for s, a, n in where:
            outs[s][a:a + n] = o[i:i + n]
            i += n
    return outs


def combine(rec: RankRecord, returned: Sequence[torch.Tensor], weights: Dict[str, torch.Tensor], top_k: int,
            rms_eps: float = 1e-6) -> Dict[str, torch.Tensor]:
    """The source rank: returned[d] = outputs for the rows it sent to d.  The
    rows are in dispatch order again; each is scaled by its w' and added to its
    token in that order (the single-GPU oracle's order), then the shared
    expert, RMSNorm and the up-projection."""
    o = torch.cat(list(returned)) if len(returned) else torch.zeros(0)
    T, L = rec.z.shape
    c = torch.zeros(T, L, dtype=F64)
    E = rec.counts.numel()
    for e in range(E):
        a, b = int(rec.offsets[e]), int(rec.offsets[e + 1])
        if a == b:
            continue
        flat = rec.perm[a:b]
        tok, slot = flat // top_k, flat % top_k
        c.index_add_(0, tok, o[a:b] * rec.wsc[tok, slot].to(F64)[:, None])
    c += expert_glu(rec.z, weights["w_sh_gate"], weights["w_sh_up"], weights["w_sh_down"])
    n = bf16_round(rmsnorm(c, weights["rms_gain"], rms_eps))
    y = bf16_round(n @ _as_f64(weights["w_up"]).T)
    return {"c": c, "n": n, "y": y}


def ep_forward(xs: Sequence[torch.Tensor], weights: Dict[str, torch.Tensor], bias: torch.Tensor, top_k: int,
               rms_eps: float = 1e-6, aggregation: str = "mean"):
    """All ranks in one process: the two all-to-alls are list transposes."""
    n = len(xs)
    recs = [route_and_dispatch(x, weights, bias, top_k, aggregation) for x in xs]
    sends = [send_buffers(r, n) for r in recs]
    back = [[None] * n for _ in range(n)]
    for d in range(n):
        outs = run_local_experts(d, n, [sends[s][d] for s in range(n)], weights)
        for s in range(n):
            back[s][d] = outs[s]
    return [combine(recs[s], back[s], weights, top_k, rms_eps) for s in range(n)], recs


def exchange_bytes(recs: Sequence[RankRecord], n_ranks: int, width: int, elem_bytes: int = 2) -> Dict[str, int]:
    """Bytes that cross between ranks in one dispatch (and again in the
    combine), rows of `width` elements: only rows whose expert lives on
    another rank count."""
    remote = local = 0
    for s, rec in enumerate(recs):
        for d, (rows, _) in enumerate(send_buffers(rec, n_ranks)):
            if d == s:
                local += rows.shape[0]
            else:
                remote += rows.shape[0]
    return {"remote_rows": remote, "local_rows": local, "bytes": remote * width * elem_bytes}
