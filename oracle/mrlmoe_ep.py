"""Expert-parallel form of the layer (forward, and the backward of a training
step), plain CPU reference.

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
           "ep_forward", "exchange_bytes", "ep_backward"]


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


# ---------------------------------------------------------------------------
# backward (training step) in the expert-parallel layout
# ---------------------------------------------------------------------------
def ep_backward(xs: Sequence[torch.Tensor], dys: Sequence[torch.Tensor], weights: Dict[str, torch.Tensor],
                bias: torch.Tensor, top_k: int, rms_eps: float = 1e-6, aggregation: str = "mean"):
    """Gradients of sum_r <y_r, dy_r> with every rank holding its own tokens.

    Exchange plan (the forward's, run backwards): each token's rank computes
    dc (the RMSNorm and combine backward are per token) and sends, for every
    dispatch row, dc of the row's token and the row's weight w' to the
    expert's owner, in the same slices as the forward's latent rows.  The
    owner, from what it received (the forward's z rows and these), forms
    dh' = dc W_d, dw' = <h, dh'>, dg, du and dz = dg W_g + du W_u per row,
    accumulates its experts' weight gradients over all sources, and returns
    dz and dw' per row.  The token's rank finishes the router and alpha terms
    and dx.  Replicated tensors (projections, routers, gain, alpha, shared
    expert) get one partial gradient per rank, summed here as an all-reduce
    would; the routed experts' gradients are complete on their owner.

    Returns (per-rank dx list, dict of the summed gradients)."""
    from .mrlmoe_backward import forward_for_grad

    n = len(xs)
    f64 = lambda t: _as_f64(t)
    E = weights["expert_scale"].numel()
    alpha = f64(weights["expert_scale"])
    Wr = f64(weights["w_router"])
    R = Wr.shape[0]
    # forward on every rank (the kept activations a training forward leaves)
    fcs = [forward_for_grad(x, weights, bias, top_k, rms_eps, aggregation, round_points=True) for x in xs]
    recs = [route_and_dispatch(x, weights, bias, top_k, aggregation) for x in xs]
    grads = {k: torch.zeros(weights[k].shape, dtype=F64) for k in
             ("w_down", "w_router", "w_gate", "w_up_e", "w_down_e", "w_sh_gate", "w_sh_up", "w_sh_down",
              "rms_gain", "w_up", "expert_scale")}
    # 1) token side, up to dc, and the shared expert
    dcs, sends = [], []
    for s in range(n):
        fc, rec, dy = fcs[s], recs[s], f64(dys[s])
        dn = dy @ f64(weights["w_up"])
        grads["w_up"] += dy.T @ fc.n
        cn = fc.c * fc.r
        grads["rms_gain"] += (dn * cn).sum(0)
        dcn = dn * f64(weights["rms_gain"])[None, :]
        dc = fc.r * (dcn - cn * (cn * dcn).mean(1, keepdim=True))
        dcs.append(dc)
        flat = rec.perm
        tok, slot = flat // top_k, flat % top_k
        wrow = fc.ws[tok, slot]                      # w' per dispatch row (as the forward kept it)
        out = []
        for d in range(n):
            lo, hi = owned_range(E, n, d)
            a, b = int(rec.offsets[lo]), int(rec.offsets[hi])
            out.append((dc[tok[a:b]], wrow[a:b], rec.counts[lo:hi].clone()))
        sends.append(out)
    fwd_rows = [send_buffers(rec, n) for rec in recs]   # what each owner received in the forward
    # 2) owners
    back = [[None] * n for _ in range(n)]
    for d in range(n):
        lo, hi = owned_range(E, n, d)
        res = [(torch.zeros(sends[s][d][0].shape, dtype=F64), torch.zeros(sends[s][d][1].shape, dtype=F64))
               for s in range(n)]
        for s in range(n):
            z_rows, cnt = fwd_rows[s][d]
            dc_rows, w_rows, _ = sends[s][d]
            start = 0
            for e in range(lo, hi):
                m = int(cnt[e - lo])
                if m == 0:
                    continue
                z = z_rows[start:start + m]
                wg, wu, wd = f64(weights["w_gate"][e]), f64(weights["w_up_e"][e]), f64(weights["w_down_e"][e])
                g, u = z @ wg.T, z @ wu.T
                h = bf16_round(g / (1.0 + torch.exp(-g)) * u)
                dcr, wr_ = dc_rows[start:start + m], w_rows[start:start + m]
                dhp = dcr @ wd
                dws = (h * dhp).sum(1)
                dh = wr_[:, None] * dhp
                sg = 1.0 / (1.0 + torch.exp(-g))
                dg = dh * u * sg * (1.0 + g * (1.0 - sg))
                du = dh * (g * sg)
                grads["w_gate"][e] += dg.T @ z
                grads["w_up_e"][e] += du.T @ z
                grads["w_down_e"][e] += (wr_[:, None] * dcr).T @ h
                res[s][0][start:start + m] = dg @ wg + du @ wu
                res[s][1][start:start + m] = dws
                start += m
        for s in range(n):
            back[s][d] = res[s]
    # 3) token side: router, alpha, dx
    dxs = []
    for s in range(n):
        fc, rec, dc = fcs[s], recs[s], dcs[s]
        T, L = dc.shape
        dz_rows = torch.cat([back[s][d][0] for d in range(n)])
        dws_rows = torch.cat([back[s][d][1] for d in range(n)])
        flat = rec.perm
        tok = flat // top_k
        dz = torch.zeros(T, L, dtype=F64).index_add_(0, tok, dz_rows)
        # shared expert (replicated), on every token
        zs = fc.z
        gs, us = zs @ f64(weights["w_sh_gate"]).T, zs @ f64(weights["w_sh_up"]).T
        hs = bf16_round(gs / (1.0 + torch.exp(-gs)) * us)
        dhs = dc @ f64(weights["w_sh_down"])
        sgs = 1.0 / (1.0 + torch.exp(-gs))
        dgs = dhs * us * sgs * (1.0 + gs * (1.0 - sgs))
        dus = dhs * (gs * sgs)
        grads["w_sh_down"] += dc.T @ hs
        grads["w_sh_gate"] += dgs.T @ zs
        grads["w_sh_up"] += dus.T @ zs
        dz += dgs @ f64(weights["w_sh_gate"]) + dus @ f64(weights["w_sh_up"])
        # weights and routers
        dws = torch.zeros(T * top_k, dtype=F64)
        dws[flat] = dws_rows
        idxf = fc.idx.reshape(-1)
        grads["expert_scale"] += torch.zeros(E, dtype=F64).index_add_(0, idxf, fc.w.reshape(-1) * dws)
        dw = (dws * alpha[idxf]).view(T, top_k)
        S = fc.ssel.sum(1, keepdim=True)
        dssel = (dw - (fc.w * dw).sum(1, keepdim=True)) / S
        ds = torch.zeros(T, E, dtype=F64).scatter_add_(1, fc.idx, dssel)
        dzx = dz.clone()
        for r in range(R):
            if aggregation == "mean":
                dp = ds / R
            elif aggregation == "sum":
                dp = ds
            else:
                dp = torch.where(fc.rmax == r, ds, torch.zeros_like(ds))
            dl = dp * fc.p[r] * (1.0 - fc.p[r])
            grads["w_router"][r] += dl.T @ fc.zx
            dzx += dl @ Wr[r]
        dxs.append(dzx @ f64(weights["w_down"]))
        grads["w_down"] += dzx.T @ fc.x
    return dxs, grads
