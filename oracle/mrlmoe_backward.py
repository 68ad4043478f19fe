"""Plain fp64 CPU definition of the backward pass of the Multi-Router Latent MoE
layer: the gradients of a loss <y, dy> with respect to the layer's input and
every learnable tensor, written out step by step (no automatic
differentiation).

TEST INFRASTRUCTURE ONLY, like the forward oracle in this package.

The pages describe a model trained with this layer (the release blog's
"多路由潛在 MoE (Multi-Router Latent MoE)" section of blog.derekhsu.net:
the multi-router design is motivated by how the routers learn) but give no
formula for its gradients.  The readings taken here (each an assumption):
  * the bf16 rounding points of the forward (z, h, n, y) and the fp32 score
    pass gradients through unchanged (the rounding belongs to storage; the
    gradient is computed in higher precision);
  * the top-k selection is a discrete choice: no gradient flows through it;
    the selected experts' scores receive gradient through the renormalised
    weights w_j = s_j / sum_j s_j;
  * the balancing bias b receives no gradient (it moves by the count rule);
  * the per-expert scalar alpha and the RMSNorm gain are learnable;
  * "max" aggregation passes the score's gradient to the router attaining
    the maximum (the lowest-numbered one on ties);
  * the routers read the unrounded latent x W_dn^T, the experts its bf16
    rounding z; both paths send gradient back to x W_dn^T.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict

import torch

from .mrlmoe_oracle import bf16_round, select_topk

F64 = torch.float64
F32 = torch.float32

__all__ = ["ForwardCache", "forward_for_grad", "backward", "GRAD_NAMES"]

GRAD_NAMES = ("x", "w_down", "w_router", "w_gate", "w_up_e", "w_down_e", "w_sh_gate", "w_sh_up",
              "w_sh_down", "rms_gain", "w_up", "expert_scale")


def _f(t: torch.Tensor) -> torch.Tensor:
    return t.to(F64)


def _round(v: torch.Tensor, on: bool) -> torch.Tensor:
    return bf16_round(v) if on else v


@dataclass
class ForwardCache:
    x: torch.Tensor        # [T, D]
    zx: torch.Tensor       # [T, L] unrounded latent (router input)
    z: torch.Tensor        # [T, L] expert input (bf16 values when rounding)
    p: torch.Tensor        # [R, T, E] router sigmoids
    s: torch.Tensor        # [T, E] aggregated scores (as used for the weights)
    rmax: torch.Tensor     # [T, E] index of the router attaining the max (max aggregation)
    idx: torch.Tensor      # [T, k] selected experts
    ssel: torch.Tensor     # [T, k] their scores
    w: torch.Tensor        # [T, k] renormalised weights (before alpha)
    ws: torch.Tensor       # [T, k] w * alpha
    g: Dict[int, torch.Tensor]   # per expert e (and -1: shared): gate pre-activations of its rows
    u: Dict[int, torch.Tensor]
    h: Dict[int, torch.Tensor]
    o: Dict[int, torch.Tensor]
    rows: Dict[int, torch.Tensor]  # flat (t*k + j) indices of expert e's rows, ascending
    c: torch.Tensor        # [T, L] combined output
    r: torch.Tensor        # [T, 1] 1 / sqrt(mean(c^2) + eps)
    n: torch.Tensor        # [T, L]
    y: torch.Tensor        # [T, D]


def forward_for_grad(x: torch.Tensor, w: Dict[str, torch.Tensor], bias: torch.Tensor, top_k: int,
                     rms_eps: float = 1e-6, aggregation: str = "mean", round_points: bool = True) -> ForwardCache:
    """The layer forward of the oracle, keeping what the backward needs.
    With round_points the bf16/fp32 rounding points are applied as in the
    forward oracle; without them every step stays in fp64 (the form the
    finite-difference pins differentiate)."""
    xf = _f(x)
    zx = xf @ _f(w["w_down"]).T
    z = _round(zx, round_points)
    wr = _f(w["w_router"])
    R = wr.shape[0]
    p = torch.stack([1.0 / (1.0 + torch.exp(-(zx @ wr[r].T))) for r in range(R)])
    rmax = torch.argmax(p, dim=0)          # first maximum on ties
    if aggregation == "mean":
        s = p.sum(0) / R
    elif aggregation == "sum":
        s = p.sum(0)
    elif aggregation == "max":
        s = p.max(0).values
    else:
        raise ValueError(aggregation)
    if round_points:
        s = s.to(F32).to(F64)
    idx = select_topk(s.to(F32), bias, top_k)
    ssel = torch.gather(s, 1, idx)
    den = ssel.sum(1, keepdim=True)
    # a zero sum of the selected scores gives the uniform weights 1/k
    wgt = torch.where(den == 0, torch.full_like(ssel, 1.0 / top_k), ssel / torch.where(den == 0, 1.0, den))
    ws = wgt * _f(w["expert_scale"])[idx]
    T, L = z.shape
    E = w["expert_scale"].numel()
    flat = idx.reshape(-1)
    gd, ud, hd, od, rowsd = {}, {}, {}, {}, {}
    c = torch.zeros(T, L, dtype=F64)
    for e in list(range(E)) + [-1]:
        if e >= 0:
            rows = torch.nonzero(flat == e).flatten()
            if rows.numel() == 0:
                continue
            zr = z[rows // top_k]
            wg, wu, wd = _f(w["w_gate"][e]), _f(w["w_up_e"][e]), _f(w["w_down_e"][e])
        else:
            rows = torch.arange(T)
            zr = z
            wg, wu, wd = _f(w["w_sh_gate"]), _f(w["w_sh_up"]), _f(w["w_sh_down"])
        g = zr @ wg.T
        u = zr @ wu.T
        h = _round(g / (1.0 + torch.exp(-g)) * u, round_points)
        o = h @ wd.T
        gd[e], ud[e], hd[e], od[e], rowsd[e] = g, u, h, o, rows
        if e >= 0:
            c.index_add_(0, rows // top_k, o * ws.reshape(-1)[rows][:, None])
        else:
            c += o
    r = 1.0 / torch.sqrt((c * c).mean(1, keepdim=True) + rms_eps)
    n = _round(c * r * _f(w["rms_gain"])[None, :], round_points)
    y = _round(n @ _f(w["w_up"]).T, round_points)
    return ForwardCache(xf, zx, z, p, s, rmax, idx, ssel, wgt, ws, gd, ud, hd, od, rowsd, c, r, n, y)


def backward(fc: ForwardCache, w: Dict[str, torch.Tensor], dy: torch.Tensor, top_k: int,
             aggregation: str = "mean", experts=None) -> Dict[str, torch.Tensor]:
    """Gradients of sum(y * dy) for the names in GRAD_NAMES (fp64).

    ``experts`` (a list of routed expert indices) limits the routed experts'
    weight gradients to those experts, stacked in that order (the full
    tensors at full width do not fit a host's memory in fp64); every other
    gradient is complete either way."""
    sel = None if experts is None else [int(e) for e in experts]
    slot_of = None if sel is None else {e: i for i, e in enumerate(sel)}
    dy = _f(dy)
    gain = _f(w["rms_gain"])
    alpha = _f(w["expert_scale"])
    T, L = fc.c.shape
    E = alpha.numel()
    grads: Dict[str, torch.Tensor] = {}
    # y = n W_up^T
    dn = dy @ _f(w["w_up"])
    grads["w_up"] = dy.T @ fc.n
    # n = (c r) * gain, r = (mean(c^2) + eps)^-1/2
    cn = fc.c * fc.r
    grads["rms_gain"] = (dn * cn).sum(0)
    dcn = dn * gain[None, :]
    dc = fc.r * (dcn - cn * (cn * dcn).mean(1, keepdim=True))
    # c = sum_j ws_j o_j + o_shared
    dws = torch.zeros(T * top_k, dtype=F64)
    dz = torch.zeros(T, L, dtype=F64)
    ne = E if sel is None else len(sel)
    shapes = {"w_gate": (ne,) + tuple(w["w_gate"].shape[1:]), "w_up_e": (ne,) + tuple(w["w_up_e"].shape[1:]),
              "w_down_e": (ne,) + tuple(w["w_down_e"].shape[1:])}
    for nm, shp in shapes.items():
        grads[nm] = torch.zeros(shp, dtype=F64)
    for e, rows in fc.rows.items():
        tok = rows // top_k if e >= 0 else rows
        o, h, g, u = fc.o[e], fc.h[e], fc.g[e], fc.u[e]
        if e >= 0:
            do = dc[tok] * fc.ws.reshape(-1)[rows][:, None]
            dws[rows] = (o * dc[tok]).sum(1)
            wg, wu, wd = _f(w["w_gate"][e]), _f(w["w_up_e"][e]), _f(w["w_down_e"][e])
        else:
            do = dc
            wg, wu, wd = _f(w["w_sh_gate"]), _f(w["w_sh_up"]), _f(w["w_sh_down"])
        # o = h W_d^T; h = SiLU(g) * u; g = z W_g^T, u = z W_u^T
        dh = do @ wd
        dwd = do.T @ h
        sg = 1.0 / (1.0 + torch.exp(-g))
        dg = dh * u * sg * (1.0 + g * (1.0 - sg))
        du = dh * (g * sg)
        zr = fc.z[tok]
        dwg, dwu = dg.T @ zr, du.T @ zr
        dz.index_add_(0, tok, dg @ wg + du @ wu)
        if e >= 0:
            if slot_of is None or e in slot_of:
                i = e if slot_of is None else slot_of[e]
                grads["w_gate"][i], grads["w_up_e"][i], grads["w_down_e"][i] = dwg, dwu, dwd
        else:
            grads["w_sh_gate"], grads["w_sh_up"], grads["w_sh_down"] = dwg, dwu, dwd
    for nm in ("w_sh_gate", "w_sh_up", "w_sh_down"):
        grads.setdefault(nm, torch.zeros(w[nm].shape, dtype=F64))
    # ws_j = w_j * alpha[e_j]
    flat = fc.idx.reshape(-1)
    dw = dws * alpha[flat]
    grads["expert_scale"] = torch.zeros(E, dtype=F64).index_add_(0, flat, fc.w.reshape(-1) * dws)
    # w_j = s_j / S over the selected experts
    dw = dw.view(T, top_k)
    S = fc.ssel.sum(1, keepdim=True)
    # where the selected scores sum to 0 the weights are the constant 1/k: no gradient
    dssel = torch.where(S == 0, 0.0, (dw - (fc.w * dw).sum(1, keepdim=True)) / torch.where(S == 0, 1.0, S))
    ds = torch.zeros(T, E, dtype=F64).scatter_add_(1, fc.idx, dssel)
    # s = agg_r sigmoid(l_r), l_r = zx W_r^T
    wr = _f(w["w_router"])
    R = wr.shape[0]
    dzx = dz.clone()  # the experts' input z is zx rounded: the gradient passes through
    dwr = torch.zeros(wr.shape, dtype=F64)
    for r in range(R):
        if aggregation == "mean":
            dp = ds / R
        elif aggregation == "sum":
            dp = ds
        else:
            dp = torch.where(fc.rmax == r, ds, torch.zeros_like(ds))
        dl = dp * fc.p[r] * (1.0 - fc.p[r])
        dwr[r] = dl.T @ fc.zx
        dzx += dl @ wr[r]
    grads["w_router"] = dwr
    # zx = x W_dn^T
    grads["x"] = dzx @ _f(w["w_down"])
    grads["w_down"] = dzx.T @ fc.x
    return grads
