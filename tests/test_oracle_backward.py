"""Pins of the oracle's backward definition (CPU only).

The backward is written out by hand; these tests hold it against things that
do not share its arithmetic:
  * central finite differences of the forward, per learnable tensor, along a
    random direction (fp64, unrounded form, the top-k selection checked to stay
    the same at both probe points);
  * Euler's theorem on the parts of the layer that are homogeneous: y is linear
    in W_up and in the RMSNorm gain, and (with eps = 0) the normalised output
    does not change when every expert's output matrix is scaled together;
  * the straight-through reading: with the rounding points applied, the
    gradient stays close to the unrounded one;
  * the forward kept for the backward agrees with the forward oracle.
"""
import pytest
import torch

from helpers import train_loop_oracle
from oracle import mrlmoe_backward as B
from oracle import mrlmoe_oracle as O

F64 = torch.float64


def _params(T=5, D=8, L=8, E=6, F=4, R=2, seed=0):
    g = torch.Generator().manual_seed(seed)

    def nrm(*shape, std=1.0):
        return torch.randn(*shape, generator=g, dtype=F64) * std

    w = {
        "w_down": nrm(L, D, std=D ** -0.5),
        "w_router": nrm(R, E, L, std=2.0 * L ** -0.5),
        "w_gate": nrm(E, F, L, std=L ** -0.5),
        "w_up_e": nrm(E, F, L, std=L ** -0.5),
        "w_down_e": nrm(E, L, F, std=F ** -0.5),
        "w_sh_gate": nrm(F, L, std=L ** -0.5),
        "w_sh_up": nrm(F, L, std=L ** -0.5),
        "w_sh_down": nrm(L, F, std=F ** -0.5),
        "w_up": nrm(D, L, std=L ** -0.5),
        "rms_gain": 1.0 + 0.3 * nrm(L),
        "expert_scale": 0.5 + torch.rand(E, generator=g, dtype=F64),
    }
    x = nrm(T, D)
    dy = nrm(T, D)
    bias = 0.01 * torch.randn(E, generator=g, dtype=torch.float32)
    return x, w, bias, dy


def _loss(x, w, bias, dy, k, agg, eps):
    fc = B.forward_for_grad(x, w, bias, k, rms_eps=eps, aggregation=agg, round_points=False)
    return float((fc.y * dy).sum()), fc.idx


CASES = [  # (T, D, L, E, F, R, k, aggregation, seed)
    (5, 8, 8, 6, 4, 2, 2, "mean", 1),
    (7, 8, 8, 6, 4, 3, 3, "sum", 2),
    (6, 8, 8, 6, 4, 3, 2, "max", 3),
    (4, 8, 8, 5, 4, 1, 5, "mean", 4),     # k = E: every expert selected
    (9, 12, 8, 8, 6, 2, 1, "mean", 5),    # k = 1: weight 1 for the chosen expert
    (3, 8, 8, 16, 4, 2, 2, "mean", 6),    # experts without rows
]


@pytest.mark.parametrize("case", CASES)
def test_finite_differences(case):
    T, D, L, E, F, R, k, agg, seed = case
    x, w, bias, dy = _params(T, D, L, E, F, R, seed)
    eps = 1e-6
    fc = B.forward_for_grad(x, w, bias, k, rms_eps=eps, aggregation=agg, round_points=False)
    grads = B.backward(fc, w, dy, k, aggregation=agg)
    assert set(grads) == set(B.GRAD_NAMES)
    g = torch.Generator().manual_seed(100 + seed)
    h = 1e-6
    for name in B.GRAD_NAMES:
        base = x if name == "x" else w[name]
        assert grads[name].shape == base.shape, name
        v = torch.randn(base.shape, generator=g, dtype=F64)
        vals, sel = [], []
        for sgn in (1.0, -1.0):
            if name == "x":
                lv, idx = _loss(x + sgn * h * v, w, bias, dy, k, agg, eps)
            else:
                wp = dict(w)
                wp[name] = base + sgn * h * v
                lv, idx = _loss(x, wp, bias, dy, k, agg, eps)
            vals.append(lv)
            sel.append(idx)
        assert torch.equal(sel[0], fc.idx) and torch.equal(sel[1], fc.idx), f"selection moved ({name})"
        fd = (vals[0] - vals[1]) / (2 * h)
        an = float((grads[name] * v).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


@pytest.mark.parametrize("case", CASES)
def test_homogeneity(case):
    T, D, L, E, F, R, k, agg, seed = case
    x, w, bias, dy = _params(T, D, L, E, F, R, seed)
    fc = B.forward_for_grad(x, w, bias, k, rms_eps=0.0, aggregation=agg, round_points=False)
    grads = B.backward(fc, w, dy, k, aggregation=agg)
    loss = float((fc.y * dy).sum())
    # y = n W_up^T is linear in W_up; n is linear in the gain
    assert abs(float((grads["w_up"] * w["w_up"]).sum()) - loss) < 1e-10 * max(1.0, abs(loss))
    assert abs(float((grads["rms_gain"] * w["rms_gain"]).sum()) - loss) < 1e-10 * max(1.0, abs(loss))
    # c is linear in the output matrices of all experts together; RMSNorm with
    # eps = 0 removes that scale, so the directional derivative is zero
    tot = float((grads["w_down_e"] * w["w_down_e"]).sum() + (grads["w_sh_down"] * w["w_sh_down"]).sum())
    scale = float(grads["w_down_e"].abs().sum() + grads["w_sh_down"].abs().sum())
    assert abs(tot) < 1e-12 * max(1.0, scale)


def test_alpha_scale_invariance_without_shared_expert():
    # with the shared expert switched off, c is linear in alpha and the
    # eps = 0 norm removes it: <dL/dalpha, alpha> = 0
    x, w, bias, dy = _params(seed=7)
    w = dict(w)
    w["w_sh_down"] = torch.zeros_like(w["w_sh_down"])
    fc = B.forward_for_grad(x, w, bias, 2, rms_eps=0.0, round_points=False)
    g = B.backward(fc, w, dy, 2)
    assert abs(float((g["expert_scale"] * w["expert_scale"]).sum())) < 1e-12 * float(g["expert_scale"].abs().sum())
    # and the weights' renormalisation makes the scores' scale irrelevant to y:
    # the routers' gradient then only comes through the ratios, not through a
    # common factor (no closed form to compare, but it is finite and nonzero)
    assert torch.isfinite(g["w_router"]).all() and g["w_router"].abs().sum() > 0


def test_k_equals_one_gives_no_router_gradient():
    # with k = 1 the renormalised weight is exactly 1 whatever the score, so no
    # gradient reaches the routers
    x, w, bias, dy = _params(T=9, D=12, E=8, F=6, seed=5)
    fc = B.forward_for_grad(x, w, bias, 1, round_points=False)
    g = B.backward(fc, w, dy, 1)
    assert torch.all(fc.w == 1.0)
    assert float(g["w_router"].abs().max()) < 1e-14


def test_unselected_experts_get_no_gradient():
    x, w, bias, dy = _params(T=3, E=16, seed=6)
    fc = B.forward_for_grad(x, w, bias, 2, round_points=False)
    g = B.backward(fc, w, dy, 2)
    used = set(fc.idx.flatten().tolist())
    assert len(used) < 16
    for e in range(16):
        for nm in ("w_gate", "w_up_e", "w_down_e"):
            nz = bool(g[nm][e].abs().sum() > 0)
            assert nz == (e in used), (nm, e)


def test_rounded_gradient_close_to_unrounded():
    x, w, bias, dy = _params(T=16, D=16, L=16, E=8, F=8, R=2, seed=11)
    fu = B.forward_for_grad(x, w, bias, 2, round_points=False)
    fr = B.forward_for_grad(x, w, bias, 2, round_points=True)
    assert torch.equal(fu.idx, fr.idx)
    gu, gr = B.backward(fu, w, dy, 2), B.backward(fr, w, dy, 2)
    for nm in B.GRAD_NAMES:
        num = float((gu[nm] - gr[nm]).norm())
        den = float(gu[nm].norm())
        assert num <= 0.05 * den + 1e-12, (nm, num, den)


def test_kept_forward_matches_the_forward_oracle():
    x, w, bias, dy = _params(T=16, D=16, L=16, E=8, F=8, R=2, seed=12)
    w32 = {n: t.to(torch.float32) for n, t in w.items()}
    ref = O.forward(x.to(torch.float32), w32, bias, 2)
    fc = B.forward_for_grad(x.to(torch.float32), w32, bias, 2, round_points=True)
    assert torch.equal(fc.idx, ref.topk_idx)
    assert torch.allclose(fc.s.to(torch.float32), ref.s)
    assert torch.allclose(fc.z, ref.z)
    # the forward oracle keeps w and w * alpha in fp32, this one in fp64: the
    # difference is a few fp32 steps of |o| ~ 1
    assert torch.allclose(fc.c, ref.c, rtol=1e-6, atol=1e-6)
    # n and y are bf16 values: allow one bf16 step where fp32 vs fp64 weights
    # moved a value across a rounding boundary
    assert torch.allclose(fc.n, ref.n, rtol=2 ** -7, atol=1e-6)
    assert torch.allclose(fc.y, ref.y, rtol=2 ** -6, atol=1e-3)


def test_gradient_descent_lowers_the_loss():
    # the oracle's gradients, used as a training step, lower the loss at every step
    losses = train_loop_oracle(12)
    assert all(b < a for a, b in zip(losses, losses[1:])), losses
    assert losses[-1] < 0.2 * losses[0], losses


def test_expert_subset_equals_the_full_gradients():
    # the memory-saving `experts` option computes the same numbers, stacked in the given order
    x, w, bias, dy = _params(T=6, E=8, seed=9)
    fc = B.forward_for_grad(x, w, bias, 2, round_points=False)
    full = B.backward(fc, w, dy, 2)
    pick = [5, 0, 3, 7]
    sub = B.backward(fc, w, dy, 2, experts=pick)
    for nm in ("w_gate", "w_up_e", "w_down_e"):
        assert torch.equal(sub[nm], full[nm][pick]), nm
    for nm in set(B.GRAD_NAMES) - {"w_gate", "w_up_e", "w_down_e"}:
        assert torch.equal(sub[nm], full[nm]), nm


def _autograd_loss(x, w, idx, top_k, eps, aggregation):
    """The layer written again, densely (every expert on every token, masked
    by the given selection), differentiable by torch.autograd; fp64, no
    rounding points."""
    zx = x @ w["w_down"].T
    logits = torch.einsum("tl,rel->rte", zx, w["w_router"])
    p = torch.sigmoid(logits)
    if aggregation == "mean":
        s = p.mean(0)
    elif aggregation == "sum":
        s = p.sum(0)
    else:
        s = p.max(0).values
    T, E = s.shape
    mask = torch.zeros(T, E, dtype=F64)
    mask.scatter_(1, idx, 1.0)
    ssel = s * mask
    wts = ssel / ssel.sum(1, keepdim=True) * w["expert_scale"][None, :]   # zero off the selection
    g = torch.einsum("tl,efl->tef", zx, w["w_gate"])
    u = torch.einsum("tl,efl->tef", zx, w["w_up_e"])
    o = torch.einsum("tef,elf->tel", torch.nn.functional.silu(g) * u, w["w_down_e"])
    c = (o * wts[:, :, None]).sum(1)
    gs, us = zx @ w["w_sh_gate"].T, zx @ w["w_sh_up"].T
    c = c + (torch.nn.functional.silu(gs) * us) @ w["w_sh_down"].T
    n = c * torch.rsqrt((c * c).mean(1, keepdim=True) + eps) * w["rms_gain"][None, :]
    return n @ w["w_up"].T


@pytest.mark.parametrize("case", CASES)
def test_matches_automatic_differentiation(case):
    T, D, L, E, F, R, k, agg, seed = case
    x, w, bias, dy = _params(T, D, L, E, F, R, seed)
    eps = 1e-6
    fc = B.forward_for_grad(x, w, bias, k, rms_eps=eps, aggregation=agg, round_points=False)
    grads = B.backward(fc, w, dy, k, aggregation=agg)
    xa = x.clone().requires_grad_(True)
    wa = {n: t.clone().requires_grad_(True) for n, t in w.items()}
    y = _autograd_loss(xa, wa, fc.idx, k, eps, agg)
    assert torch.allclose(y, fc.y, rtol=1e-12, atol=1e-12)
    (y * dy).sum().backward()
    for name in B.GRAD_NAMES:
        ref = xa.grad if name == "x" else wa[name].grad
        d = (grads[name] - ref).abs().max().item()
        assert d <= 1e-10 * max(1.0, ref.abs().max().item()), (name, d)
