"""Plain, slow, fp64 CPU definition of the Multi-Router Latent MoE layer forward.

TEST INFRASTRUCTURE ONLY (see the package docstring): tests, the smoke check
and the CPU-baseline leg of the benchmark use it; the CUDA product path does not.

Sources (the ERNIE 5.5 Flash release pages):
  [derekhsu]  blog.derekhsu.net, "ERNIE-5.5-Flash-Base" full translation,
              section "多路由潛在 MoE (Multi-Router Latent MoE)": several
              independently initialised sigmoid routers score the experts
              together; 512 routed experts (top-10) plus 1 shared expert;
              aux-loss-free bias-corrected balancing; tokens projected
              4096 -> 2048, experts (intermediate 2048) run in the latent space,
              a shared up-projection maps back to 4096; Stable LatentMoE:
              RMSNorm before the up-projection, gated activation (printed
              "SiTU-GLU", read here as SiLU-GLU); each routed expert multiplies
              its routing weight by a learnable scalar.
  [aitest123] aitest123.com, "ERNIE-5.5-Flash-Base开源：280B总参数，激活仅14B",
              section "模型结构": the routers' scores are aggregated; experts
              compute in the 2048-d latent space.
  [knowflow]  knowflowhub.com release digest, table "关键信息", row "专家路由":
              the routers decide together in the 2048-d latent space.
  [lininn]    lininn.cn, "2800 亿参数的模型，每次只叫醒 140 亿", section
              "路由器，不止一个": balancing by bias correction, no auxiliary loss.

Readings where the pages leave a step open (each is an assumption, listed in
the design notes):
  * aggregation = mean of the R sigmoid scores; R is a parameter (4 at full width);
  * router input is the latent z; routers have no bias of their own;
  * the selection bias b enters selection only; weights use the unbiased s;
  * weights are renormalised over the k selected experts, then x alpha[e];
  * ties in selection go to the lower expert index (IEEE equality, +0 == -0);
  * shared expert: routed-expert shape, weight 1, no alpha, latent space;
  * RMSNorm eps 1e-6 with a learnable gain; no norm after the down-projection;
  * bias update b += gamma * sign(T*k - E*count[e]) with sign(0) = 0;
  * rounding points: z, h, n, y are bf16 (round to nearest even);
    s, w fp32; everything else fp64;
  * FP8 variant: every GEMM input is a bf16 tensor (x, z, h, n) quantised
    per 1x128 block from those bf16 values; weights are e4m3 codes with fp32
    scales per 128x128 block;
  * the routers read the latent before its bf16 rounding (the experts read
    bf16 z), so that top-k decisions do not hinge on bf16 rounding of z.
PARITY UNPINNED by the pages: the choice of mean (vs sum/max), R=4, eps, gamma.
Those are stated assumptions; the tests pin only the arithmetic under them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

__all__ = [
    "bf16_round", "linear_bf16", "router_scores", "select_topk", "route_weights",
    "permutation", "expert_glu", "rmsnorm", "forward", "bias_update",
    "e4m3_decode", "e4m3_encode", "quantize_act_1x128", "dequantize_weight_128x128",
    "e2m1_decode", "unpack_e2m1", "dequantize_weight_fp4_128x128", "FP4_MATRICES",
    "OracleResult", "topk_boundary_gap",
]

F64 = torch.float64
F32 = torch.float32


# ---------------------------------------------------------------------------
# rounding
# ---------------------------------------------------------------------------
def bf16_round(v: torch.Tensor) -> torch.Tensor:
    """Round float64 values to the nearest bf16 (ties to even); returns float64.

    bf16 keeps the float64 sign and an 8-bit exponent with 7 stored mantissa
    bits, so for values in bf16's normal range the 45 low mantissa bits of the
    float64 pattern are rounded away directly (no double rounding through
    fp32).  Magnitudes below 2^-126 (bf16 subnormals) go through torch's
    conversion; they do not occur in this layer's workloads.
    """
    v = v.to(F64).contiguous()
    bits = v.view(torch.int64)
    lsb = (bits >> 45) & 1
    rnd = (bits + ((1 << 44) - 1) + lsb) & ~((1 << 45) - 1)
    out = rnd.view(F64).clone()
    tiny = v.abs() < 2.0 ** -126
    if bool(tiny.any()):
        out[tiny] = v[tiny].to(F32).to(torch.bfloat16).to(F64)
    return out


def _as_f64(t: torch.Tensor) -> torch.Tensor:
    return t.to(F64)


def linear_bf16(a: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    """bf16(a @ w^T) with fp64 accumulation: the down-projection (4096 -> 2048)
    and the shared up-projection (2048 -> 4096) of [derekhsu].  w is [out, in]."""
    return bf16_round(_as_f64(a) @ _as_f64(w).T)


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------
def router_scores(z: torch.Tensor, w_router: torch.Tensor, aggregation: str = "mean") -> torch.Tensor:
    """s[t, e] = fp32( agg_r sigmoid(z[t] . w_router[r, e]) ), agg over the R
    routers: "mean" (1/R) sum_r, "sum" sum_r, or "max" max_r (in fp64, one
    rounding to fp32 at the end).

    R independently initialised sigmoid routers score every expert from the
    latent z [derekhsu; knowflow "关键信息"]; their scores are aggregated
    [aitest123 "模型结构"] by a rule the pages do not give: the mean is the
    layer's reading, sum and max are the alternatives it is compared with.
    """
    if aggregation not in ("mean", "sum", "max"):
        raise ValueError(f"unknown aggregation {aggregation!r}")
    z64 = _as_f64(z)
    R = w_router.shape[0]
    acc = torch.zeros(z.shape[0], w_router.shape[1], dtype=F64)
    for r in range(R):
        logit = z64 @ _as_f64(w_router[r]).T
        p = 1.0 / (1.0 + torch.exp(-logit))
        acc = torch.maximum(acc, p) if aggregation == "max" else acc + p
    return (acc / R if aggregation == "mean" else acc).to(F32)


def select_topk(s: torch.Tensor, bias: torch.Tensor, k: int) -> torch.Tensor:
    """Top-k experts per token by the biased score sb = fp32(s + b).

    The bias corrects load without an auxiliary loss and acts on selection
    only [derekhsu; lininn].  Order: a stable sort of (-sb, e) ascending, i.e.
    descending biased score, ties to the lower index (IEEE equality, so +0 and
    -0 tie).  Returns int64 [T, k] in that order.
    """
    sb = (s.to(F32) + bias.to(F32)[None, :]).numpy()
    E = sb.shape[1]
    eidx = np.broadcast_to(np.arange(E), sb.shape)
    order = np.lexsort((eidx, -sb), axis=-1)
    return torch.from_numpy(np.ascontiguousarray(order[:, :k])).to(torch.int64)


def topk_boundary_gap(s: torch.Tensor, bias: torch.Tensor, k: int) -> torch.Tensor:
    """sb_(k) - sb_(k+1) per token (fp64): the margin of the k-th selection."""
    sb = (s.to(F32) + bias.to(F32)[None, :]).to(F64)
    top = torch.sort(sb, dim=1, descending=True).values
    return top[:, k - 1] - top[:, k]


def route_weights(s: torch.Tensor, idx: torch.Tensor, alpha: torch.Tensor):
    """w_j = s_j / sum_j s_j over the selected experts (fp32, summed in slot
    order j = 0..k-1), then w'_j = w_j * alpha[e_j] (fp32).

    Renormalisation over the selected experts is an assumption; the per-expert
    learnable scalar multiplies the routing weight [derekhsu, Stable LatentMoE].
    The renormalisation is undefined when the selected scores sum to 0 (every
    selected sigmoid underflowed to 0 in fp32); the weights are then taken as
    the uniform fp32(1/k), the limit of equal scores.
    Returns (w, w_scaled), both fp32 [T, k].
    """
    ssel = torch.gather(s.to(F32), 1, idx)
    k = idx.shape[1]
    den = ssel[:, 0].clone()
    for j in range(1, k):
        den = den + ssel[:, j]
    zero = den == 0
    w = ssel / torch.where(zero, torch.ones_like(den), den)[:, None]
    w = torch.where(zero[:, None], torch.tensor(1.0, dtype=F32) / k, w)
    return w, w * alpha.to(F32)[idx]


def permutation(idx: torch.Tensor, n_experts: int):
    """Dispatch record: counts[E], offsets[E+1] (exclusive), perm[T*k]
    (row -> t*k + j) and inv_perm[T*k] ((t, j) -> row).

    Rows are grouped by expert in expert order; inside an expert, entries keep
    ascending token order: a stable sort of the flat (t, j) list by expert.
    """
    flat = idx.reshape(-1).numpy()
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return (torch.from_numpy(counts), torch.from_numpy(offsets),
            torch.from_numpy(perm), torch.from_numpy(inv))


# ---------------------------------------------------------------------------
# experts, combine, norm
# ---------------------------------------------------------------------------
def expert_glu(zrows: torch.Tensor, w_gate: torch.Tensor, w_up: torch.Tensor,
               w_down: torch.Tensor, quant: bool = False,
               wdeq: Optional[Dict[str, torch.Tensor]] = None) -> torch.Tensor:
    """One latent expert on its rows: h = bf16(SiLU(z W_g^T) * (z W_u^T)),
    o = h W_d^T (fp64).  Intermediate size d_ff, operating in the latent space
    [derekhsu, 潛在專家]; the gated activation is SiLU-GLU (reading of the
    garbled "SiTU-GLU").  In FP8 mode the GEMM inputs (bf16 z, bf16 h) are
    fake-quantised per 1x128 block and the weights passed are already
    dequantised.
    """
    a = _as_f64(zrows)
    if quant:
        a = quantize_act_1x128(a)
    g = a @ _as_f64(w_gate).T
    u = a @ _as_f64(w_up).T
    h = bf16_round(g / (1.0 + torch.exp(-g)) * u)
    if quant:
        h = quantize_act_1x128(h)
    return h @ _as_f64(w_down).T


def rmsnorm(c: torch.Tensor, gain: torch.Tensor, eps: float) -> torch.Tensor:
    """c / sqrt(mean(c^2) + eps) * gain, fp64 (unrounded).  RMSNorm sits
    before the shared up-projection [derekhsu, Stable LatentMoE]."""
    c = _as_f64(c)
    return c / torch.sqrt((c * c).mean(dim=1, keepdim=True) + eps) * _as_f64(gain)[None, :]


def bias_update(bias: torch.Tensor, counts: torch.Tensor, T: int, k: int,
                gamma: float) -> torch.Tensor:
    """Aux-loss-free balancing step [derekhsu; lininn]: b[e] += gamma * sign(
    mean load - load[e]), with load = count of (token, slot) pairs, mean load
    T*k/E, the sign taken exactly in integers as sgn(T*k - E*count[e]) and
    sign(0) = 0.  The add is one fp32 add of fp32(gamma * sign)."""
    E = counts.numel()
    d = T * k - E * counts.to(torch.int64)
    sgn = torch.sign(d).to(F32)
    return bias.to(F32) + torch.tensor(gamma, dtype=F32) * sgn


# ---------------------------------------------------------------------------
# FP8 e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no inf,
# max finite 448) and the 1x128 / 128x128 block scaling of the FP8 variant
# ---------------------------------------------------------------------------
def e4m3_decode(codes: torch.Tensor) -> torch.Tensor:
    """Value of each e4m3 byte (NaN for S.1111.111), float64."""
    c = codes.to(torch.int64) & 0xFF
    sign = torch.where((c >> 7) == 1, -1.0, 1.0).to(F64)
    e = (c >> 3) & 0xF
    m = (c & 7).to(F64)
    normal = (1.0 + m / 8.0) * torch.pow(2.0, (e - 7).to(F64))
    sub = (m / 8.0) * 2.0 ** -6
    v = torch.where(e == 0, sub, normal) * sign
    return torch.where((c & 0x7F) == 0x7F, torch.full_like(v, float("nan")), v)


def _rne(x: torch.Tensor) -> torch.Tensor:
    """Round half to even (float64)."""
    return torch.round(x)  # torch.round rounds half to even


def e4m3_encode(v: torch.Tensor) -> torch.Tensor:
    """Round each value to the nearest e4m3 value, ties to even, saturating to
    +-448 (satfinite).  Input values are taken as float64; returns uint8 codes."""
    v = _as_f64(v)
    a = v.abs()
    # binade exponent floor(log2 a) (exact, via frexp: a = m 2^x, m in [0.5, 1)),
    # clamped to the subnormal floor -6; the quantum of that binade is 2^(e-3)
    e = (torch.frexp(torch.where(a > 0, a, torch.ones_like(a))).exponent - 1).to(F64)
    e = torch.clamp(e, min=-6.0)
    q = torch.pow(2.0, e - 3.0)
    r = torch.clamp(_rne(a / q) * q, max=448.0)
    # encode r exactly
    re = (torch.frexp(torch.where(r > 0, r, torch.ones_like(r))).exponent - 1).to(F64)
    is_sub = (r < 2.0 ** -6)
    mant_sub = torch.round(r / 2.0 ** -9)                       # 0..7 (8 -> becomes normal)
    mant_n = torch.round((r / torch.pow(2.0, re) - 1.0) * 8.0)  # 0..7
    code = torch.where(is_sub, mant_sub, (re + 7.0) * 8.0 + mant_n).to(torch.int64)
    code = code | torch.where(torch.signbit(v), 0x80, 0)
    return code.to(torch.uint8)


def quantize_act_1x128(v: torch.Tensor) -> torch.Tensor:
    """Fake-quantise activations [rows, K] per 1x128 block along K.

    Per block: amax = max|v|; amax == 0 -> scale 1, q = 0; else scale =
    fp32(amax / 448) and q = e4m3_RNE_satfinite(fp32(v * fp32(448 / amax))).
    The quantiser's inputs are first rounded to fp32 so it decides in the
    kernel's precision.  Returns the dequantised values q * scale (float64).
    """
    x = v.to(F32)
    rows, K = x.shape
    assert K % 128 == 0
    xb = x.reshape(rows, K // 128, 128)
    amax = xb.abs().amax(dim=2, keepdim=True)
    zero = amax == 0
    safe = torch.where(zero, torch.ones_like(amax), amax)
    scale = torch.where(zero, torch.ones_like(amax), safe / torch.tensor(448.0, dtype=F32))
    inv = torch.tensor(448.0, dtype=F32) / safe
    codes = e4m3_encode((xb * inv).to(F64))
    deq = e4m3_decode(codes) * scale.to(F64)
    deq = torch.where(zero.expand_as(deq), torch.zeros_like(deq), deq)
    return deq.reshape(rows, K)


def dequantize_weight_128x128(codes: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """W = decode(q) * scale[block] for 128x128 blocks of an [out, in] matrix."""
    out, inn = codes.shape
    s = scales.to(F64).repeat_interleave(128, 0)[:out].repeat_interleave(128, 1)[:, :inn]
    return e4m3_decode(codes) * s


# ---------------------------------------------------------------------------
# FP4 e2m1 (OCP Microscaling Formats v1.0, FP4 element type: 1 sign, 2
# exponent bits with bias 1, 1 mantissa bit, no inf or NaN, max 6) for the
# FP4 expert variant.  The pages say only that the post-trained release ships
# FP4 weights; this variant's reading: every expert matrix (routed and
# shared) holds e2m1 codes, two per byte along K (element 2i in the low
# nibble), with one fp32 scale per 128x128 block as in the FP8 variant; the
# projections, activations and routers are as in the FP8 variant.
# ---------------------------------------------------------------------------
FP4_MATRICES = ("w_gate", "w_up_e", "w_down_e", "w_sh_gate", "w_sh_up", "w_sh_down")


def e2m1_decode(codes: torch.Tensor) -> torch.Tensor:
    """Value of each 4-bit e2m1 code (low nibble of the input), float64:
    exponent field 0 is subnormal (0 or 0.5), else (1 + m/2) 2^(e-1)."""
    c = codes.to(torch.int64) & 0xF
    e = (c >> 1) & 3
    m = (c & 1).to(F64)
    v = torch.where(e == 0, m * 0.5, (1.0 + m / 2.0) * torch.pow(2.0, (e - 1).to(F64)))
    return torch.where((c >> 3) == 1, -v, v)


def unpack_e2m1(packed: torch.Tensor) -> torch.Tensor:
    """[..., n] bytes -> [..., 2n] codes: byte i holds element 2i in its low
    nibble and element 2i + 1 in its high nibble."""
    b = packed.to(torch.int64) & 0xFF
    return torch.stack((b & 0xF, b >> 4), dim=-1).reshape(*b.shape[:-1], 2 * b.shape[-1])


def dequantize_weight_fp4_128x128(packed: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """W = e2m1(code) * scale[block] for 128x128 blocks of an [out, in]
    matrix given as packed codes [out, in / 2]."""
    codes = unpack_e2m1(packed)
    out, inn = codes.shape
    s = scales.to(F64).repeat_interleave(128, 0)[:out].repeat_interleave(128, 1)[:, :inn]
    return e2m1_decode(codes) * s


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------
@dataclass
class OracleResult:
    z: torch.Tensor          # [T, L] bf16 values (fp64)
    s: torch.Tensor          # [T, E] fp32
    topk_idx: torch.Tensor   # [T, k] int64
    topk_w: torch.Tensor     # [T, k] fp32 (before alpha)
    counts: torch.Tensor
    offsets: torch.Tensor
    perm: torch.Tensor
    inv_perm: torch.Tensor
    c: torch.Tensor          # [T, L] fp64 combined expert output before the norm
    n: torch.Tensor          # [T, L] bf16 values (fp64)
    y: torch.Tensor          # [T, D] bf16 values (fp64)


def _w(weights, name, fp8_deq, e=None):
    if fp8_deq is not None and name in fp8_deq:
        return fp8_deq[name](e) if e is not None else fp8_deq[name]()
    t = weights[name]
    return t if e is None else t[e]


def forward(x: torch.Tensor, weights: Dict[str, torch.Tensor], bias: torch.Tensor,
            top_k: int, rms_eps: float = 1e-6, fp8: bool = False,
            scores: Optional[torch.Tensor] = None, aggregation: str = "mean",
            fp4: bool = False) -> OracleResult:
    """The layer on CPU, step by step.

    1. z = bf16(x W_dn^T)                          down-projection 4096 -> 2048
    2-3. s = agg_r sigmoid(zx W_r^T) (fp32)         multi-router scores (agg: mean by
         default, or sum / max, see router_scores), where zx
         is the unrounded latent x W_dn^T (the routers read it at full precision)
    4-5. top-k of s + b; w = renormalised s; w' = w * alpha
    6. dispatch record (counts, offsets, perm, inv_perm)
    7-9. routed experts on their rows, shared expert on every token
    10. c = sum_j w'_j o_j + o_shared (fp64)
    11. n = bf16(RMSNorm(c) * gain)
    12. y = bf16(n W_up^T)                         shared up-projection 2048 -> 4096
    ``scores`` replaces steps 1-3 with the given fp32 s (routing-only use; z,
    c, n and y are then not computed).  In FP8 mode ``weights`` carries e4m3
    codes for every projection and expert matrix w_<x> and its 128x128 block
    scales as s_<x>; the routers stay bf16.  FP4 mode (``fp4``) is FP8 mode
    with the expert matrices (FP4_MATRICES) given as packed e2m1 codes
    [.., out, in / 2] with the same 128x128 block scales.
    """
    E = weights["expert_scale"].numel()
    deq = None
    if fp4:
        fp8 = True                 # projections, activations and routers as in FP8 mode
    if fp8:
        def mk(nm):
            codes, sc = weights[nm], weights["s_" + nm[2:]]   # scale array: w_<x> -> s_<x>
            dq = dequantize_weight_fp4_128x128 if (fp4 and nm in FP4_MATRICES) else dequantize_weight_128x128
            if codes.dim() == 3:
                return lambda e: dq(codes[e], sc[e])
            return lambda: dq(codes, sc)
        deq = {nm: mk(nm) for nm in ("w_down", "w_gate", "w_up_e", "w_down_e",
                                      "w_sh_gate", "w_sh_up", "w_sh_down", "w_up")}
    if scores is None:
        xin = quantize_act_1x128(_as_f64(x)) if fp8 else _as_f64(x)
        zx = xin @ _as_f64(_w(weights, "w_down", deq)).T
        z = bf16_round(zx)
        s = router_scores(zx, weights["w_router"], aggregation)
    else:
        z, s = None, scores.to(F32)
    T = s.shape[0]
    idx = select_topk(s, bias, top_k)
    w, wsc = route_weights(s, idx, weights["expert_scale"])
    counts, offsets, perm, inv = permutation(idx, E)
    if scores is not None:
        return OracleResult(None, s, idx, w, counts, offsets, perm, inv, None, None, None)

    L = z.shape[1]
    c = torch.zeros(T, L, dtype=F64)
    for e in range(E):
        rows = perm[offsets[e]:offsets[e + 1]]
        if rows.numel() == 0:
            continue
        tok = rows // top_k
        slot = rows % top_k
        o = expert_glu(z[tok], _w(weights, "w_gate", deq, e), _w(weights, "w_up_e", deq, e),
                       _w(weights, "w_down_e", deq, e), quant=fp8)
        c.index_add_(0, tok, o * wsc[tok, slot].to(F64)[:, None])
    c += expert_glu(z, _w(weights, "w_sh_gate", deq), _w(weights, "w_sh_up", deq),
                    _w(weights, "w_sh_down", deq), quant=fp8)
    n = bf16_round(rmsnorm(c, weights["rms_gain"], rms_eps))
    nin = quantize_act_1x128(n) if fp8 else n
    y = bf16_round(nin @ _as_f64(_w(weights, "w_up", deq)).T)
    return OracleResult(z, s, idx, w, counts, offsets, perm, inv, c, n, y)
