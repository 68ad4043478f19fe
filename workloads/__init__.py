"""Seeded synthetic inputs for the Multi-Router Latent MoE layer.

This module holds layer shapes and random draws only; none of the layer's
arithmetic lives here.  Both the CUDA path's tests/benchmarks and the CPU
oracle draw their inputs from it, so that the two sides see the same bits.

Random numbers come from one counter-based generator, Philox4x32-10
(Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
SC 2011), written out below with torch integer ops so it gives identical words
on the CPU and on a GPU.  Normal variates use the Box-Muller transform in
float64 and are then rounded to bf16.

Shapes follow the ERNIE 5.5 Flash release pages: hidden 4096 projected to a
2048-d latent, 512 routed experts with top-10 plus one shared expert,
expert intermediate size 2048 (blog.derekhsu.net, "Multi-Router Latent MoE"
section; lininn.cn, "routers, more than one" section).  The number of routers
R=4, the tiny configuration and the value distributions are stated
assumptions of this implementation (the pages fix neither).
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

__all__ = [
    "LayerShape", "CONFIGS", "philox4x32_10", "random_words", "normal",
    "uniform", "make_weights", "make_x", "make_bias", "zipf_ln_ratio",
    "flops_per_token",
]


@dataclass(frozen=True)
class LayerShape:
    """One layer configuration.

    T tokens; d_model hidden; d_lat latent; n_experts routed experts; top_k
    selected per token; d_ff expert intermediate; n_routers sigmoid routers.
    ``fp8`` selects the e4m3 block-scaled expert/projection variant; ``fp4``
    (with ``fp8``) gives the expert matrices as packed e2m1 codes instead.
    """
    name: str
    T: int
    d_model: int
    d_lat: int
    n_experts: int
    top_k: int
    d_ff: int
    n_routers: int
    rms_eps: float = 1e-6
    fp8: bool = False
    fp4: bool = False              # expert matrices e2m1 (implies the FP8 variant elsewhere)
    bias_kind: str = "zero"        # "zero" | "zipf"
    aggregation: str = "mean"      # router score aggregation: "mean" | "sum" | "max"
    outlier_frac: float = 0.0      # fraction of x channels scaled by outlier_scale
    outlier_scale: float = 20.0
    seed: int = 0

    def with_T(self, T: int) -> "LayerShape":
        return replace(self, T=T)


_FULL = dict(d_model=4096, d_lat=2048, n_experts=512, top_k=10, d_ff=2048, n_routers=4)

CONFIGS: Dict[str, LayerShape] = {
    # tiny CPU-checkable layer
    "c0_tiny": LayerShape("c0_tiny", T=64, d_model=256, d_lat=128, n_experts=16,
                          top_k=2, d_ff=128, n_routers=2),
    # full width, decode-sized batch: weight-streaming bound
    "c1_decode": LayerShape("c1_decode", T=128, **_FULL),
    # full width prefill, near-uniform routing: the headline workload
    "c2_prefill": LayerShape("c2_prefill", T=8192, **_FULL),
    # full width, Zipf(1.1) expert popularity through the balancing bias
    "c3_skew": LayerShape("c3_skew", T=32768, bias_kind="zipf", **_FULL),
    # full width, e4m3 experts/projections with 1% outlier channels in x
    "c4_fp8": LayerShape("c4_fp8", T=16384, fp8=True, outlier_frac=0.01, **_FULL),
    # test case: the tiny layer in the FP8 variant (2 of the 256 x channels are outliers)
    "c0_fp8": LayerShape("c0_fp8", T=64, d_model=256, d_lat=128, n_experts=16, top_k=2, d_ff=128,
                         n_routers=2, fp8=True, outlier_frac=0.01),
    # FP4 expert weights (e2m1, 128x128 block scales), the rest as in the FP8
    # variant: the decode-sized full-width layer, and the tiny test layer
    "c1_fp4": LayerShape("c1_fp4", T=128, fp8=True, fp4=True, outlier_frac=0.01, **_FULL),
    "c0_fp4": LayerShape("c0_fp4", T=64, d_model=256, d_lat=128, n_experts=16, top_k=2, d_ff=128,
                         n_routers=2, fp8=True, fp4=True, outlier_frac=0.01),
}

# Scalar lambda for the c3_skew bias b_e = lambda * ln(p_rank(e) / p_1), with
# p_i proportional to i^-1.1 over a seeded random expert permutation.  Fitted by
# bisection on the oracle's routing of this config's inputs (oracle/fit_zipf_bias.py)
# so that max(count)/mean(count) lands in [28, 32].  The fit result is stored
# in tests/golden/c3_zipf_lambda.json; this is the fallback before that exists.
_ZIPF_S = 1.1


def flops_per_token(s: LayerShape) -> int:
    """Algorithmic FLOPs per token: down-proj, routers, (k+1) SiLU-GLU experts, up-proj."""
    return 2 * (s.d_model * s.d_lat + s.n_routers * s.d_lat * s.n_experts
                + (s.top_k + 1) * 3 * s.d_lat * s.d_ff + s.d_lat * s.d_model)


# --------------------------------------------------------------------------
# Philox4x32-10 with torch int64 tensors (values kept in [0, 2^32)).
# --------------------------------------------------------------------------
_M0 = 0xD2511F53
_M1 = 0xCD9E8D57
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_MASK32 = 0xFFFFFFFF


def _mulhilo(a: torch.Tensor, m: int):
    """Exact (hi, lo) 32-bit halves of a*m for a in [0,2^32), m a 32-bit constant.

    The 64-bit product does not fit a signed int64, so a is split in 16-bit
    halves; each partial product stays below 2^48.
    """
    a_lo = a & 0xFFFF
    a_hi = a >> 16
    p_lo = a_lo * m                      # < 2^48
    p_hi = a_hi * m                      # < 2^48
    hi = (p_hi + (p_lo >> 16)) >> 16
    lo = (((p_hi & 0xFFFF) << 16) + p_lo) & _MASK32
    return hi, lo


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32 with 10 rounds.  Counters are int64 tensors holding uint32 values."""
    k0 &= _MASK32
    k1 &= _MASK32
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK32
            k1 = (k1 + _W1) & _MASK32
        hi0, lo0 = _mulhilo(c0, _M0)
        hi1, lo1 = _mulhilo(c2, _M1)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


_CHUNK_BLOCKS = 1 << 22  # Philox blocks per generation chunk (16M words)


def random_words(n_words: int, seed: int, stream: int, device, start_block: int = 0):
    """n_words uint32 words (as int64) from stream ``stream`` of ``seed``.

    Block i of the stream is Philox4x32-10 with counter (i mod 2^32, i >> 32, 0, 0)
    and key (seed, stream); its four words are elements 4i..4i+3.
    """
    n_blocks = (n_words + 3) // 4
    idx = torch.arange(start_block, start_block + n_blocks, dtype=torch.int64, device=device)
    c0 = idx & _MASK32
    c1 = idx >> 32
    z = torch.zeros_like(idx)
    o = philox4x32_10(c0, c1, z, z, seed, stream)
    return torch.stack(o, dim=1).reshape(-1)[:n_words]


def _normals_from_words(w: torch.Tensor) -> torch.Tensor:
    """Box-Muller in float64: words (a,b) pairs -> (r cos, r sin)."""
    w = w.reshape(-1, 2).to(torch.float64)
    u1 = (w[:, 0] + 0.5) * (1.0 / 4294967296.0)
    u2 = (w[:, 1] + 0.5) * (1.0 / 4294967296.0)
    r = torch.sqrt(-2.0 * torch.log(u1))
    th = (2.0 * math.pi) * u2
    return torch.stack((r * torch.cos(th), r * torch.sin(th)), dim=1).reshape(-1)


def normal(shape, seed: int, stream: int, device, std: float = 1.0,
           dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
           col_scale: Optional[torch.Tensor] = None) -> torch.Tensor:
    """N(0, std^2) draws of ``shape`` rounded to ``dtype``.

    Element i comes from word pair p = i // 2 (words 2p, 2p+1 of the stream):
    r cos(theta) for even i, r sin(theta) for odd i.  Results therefore do not
    depend on how the work is chunked.  ``col_scale`` (float64, length
    shape[-1]) multiplies each column before the final rounding (outlier
    channels).
    """
    numel = 1
    for d in shape:
        numel *= int(d)
    if out is None:
        out = torch.empty(numel, dtype=dtype, device=device)
    flat = out.view(-1)
    ncols = int(shape[-1])
    step = _CHUNK_BLOCKS * 4          # 4 normals per Philox block
    cs = None if col_scale is None else col_scale.to(torch.float64).to(device)
    done = 0
    while done < numel:
        n = min(step, numel - done)
        words = random_words(4 * ((n + 3) // 4), seed, stream, device, start_block=done // 4)
        vals = _normals_from_words(words)[:n] * std
        if cs is not None:
            cols = torch.arange(done, done + n, device=device) % ncols
            vals = vals * cs[cols]
        flat[done:done + n] = vals.to(torch.float32).to(dtype)
        done += n
    return out.view(*shape)


def uniform(shape, lo: float, hi: float, seed: int, stream: int, device,
            dtype=torch.float32) -> torch.Tensor:
    """U(lo, hi) from one word per element: lo + (w + 0.5) 2^-32 (hi - lo)."""
    numel = 1
    for d in shape:
        numel *= int(d)
    w = random_words(numel, seed, stream, device).to(torch.float64)
    u = (w + 0.5) * (1.0 / 4294967296.0)
    return (lo + u * (hi - lo)).to(dtype).reshape(*shape)


def _perm(n: int, seed: int, stream: int, device) -> torch.Tensor:
    """Seeded random permutation of range(n): argsort of n random words (ties by index)."""
    w = random_words(n, seed, stream, device)
    return torch.sort(w, stable=True).indices


# Stream ids, one per tensor.
_S_X, _S_WDN, _S_WR, _S_WG, _S_WU, _S_WD, _S_SG, _S_SU, _S_SD, _S_WUP, _S_ALPHA, \
    _S_ZIPF_PERM, _S_OUTLIER, _S_DY, _S_GAIN = range(1, 16)


def make_weights(s: LayerShape, device, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """bf16 weights ~N(0, 1/fan_in), stored [out, in]; alpha ~U(0.5, 1.5); RMS gain 1."""
    seed = s.seed if seed is None else seed
    D, L, E, F, R = s.d_model, s.d_lat, s.n_experts, s.d_ff, s.n_routers
    w = {}
    w["w_down"] = normal((L, D), seed, _S_WDN, device, std=1.0 / math.sqrt(D))
    w["w_router"] = normal((R, E, L), seed, _S_WR, device, std=1.0 / math.sqrt(L))
    w["w_gate"] = normal((E, F, L), seed, _S_WG, device, std=1.0 / math.sqrt(L))
    w["w_up_e"] = normal((E, F, L), seed, _S_WU, device, std=1.0 / math.sqrt(L))
    w["w_down_e"] = normal((E, L, F), seed, _S_WD, device, std=1.0 / math.sqrt(F))
    w["w_sh_gate"] = normal((F, L), seed, _S_SG, device, std=1.0 / math.sqrt(L))
    w["w_sh_up"] = normal((F, L), seed, _S_SU, device, std=1.0 / math.sqrt(L))
    w["w_sh_down"] = normal((L, F), seed, _S_SD, device, std=1.0 / math.sqrt(F))
    w["w_up"] = normal((D, L), seed, _S_WUP, device, std=1.0 / math.sqrt(L))
    w["rms_gain"] = torch.ones(L, dtype=torch.float32, device=device)
    w["expert_scale"] = uniform((E,), 0.5, 1.5, seed, _S_ALPHA, device)
    return w


def make_routing_weights(s: LayerShape, device, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The tensors routing from x needs (down-projection, routers, alpha): the
    same draws as make_weights, without the expert weights."""
    seed = s.seed if seed is None else seed
    D, L, E, R = s.d_model, s.d_lat, s.n_experts, s.n_routers
    return {"w_down": normal((L, D), seed, _S_WDN, device, std=1.0 / math.sqrt(D)),
            "w_router": normal((R, E, L), seed, _S_WR, device, std=1.0 / math.sqrt(L)),
            "expert_scale": uniform((E,), 0.5, 1.5, seed, _S_ALPHA, device)}


FP8_MATRICES = ("w_down", "w_gate", "w_up_e", "w_down_e", "w_sh_gate", "w_sh_up", "w_sh_down", "w_up")


def to_fp8_blocks(w: torch.Tensor):
    """e4m3 codes and fp32 scales per 128x128 block of the trailing [out, in]
    dims: scale = fp32(amax / 448) (1 for an all-zero block), codes from the
    library's float8_e4m3fn conversion of w / scale (clamped to +-448)."""
    *lead, out, inn = w.shape
    ob, ib = (out + 127) // 128, (inn + 127) // 128
    wf = w.to(torch.float32)
    pad = torch.zeros(*lead, ob * 128, ib * 128, dtype=torch.float32, device=w.device)
    pad[..., :out, :inn] = wf
    blk = pad.reshape(*lead, ob, 128, ib, 128)
    amax = blk.abs().amax(dim=(-3, -1))                       # [..., ob, ib]
    scale = torch.where(amax == 0, torch.ones_like(amax), amax / torch.tensor(448.0))
    q = (blk / scale[..., :, None, :, None]).clamp(-448.0, 448.0)
    codes = q.to(torch.float8_e4m3fn).reshape(*lead, ob * 128, ib * 128)[..., :out, :inn]
    return codes.contiguous().view(torch.uint8), scale.contiguous()


def make_weights_fp8(s: LayerShape, device, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The FP8 variant's inputs: the bf16 weights of make_weights, with every
    projection and expert matrix given as e4m3 codes (uint8) plus its fp32
    128x128 block scales under the C ABI's name (w_down -> s_down, w_up_e ->
    s_up_e, ...); the routers stay bf16."""
    w = make_weights(s, device, seed)
    for nm in FP8_MATRICES:
        codes, scale = to_fp8_blocks(w[nm])
        w[nm] = codes
        w[fp8_scale_name(nm)] = scale
    return w


FP4_MATRICES = ("w_gate", "w_up_e", "w_down_e", "w_sh_gate", "w_sh_up", "w_sh_down")
_E2M1_UP = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)   # midpoints of the e2m1 magnitudes


def to_fp4_blocks(w: torch.Tensor):
    """Packed e2m1 codes and fp32 scales per 128x128 block of the trailing
    [out, in] dims (in even): scale = fp32(amax / 6) (1 for an all-zero
    block); each w / scale goes to the nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6
    (the midpoint 0.75, 1.75 and 3.5 upward, the others downward) with its
    sign; byte i of a row holds element 2i in its low nibble.  Codes [..,
    out, in / 2] uint8."""
    *lead, out, inn = w.shape
    ob, ib = (out + 127) // 128, (inn + 127) // 128
    pad = torch.zeros(*lead, ob * 128, ib * 128, dtype=torch.float32, device=w.device)
    pad[..., :out, :inn] = w.to(torch.float32)
    blk = pad.reshape(*lead, ob, 128, ib, 128)
    amax = blk.abs().amax(dim=(-3, -1))
    scale = torch.where(amax == 0, torch.ones_like(amax), amax / torch.tensor(6.0))
    q = (blk / scale[..., :, None, :, None]).reshape(*lead, ob * 128, ib * 128)[..., :out, :inn]
    a = q.abs()
    mag = torch.zeros_like(a, dtype=torch.uint8)
    for i, t in enumerate(_E2M1_UP):
        mag += (a >= t) if i in (1, 3, 5) else (a > t)
    code = mag | (torch.signbit(q).to(torch.uint8) << 3)
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    return packed.contiguous(), scale.contiguous()


def make_weights_fp4(s: LayerShape, device, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The FP4 expert variant's inputs: the FP8 variant's, with the expert
    matrices (routed and shared) re-quantised from the bf16 draws as packed
    e2m1 codes plus fp32 128x128 block scales under the same names."""
    w = make_weights(s, device, seed)
    for nm in FP8_MATRICES:
        codes, scale = (to_fp4_blocks if nm in FP4_MATRICES else to_fp8_blocks)(w[nm])
        w[nm] = codes
        w[fp8_scale_name(nm)] = scale
    return w


def make_layer_weights(s: LayerShape, device, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The weights of a config in its variant (bf16, FP8 or FP4 experts)."""
    if s.fp4:
        return make_weights_fp4(s, device, seed)
    return (make_weights_fp8 if s.fp8 else make_weights)(s, device, seed)


def fp8_scale_name(matrix: str) -> str:
    """Name of a matrix's block-scale array: w_<x> -> s_<x>."""
    return "s_" + matrix[2:]


def outlier_channels(s: LayerShape, device, seed: Optional[int] = None) -> torch.Tensor:
    """Indices of the round(outlier_frac * d_model) outlier channels (seeded choice)."""
    seed = s.seed if seed is None else seed
    n = int(round(s.outlier_frac * s.d_model))
    return torch.sort(_perm(s.d_model, seed, _S_OUTLIER, device)[:n]).values


def make_x(s: LayerShape, device, seed: Optional[int] = None, T: Optional[int] = None,
           token0: int = 0) -> torch.Tensor:
    """x ~ N(0,1) [T, d_model] bf16; outlier channels scaled before rounding.

    ``token0``/``T`` select a contiguous token window of the full x, with the
    same values as the corresponding rows of the full tensor.
    """
    seed = s.seed if seed is None else seed
    T = s.T if T is None else T
    col_scale = None
    if s.outlier_frac > 0:
        col_scale = torch.ones(s.d_model, dtype=torch.float64)
        col_scale[outlier_channels(s, "cpu", seed)] = s.outlier_scale
    if token0 == 0:
        return normal((T, s.d_model), seed, _S_X, device, col_scale=col_scale)
    # window: generate the covering range and slice (elements are position-addressed)
    full = normal(((token0 + T), s.d_model), seed, _S_X, device, col_scale=col_scale)
    return full[token0:].contiguous()


def make_dy(s: LayerShape, device, seed: Optional[int] = None, T: Optional[int] = None) -> torch.Tensor:
    """Incoming gradient of the layer output for the backward pass: dy ~ N(0,1)
    [T, d_model] bf16 (a loss with unit-variance output gradients)."""
    seed = s.seed if seed is None else seed
    T = s.T if T is None else T
    return normal((T, s.d_model), seed, _S_DY, device)


def make_train_gain(s: LayerShape, device, seed: Optional[int] = None) -> torch.Tensor:
    """A trained-looking RMSNorm gain for the backward tests: 1 + 0.1 N(0,1)
    (fp32), so that a gain dropped or misplaced in a gradient shows."""
    seed = s.seed if seed is None else seed
    return 1.0 + 0.1 * normal((s.d_lat,), seed, _S_GAIN, device, dtype=torch.float32)


def zipf_ln_ratio(s: LayerShape, device, seed: Optional[int] = None) -> torch.Tensor:
    """ln(p_rank(e)/p_1) for p_i ∝ i^-1.1 over a seeded random expert ranking (fp32)."""
    seed = s.seed if seed is None else seed
    rank_of = torch.empty(s.n_experts, dtype=torch.int64)
    order = _perm(s.n_experts, seed, _S_ZIPF_PERM, "cpu")
    rank_of[order] = torch.arange(1, s.n_experts + 1)
    return (-_ZIPF_S * torch.log(rank_of.to(torch.float64))).to(torch.float32).to(device)


_GOLDEN = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "tests", "golden")


def zipf_lambda(s: LayerShape) -> float:
    """The fitted lambda for a zipf-bias config (see tests/golden/c3_zipf_lambda.json)."""
    p = os.path.join(_GOLDEN, f"{s.name}_zipf_lambda.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["lambda"])
    raise FileNotFoundError(f"{p} missing: run oracle/fit_zipf_bias.py")


def make_bias(s: LayerShape, device, lam: Optional[float] = None) -> torch.Tensor:
    """Selection bias b [E] fp32: zero, or lambda * ln(p_rank/p_1) for the Zipf config."""
    if s.bias_kind == "zero":
        return torch.zeros(s.n_experts, dtype=torch.float32, device=device)
    lam = zipf_lambda(s) if lam is None else lam
    return (torch.tensor(lam, dtype=torch.float32) * zipf_ln_ratio(s, "cpu")).to(device)
