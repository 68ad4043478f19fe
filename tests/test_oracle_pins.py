"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test checks one oracle function against a closed form, a hand-worked
fixture, brute force on tiny inputs, an invariant stated by the pages, or a
library routine on a special case — chosen so that a dropped term, a wrong
sign or index, or a transposed operand fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")
F64 = torch.float64


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- rounding
def test_bf16_round_matches_library_on_fp32_inputs():
    g = torch.Generator().manual_seed(1)
    v = torch.randn(100000, generator=g, dtype=torch.float32) * 10
    ref = v.to(torch.bfloat16).to(F64)          # torch's fp32 -> bf16 is RNE
    assert torch.equal(O.bf16_round(v.to(F64)), ref)


def test_bf16_round_ties_and_no_double_rounding():
    one = 1.0
    assert O.bf16_round(torch.tensor([one + 2 ** -8], dtype=F64)).item() == 1.0        # tie -> even
    assert O.bf16_round(torch.tensor([one + 3 * 2 ** -8], dtype=F64)).item() == 1.015625
    # just above the midpoint: fp32 would first round onto the midpoint, then to 1.0
    assert O.bf16_round(torch.tensor([one + 2 ** -8 + 2 ** -40], dtype=F64)).item() == 1.0078125
    assert O.bf16_round(torch.tensor([-(one + 2 ** -8 + 2 ** -40)], dtype=F64)).item() == -1.0078125
    assert O.bf16_round(torch.tensor([0.0], dtype=F64)).item() == 0.0


# ------------------------------------------------------------ projections
def test_linear_selection_matrix_closed_form():
    # W = [I | 0] picks the first L input channels: z = x[:, :L] exactly.
    T, D, L = 5, 12, 4
    x = torch.randn(T, D, dtype=torch.float32).to(torch.bfloat16)
    w = torch.zeros(L, D)
    w[:, :L] = torch.eye(L)
    z = O.linear_bf16(x, w.to(torch.bfloat16))
    assert torch.equal(z, x[:, :L].to(F64))
    # a permutation matrix permutes channels: catches a transposed operand
    p = torch.tensor([2, 0, 3, 1])
    wp = torch.zeros(L, D)
    wp[torch.arange(L), p] = 1.0
    assert torch.equal(O.linear_bf16(x, wp.to(torch.bfloat16)), x[:, p].to(F64))


def test_linear_brute_force_loops():
    g = torch.Generator().manual_seed(2)
    T, D, L = 3, 7, 5
    x = torch.randn(T, D, generator=g).to(torch.bfloat16)
    w = torch.randn(L, D, generator=g).to(torch.bfloat16)
    z = O.linear_bf16(x, w)
    for t in range(T):
        for o in range(L):
            acc = math.fsum(float(x[t, i]) * float(w[o, i]) for i in range(D))
            assert z[t, o].item() == O.bf16_round(torch.tensor([acc], dtype=F64)).item()


# ----------------------------------------------------------------- routers
def _sig(v):
    return 1.0 / (1.0 + math.exp(-v))


def test_single_router_reduces_to_sigmoid():
    g = torch.Generator().manual_seed(3)
    T, L, E = 4, 6, 5
    z = torch.randn(T, L, generator=g).to(torch.bfloat16)
    wr = torch.randn(1, E, L, generator=g).to(torch.bfloat16)
    s = O.router_scores(z, wr)
    for t in range(T):
        for e in range(E):
            logit = math.fsum(float(z[t, i]) * float(wr[0, e, i]) for i in range(L))
            assert s[t, e].item() == np.float32(_sig(logit))


def test_identical_routers_equal_one_router():
    g = torch.Generator().manual_seed(4)
    z = torch.randn(8, 16, generator=g).to(torch.bfloat16)
    w1 = torch.randn(1, 6, 16, generator=g).to(torch.bfloat16)
    s1 = O.router_scores(z, w1)
    s4 = O.router_scores(z, w1.repeat(4, 1, 1))
    assert torch.allclose(s1.to(F64), s4.to(F64), rtol=0, atol=1e-7)


def test_router_aggregation_is_the_mean():
    # routers r and -r: sigmoid(a) + sigmoid(-a) = 1, so the mean is 1/2 exactly
    # (a sum would give 1, a max would give sigmoid(|a|)).
    g = torch.Generator().manual_seed(5)
    z = torch.randn(6, 8, generator=g).to(torch.bfloat16)
    w = torch.randn(1, 5, 8, generator=g).to(torch.bfloat16)
    s = O.router_scores(z, torch.cat([w, -w]))
    assert torch.all(s == 0.5)
    # zero weights: every router says sigmoid(0) = 1/2
    assert torch.all(O.router_scores(z, torch.zeros(3, 5, 8, dtype=torch.bfloat16)) == 0.5)


def test_router_sum_and_max_closed_forms():
    # the alternative aggregations on routers r and -r: the sum is exactly 1,
    # the max is sigmoid(|a|), computed here from a hand-summed logit
    g = torch.Generator().manual_seed(6)
    z = torch.randn(5, 8, generator=g).to(torch.bfloat16)
    w = torch.randn(1, 4, 8, generator=g).to(torch.bfloat16)
    assert torch.all(O.router_scores(z, torch.cat([w, -w]), "sum") == 1.0)
    smax = O.router_scores(z, torch.cat([w, -w]), "max")
    for t in range(5):
        for e in range(4):
            a = math.fsum(float(z[t, i]) * float(w[0, e, i]) for i in range(8))
            assert smax[t, e].item() == np.float32(_sig(abs(a)))


def test_router_aggregations_relate_exactly():
    g = torch.Generator().manual_seed(7)
    z = torch.randn(16, 12, generator=g).to(torch.bfloat16)
    w4 = torch.randn(4, 7, 12, generator=g).to(torch.bfloat16)
    # R = 4: the sum is 4 x the mean (scaling by 2^2 commutes with the fp32 rounding)
    assert torch.equal(O.router_scores(z, w4, "sum"), 4 * O.router_scores(z, w4, "mean"))
    # R = 1: all three rules are the single router's sigmoid
    w1 = w4[:1]
    m = O.router_scores(z, w1, "mean")
    assert torch.equal(m, O.router_scores(z, w1, "sum")) and torch.equal(m, O.router_scores(z, w1, "max"))
    # the max is at least the mean and at most the sum
    mx, mn, sm = (O.router_scores(z, w4, a) for a in ("max", "mean", "sum"))
    assert torch.all(mx >= mn) and torch.all(mx <= sm)
    with pytest.raises(ValueError):
        O.router_scores(z, w4, "median")


def test_router_max_brute_force():
    g = torch.Generator().manual_seed(8)
    T, L, E, R = 3, 10, 4, 3
    z = torch.randn(T, L, generator=g).to(torch.bfloat16)
    wr = torch.randn(R, E, L, generator=g).to(torch.bfloat16)
    s = O.router_scores(z, wr, "max")
    for t in range(T):
        for e in range(E):
            best = max(_sig(math.fsum(float(z[t, i]) * float(wr[r, e, i]) for i in range(L)))
                       for r in range(R))
            assert s[t, e].item() == np.float32(best)


# --------------------------------------------------------------- selection
def _valid_topk(sb, sel, k):
    E = sb.shape[0]
    S = set(sel)
    if len(S) != k:
        return False
    for i in S:
        for j in range(E):
            if j in S:
                continue
            if not (sb[i] > sb[j] or (sb[i] == sb[j] and i < j)):
                return False
    return True


def test_select_brute_force_E16_k2_with_ties():
    rng = np.random.default_rng(6)
    E, k = 16, 2
    # dyadic scores on a coarse grid: many exact ties
    s = torch.from_numpy(rng.integers(0, 6, size=(200, E)).astype(np.float32) / 8)
    b = torch.from_numpy(rng.integers(-2, 3, size=E).astype(np.float32) / 16)
    idx = O.select_topk(s, b, k)
    sb = (s + b).numpy()
    for t in range(s.shape[0]):
        sel = idx[t].tolist()
        assert _valid_topk(sb[t], sel, k), (t, sel)
        # maximises the sum over all k-subsets
        best = max(sum(sb[t][list(c)]) for c in itertools.combinations(range(E), k))
        assert sum(sb[t][sel]) == best
        # output order: descending biased score, ties by index
        keys = [(-sb[t][e], e) for e in sel]
        assert keys == sorted(keys)


def test_select_crafted_ties():
    E, k = 8, 3
    # all equal -> the k lowest indices
    assert O.select_topk(torch.full((1, E), 0.5), torch.zeros(E), k).tolist() == [[0, 1, 2]]
    # +0 and -0 tie: lower index wins
    s = torch.tensor([[-0.0, 0.0, -1.0, -1.0, -1.0, -1.0, -1.0, -1.0]])
    assert O.select_topk(s, torch.zeros(E), 2).tolist() == [[0, 1]]
    s = torch.tensor([[-1.0, 0.0, -1.0, -0.0, -1.0, -1.0, -1.0, -1.0]])
    assert O.select_topk(s, torch.zeros(E), 2).tolist() == [[1, 3]]
    # duplicates straddling the k-th boundary
    s = torch.tensor([[0.1, 0.9, 0.5, 0.5, 0.5, 0.2, 0.5, 0.0]])
    assert O.select_topk(s, torch.zeros(E), 3).tolist() == [[1, 2, 3]]
    # bias breaks a tie the other way
    b = torch.zeros(E)
    b[6] = 0.25
    assert O.select_topk(s, b, 3).tolist() == [[1, 6, 2]]      # 0.9 > 0.75 > 0.5


def test_select_bias_zero_and_constant_shift():
    rng = np.random.default_rng(7)
    s = torch.from_numpy(rng.integers(0, 64, size=(50, 32)).astype(np.float32) / 64)
    base = O.select_topk(s, torch.zeros(32), 5)
    ref = torch.from_numpy(np.argsort(-s.numpy(), axis=1, kind="stable")[:, :5])
    assert torch.equal(base, ref)
    # an exactly representable constant shift of b keeps the selection
    assert torch.equal(O.select_topk(s, torch.full((32,), 0.5), 5), base)


# ----------------------------------------------------------------- weights
def test_route_weights_sum_and_closed_form():
    s = torch.tensor([[0.75, 0.1, 0.25, 0.0]], dtype=torch.float32)
    idx = torch.tensor([[0, 2]])
    w, ws = O.route_weights(s, idx, torch.ones(4))
    assert w.tolist() == [[0.75, 0.25]] and torch.equal(w, ws)
    w, ws = O.route_weights(s, idx, torch.tensor([2.0, 1.0, 0.5, 1.0]))
    assert ws.tolist() == [[1.5, 0.125]]
    g = torch.Generator().manual_seed(8)
    s = torch.rand(100, 64, generator=g)
    idx = O.select_topk(s, torch.zeros(64), 10)
    w, _ = O.route_weights(s, idx, torch.ones(64))
    assert torch.all((w.sum(1).to(F64) - 1).abs() <= 10 * 2 ** -23)
    # the denominator is accumulated in slot order in fp32
    ssel = torch.gather(s, 1, idx).numpy()
    den = np.float32(0)
    for j in range(10):
        den = np.float32(den + ssel[0, j])
    assert w[0, 3].item() == np.float32(ssel[0, 3] / den)


def test_route_weights_zero_sum_gives_uniform_weights():
    # w = s / sum(s) is undefined when the selected scores sum to 0 (sigmoids
    # that underflowed to 0 in fp32); the reading is the uniform fp32(1/k),
    # the limit of equal scores.  Tokens with a non-zero sum are unaffected.
    s = torch.tensor([[0.0, 0.0, 0.0, 0.0], [0.0, 0.5, 0.0, 0.25]], dtype=torch.float32)
    idx = torch.tensor([[0, 1, 2], [1, 3, 0]])
    w, ws = O.route_weights(s, idx, torch.tensor([2.0, 1.0, 0.5, 1.0]))
    third = np.float32(1.0) / np.float32(3.0)
    assert w[0].tolist() == [float(third)] * 3
    assert ws[0].tolist() == [float(np.float32(third * np.float32(2.0))), float(third), float(np.float32(third * np.float32(0.5)))]
    assert w[1].tolist() == [float(np.float32(0.5) / np.float32(0.75)), float(np.float32(0.25) / np.float32(0.75)), 0.0]


# -------------------------------------------------------------- dispatch
def test_permutation_golden():
    g = _gold("permutation_small.json")
    c, off, perm, inv = O.permutation(torch.tensor(g["topk_idx"]), g["n_experts"])
    assert c.tolist() == g["counts"] and off.tolist() == g["offsets"]
    assert perm.tolist() == g["perm"] and inv.tolist() == g["inv_perm"]


def test_permutation_invariants():
    g = torch.Generator().manual_seed(9)
    T, E, k = 300, 40, 6
    s = torch.rand(T, E, generator=g)
    idx = O.select_topk(s, torch.zeros(E), k)
    c, off, perm, inv = O.permutation(idx, E)
    assert int(c.sum()) == T * k
    assert torch.all(off[1:] >= off[:-1]) and int(off[-1]) == T * k
    assert torch.equal(torch.sort(perm).values, torch.arange(T * k))
    assert torch.equal(inv[perm], torch.arange(T * k))
    flat = idx.reshape(-1)
    for e in range(E):
        rows = perm[off[e]:off[e + 1]]
        assert torch.all(flat[rows] == e)
        tok = rows // k
        assert torch.all(tok[1:] > tok[:-1])       # ascending tokens, no repeats


# ----------------------------------------------------------------- experts
def test_glu_closed_form_and_operand_roles():
    z = torch.ones(1, 1, dtype=torch.bfloat16)
    one = torch.ones(1, 1, dtype=torch.bfloat16)
    two = torch.full((1, 1), 2.0, dtype=torch.bfloat16)
    # g=1, u=1: h = bf16(silu(1)) = bf16(0.7310585786...) = 0.73046875; o = h
    assert O.expert_glu(z, one, one, one).item() == 0.73046875
    # g=1,u=2 vs g=2,u=1 differ: silu(1)*2 = 1.4621 -> 1.4609375 ; silu(2) = 1.7616 -> 1.7578125
    assert O.expert_glu(z, one, two, one).item() == 1.4609375
    assert O.expert_glu(z, two, one, one).item() == 1.7578125
    # g = 0 -> h = 0 regardless of u
    assert O.expert_glu(z, torch.zeros(1, 1, dtype=torch.bfloat16), two, one).item() == 0.0


def _tiny_layer(seed=0, T=24):
    s = W.CONFIGS["c0_tiny"].with_T(T)
    w = W.make_weights(s, "cpu", seed=seed)
    x = W.make_x(s, "cpu", seed=seed)
    return s, w, x


def test_sparse_dispatch_equals_dense_brute_force():
    s, w, x = _tiny_layer()
    b = torch.zeros(s.n_experts)
    r = O.forward(x, w, b, s.top_k, s.rms_eps)
    # dense: every expert on every token, masked by the routing weights
    z = r.z
    T, E = z.shape[0], s.n_experts
    mask = torch.zeros(T, E, dtype=F64)
    _, ws = O.route_weights(r.s, r.topk_idx, w["expert_scale"])
    for t in range(T):
        for j in range(s.top_k):
            mask[t, r.topk_idx[t, j]] = ws[t, j].double()
    c = torch.zeros(T, s.d_lat, dtype=F64)
    for t in range(T):
        zt = z[t:t + 1]
        for e in range(E):
            o = O.expert_glu(zt, w["w_gate"][e], w["w_up_e"][e], w["w_down_e"][e])
            c[t] += mask[t, e] * o[0]
        c[t] += O.expert_glu(zt, w["w_sh_gate"], w["w_sh_up"], w["w_sh_down"])[0]
    assert torch.allclose(c, r.c, rtol=1e-12, atol=1e-12)


def test_identical_experts_make_output_routing_independent():
    s, w, x = _tiny_layer(T=16)
    for nm in ("w_gate", "w_up_e", "w_down_e"):
        w[nm] = w[nm][:1].repeat(s.n_experts, 1, 1)
    w["expert_scale"] = torch.full((s.n_experts,), 0.75)
    r0 = O.forward(x, w, torch.zeros(s.n_experts), s.top_k)
    b = torch.linspace(-1, 1, s.n_experts)            # changes the selection
    r1 = O.forward(x, w, b, s.top_k)
    assert not torch.equal(r0.topk_idx, r1.topk_idx)
    assert torch.allclose(r0.c, r1.c, rtol=1e-6, atol=1e-7)


def test_shared_expert_always_on():
    # zero routed experts: the output is RMSNorm(shared expert) -> up-proj
    s, w, x = _tiny_layer(T=8)
    for nm in ("w_gate", "w_up_e", "w_down_e"):
        w[nm] = torch.zeros_like(w[nm])
    r = O.forward(x, w, torch.zeros(s.n_experts), s.top_k)
    sh = O.expert_glu(r.z, w["w_sh_gate"], w["w_sh_up"], w["w_sh_down"])
    assert torch.allclose(r.c, sh, rtol=0, atol=0)


# ------------------------------------------------------------------- norm
def test_rmsnorm_closed_form_and_scale_invariance():
    L, eps = 16, 1e-6
    gain = torch.linspace(0.5, 2.0, L)
    lam = 3.0
    n = O.rmsnorm(torch.full((1, L), lam, dtype=F64), gain, eps)
    assert torch.allclose(n[0], gain.to(F64) * lam / math.sqrt(lam * lam + eps), rtol=1e-15)
    c = torch.randn(4, L, dtype=F64)
    assert torch.allclose(O.rmsnorm(c * 7.0, gain, 0.0), O.rmsnorm(c, gain, 0.0), rtol=1e-13)
    assert torch.allclose(O.rmsnorm(-c, gain, eps), -O.rmsnorm(c, gain, eps), rtol=0)


# ------------------------------------------------------------ bias update
def test_bias_update_golden_and_uniform():
    g = _gold("bias_update_small.json")
    out = O.bias_update(torch.tensor(g["bias_in"]), torch.tensor(g["counts"]), g["T"],
                        g["top_k"], g["gamma"])
    assert out.tolist() == g["bias_out"]
    b = torch.randn(32)
    assert torch.equal(O.bias_update(b, torch.full((32,), 5), 16, 10, 1e-3), b)


# -------------------------------------------------------------------- FP8
def test_e4m3_decode_known_values_and_roundtrip():
    dec = O.e4m3_decode(torch.arange(256))
    assert dec[0x38].item() == 1.0 and dec[0x7E].item() == 448.0
    assert dec[0x08].item() == 2.0 ** -6 and dec[0x01].item() == 2.0 ** -9
    assert dec[0xB8].item() == -1.0 and math.isnan(dec[0x7F].item())
    ok = ~torch.isnan(dec)
    codes = O.e4m3_encode(dec[ok])
    assert torch.equal(codes.to(torch.int64), torch.arange(256)[ok])


def test_e4m3_encode_matches_library_in_range_and_saturates():
    g = torch.Generator().manual_seed(10)
    v = (torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 3))
    v = v.clamp(-448, 448).to(torch.float32)
    lib = v.to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(O.e4m3_encode(v.to(F64)), lib)
    # midpoints round to even: 1 + 1/16 lies between 1 and 1.125
    assert O.e4m3_encode(torch.tensor([1.0625], dtype=F64)).item() == 0x38
    assert O.e4m3_encode(torch.tensor([1.1875], dtype=F64)).item() == 0x3A
    assert O.e4m3_decode(O.e4m3_encode(torch.tensor([500.0, -1e6], dtype=F64))).tolist() == [448.0, -448.0]


def test_quantize_act_block_scaling():
    g = torch.Generator().manual_seed(11)
    v = torch.randn(3, 256, generator=g, dtype=F64)
    v[1, :128] = 0.0
    q = O.quantize_act_1x128(v)
    assert torch.all(q[1, :128] == 0)
    for r in range(3):
        for b in range(2):
            blk = v[r, b * 128:(b + 1) * 128].to(torch.float32)
            amax = blk.abs().max()
            if amax == 0:
                continue
            qb = q[r, b * 128:(b + 1) * 128]
            j = int(blk.abs().argmax())
            # the block maximum maps to code 448 exactly: deq = 448 * fp32(amax/448)
            sc = (amax / torch.tensor(448.0)).item()
            assert abs(qb[j].item()) == 448.0 * sc
            # relative error of e4m3 rounding: at most 2^-4 of the block's scale 2^e grid
            assert torch.all((qb - blk.to(F64)).abs() <= amax.item() / 448 * 2 ** -1 * 32 + 1e-12)


def test_weight_dequant_blocks():
    codes = torch.full((256, 128), 0x38, dtype=torch.uint8)     # all 1.0
    sc = torch.tensor([[2.0], [0.5]])
    wd = O.dequantize_weight_128x128(codes, sc)
    assert torch.all(wd[:128] == 2.0) and torch.all(wd[128:] == 0.5)


# ------------------------------------------------- FP8 layer composition
def _fp8_fixture():
    """The hand-worked FP8 layer of tests/golden/fp8_composition_small.json:
    e4m3 codes of the listed values, block scales 1, everything else 0."""
    g = _gold("fp8_composition_small.json")
    sh, inp = g["shape"], g["inputs"]
    D, L, F, E = sh["d_model"], sh["d_lat"], sh["d_ff"], sh["n_experts"]
    enc = lambda v: int(O.e4m3_encode(torch.tensor([v], dtype=F64)))

    def mat(rows, cols, entries):
        m = torch.zeros(rows, cols, dtype=torch.uint8)
        for i, j, v in entries:
            m[i, j] = enc(v)
        return m

    def experts(rows, cols, entries):
        m = torch.zeros(E, rows, cols, dtype=torch.uint8)
        m[0] = mat(rows, cols, entries)
        return m

    w = {"w_down": mat(L, D, inp["w_down"]), "w_up": mat(D, L, inp["w_up"]),
         "w_gate": experts(F, L, inp["w_gate_e0"]), "w_up_e": experts(F, L, inp["w_up_e_e0"]),
         "w_down_e": experts(L, F, inp["w_down_e_e0"]),
         "w_sh_gate": mat(F, L, inp["w_sh_gate"]), "w_sh_up": mat(F, L, inp["w_sh_up"]),
         "w_sh_down": mat(L, F, inp["w_sh_down"])}
    for nm in list(w):
        w["s_" + nm[2:]] = torch.ones(*w[nm].shape[:-2], 1, 1) if w[nm].dim() == 3 else torch.ones(1, 1)
    w["w_router"] = torch.zeros(sh["n_routers"], E, L, dtype=torch.bfloat16)
    for r, e, j, v in inp["w_router"]:
        w["w_router"][r, e, j] = v
    w["expert_scale"] = torch.tensor(inp["expert_scale"], dtype=torch.float32)
    gain = torch.full((L,), inp["rms_gain"]["default"], dtype=torch.float32)
    for j, v in inp["rms_gain"].items():
        if j != "default":
            gain[int(j)] = v
    w["rms_gain"] = gain
    x = torch.zeros(1, D, dtype=torch.bfloat16)
    for j, v in inp["x"].items():
        x[0, int(j)] = v
    return g, x, w, torch.tensor(inp["bias"], dtype=torch.float32)


def _fp8_run(x, w, b, g, skip=None):
    """The oracle's FP8 forward; with ``skip`` = i, its i-th activation
    quantisation (0 x, 1/2 the routed expert's z/h, 3/4 the shared
    expert's z/h, 5 n) is dropped: a planted mistake in the oracle."""
    import oracle.mrlmoe_oracle as MO
    real = MO.quantize_act_1x128
    calls = [0]

    def q(v):
        i = calls[0]
        calls[0] += 1
        return v.to(F64) if i == skip else real(v)

    MO.quantize_act_1x128 = q
    try:
        r = O.forward(x, w, b, g["shape"]["top_k"], g["shape"]["rms_eps"], fp8=True)
    finally:
        MO.quantize_act_1x128 = real
    return r, calls[0]


def test_fp8_layer_composition_hand_worked():
    g, x, w, b = _fp8_fixture()
    r, n_q = _fp8_run(x, w, b, g)
    assert n_q == 6                      # x; z, h of the routed expert; z, h of the shared expert; n
    ex = g["expected"]
    n = len(ex["c"])
    assert r.z[0, :4].tolist() == ex["z"]
    assert r.s[0].tolist() == ex["s"]
    assert r.topk_idx[0].tolist() == ex["topk_idx"] and r.topk_w[0].tolist() == ex["topk_w"]
    assert r.c[0, :n].tolist() == ex["c"] and torch.all(r.c[0, n:] == 0)
    assert r.n[0, :n].tolist() == ex["n"] and torch.all(r.n[0, n:] == 0)
    assert r.y[0, :n].tolist() == ex["y"] and torch.all(r.y[0, n:] == 0)


@pytest.mark.parametrize("skip", range(6))
def test_fp8_fixture_detects_each_dropped_quantisation(skip):
    # every quantisation point moves c or y of the hand-worked case: an
    # oracle that dropped any one of them would fail the fixture
    g, x, w, b = _fp8_fixture()
    r, _ = _fp8_run(x, w, b, g, skip=skip)
    ex = g["expected"]
    n = len(ex["c"])
    assert r.c[0, :n].tolist() != ex["c"] or r.y[0, :n].tolist() != ex["y"]


def test_fp8_fixture_detects_quantisation_before_rounding():
    # quantising h or n before their bf16 rounding changes the block scale,
    # so the fixture's c and y also pin the order (round, then quantise)
    g, _, _, _ = _fp8_fixture()
    un = g["unrounded"]
    for v_un, v_bf in ((un["h_routed_0"], 12.25), (un["n_0"], 7.0)):
        a = torch.zeros(1, 128, dtype=F64)
        a[0, 0] = v_un
        bq = torch.zeros(1, 128, dtype=F64)
        bq[0, 0] = v_bf
        assert O.bf16_round(a)[0, 0].item() == v_bf
        assert O.quantize_act_1x128(a)[0, 0].item() != O.quantize_act_1x128(bq)[0, 0].item() == v_bf


# ---------------------------------------------------- top-k boundary gap
def test_topk_boundary_gap_closed_forms():
    # gap = sb_(k) - sb_(k+1) of the biased scores sb = fp32(s + b), sorted descending
    gap = lambda s, b, k: O.topk_boundary_gap(torch.tensor([s], dtype=torch.float32),
                                              torch.tensor(b, dtype=torch.float32), k)[0].item()
    assert gap([0.5, 0.25, 0.75, 0.125], [0, 0, 0, 0], 2) == 0.25
    assert gap([0.5, 0.25, 0.75, 0.125], [0, 0, 0, 0], 1) == 0.25
    assert gap([0.5, 0.25, 0.75, 0.125], [0, 0, 0, 0], 3) == 0.125
    assert gap([0.5, 0.5, 0.5, 0.1], [0, 0, 0, 0], 1) == 0.0          # a tie at the boundary
    assert gap([0.5, 0.5, 0.5, 0.125], [0, 0, 0, 0], 3) == 0.375
    assert gap([0.0, -0.0, 1.0], [0, 0, 0], 2) == 0.0                 # +0 and -0 tie
    assert gap([0.5, 0.5], [0.0, 2 ** -10], 1) == 2 ** -10            # the bias decides
    assert gap([0.25, 0.75], [0.5, -0.125], 1) == 0.125               # sb = (0.75, 0.625)
    # sb is an fp32 sum: 1 + 2^-24 rounds to 1 (ties to even) before the difference
    assert gap([1.0, 1.0 + 2 ** -23], [2 ** -24, 0.0], 1) == 2 ** -23
    # the gap is taken row by row
    s = torch.tensor([[0.9, 0.1, 0.5], [0.2, 0.2, 0.3]], dtype=torch.float32)
    got = O.topk_boundary_gap(s, torch.zeros(3), 1)
    assert got.tolist() == [float(np.float32(0.9)) - float(np.float32(0.5)), float(np.float32(0.3)) - float(np.float32(0.2))]


# ------------------------------------------------------------- FP4 e2m1
# OCP Microscaling Formats (MX) v1.0, FP4 E2M1: exponent bias 1, one mantissa
# bit, exponent field 0 subnormal, no inf/NaN; the positive values are
# 0, 0.5, 1, 1.5, 2, 3, 4, 6.
E2M1_POSITIVE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_table():
    dec = O.e2m1_decode(torch.arange(16))
    assert dec[:8].tolist() == E2M1_POSITIVE
    assert dec[8:].tolist() == [-v for v in E2M1_POSITIVE]
    assert torch.signbit(dec[8])                                  # code 8 is -0
    assert torch.equal(O.e2m1_decode(torch.arange(16) + 16 * 5), dec)   # only the low nibble counts


def test_e2m1_values_are_exact_e4m3_values():
    # every e2m1 value has an e4m3 code of exactly that value (the FP4 GEMM
    # feeds its weights to the tensor core as e4m3 codes)
    dec = O.e2m1_decode(torch.arange(16))
    codes = O.e4m3_encode(dec)
    assert torch.equal(O.e4m3_decode(codes), dec)
    assert [int(c) for c in codes[:8]] == [0x00, 0x30, 0x38, 0x3C, 0x40, 0x44, 0x48, 0x4C]


def test_unpack_order_low_nibble_first():
    packed = torch.tensor([[0x21, 0xF8]], dtype=torch.uint8)
    assert O.unpack_e2m1(packed).tolist() == [[1, 2, 8, 15]]
    assert O.e2m1_decode(O.unpack_e2m1(packed)).tolist() == [[0.5, 1.0, -0.0, -6.0]]


def test_fp4_weight_dequant_blocks():
    # [200, 256]: two block rows (the second ragged) x two block columns
    codes = torch.zeros(200, 256, dtype=torch.int64)
    codes[:, :128] = 2                       # 1.0
    codes[:, 128:] = 15                      # -6.0
    codes[5, 7] = 1                          # 0.5
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).to(torch.uint8)
    sc = torch.tensor([[2.0, 0.25], [0.5, 4.0]])
    wd = O.dequantize_weight_fp4_128x128(packed, sc)
    assert wd.shape == (200, 256)
    assert torch.all(wd[:128, :128][codes[:128, :128] == 2] == 2.0) and wd[5, 7].item() == 1.0
    assert torch.all(wd[:128, 128:] == -1.5) and torch.all(wd[128:, :128] == 0.5)
    assert torch.all(wd[128:, 128:] == -24.0)


def test_fp4_layer_equals_fp8_layer_on_the_same_values():
    # the FP4 variant with e2m1 codes is the FP8 variant with the e4m3 codes
    # of the same values and the same scales: the oracle's FP4 mode must give
    # the FP8 mode's result exactly
    s = W.CONFIGS["c0_fp4"]
    w4 = W.make_layer_weights(s, "cpu")
    w8 = dict(w4)
    for nm in O.FP4_MATRICES:
        w8[nm] = O.e4m3_encode(O.e2m1_decode(O.unpack_e2m1(w4[nm])))
    x = W.make_x(s, "cpu")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, 950, "cpu")
    r4 = O.forward(x, w4, bias, s.top_k, s.rms_eps, fp4=True)
    r8 = O.forward(x, w8, bias, s.top_k, s.rms_eps, fp8=True)
    assert torch.equal(r4.y, r8.y) and torch.equal(r4.topk_idx, r8.topk_idx)
    # and it is not the bf16 layer: the weights really are 4-bit
    rb = O.forward(x, W.make_weights(s, "cpu"), bias, s.top_k, s.rms_eps)
    assert not torch.equal(r4.y, rb.y)


def test_fp4_input_quantiser_nearest_value():
    # the input generator's e2m1 rounding: every weight lands on the nearest
    # e2m1 multiple of its block scale (ties excepted), and the block maximum on +-6
    g = torch.Generator().manual_seed(12)
    w = torch.randn(256, 256, generator=g)
    packed, sc = W.to_fp4_blocks(w)
    wd = O.dequantize_weight_fp4_128x128(packed, sc)
    grid = torch.tensor(E2M1_POSITIVE, dtype=F64)
    for bi in range(2):
        for bj in range(2):
            blk = w[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128].to(F64)
            s_ = sc[bi, bj].item()
            dq = wd[bi * 128:(bi + 1) * 128, bj * 128:(bj + 1) * 128]
            assert abs(dq.abs().max().item() - 6.0 * s_) < 1e-12
            err = (dq - blk).abs()
            best = ((blk.abs()[..., None] / s_ - grid).abs().min(dim=-1).values * s_)
            assert torch.all(err <= best + 1e-9)


# ----------------------------------------------------- consistency with pages
def test_full_width_shapes_consistent_with_page_totals():
    s = W.CONFIGS["c2_prefill"]
    routed = 42 * s.n_experts * 3 * s.d_lat * s.d_ff        # 42 MoE layers (all but the first)
    assert routed <= 280e9                                    # 280B total parameters
    assert abs(routed / 42 * 2 / 1e9 - 12.88) < 0.01          # ~12.9 GB bf16 per layer
    assert W.flops_per_token(s) == 318_767_104
    assert W.flops_per_token(W.CONFIGS["c0_tiny"]) == 434_176
