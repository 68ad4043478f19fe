"""CPU reading of the routing-record invariants that the device checker
(mrlmoe_check_routing) reports, plus records to feed it: valid ones built by
the oracle's selection and dispatch, and single corruptions made on the host.

The invariants (the dispatch record of the layer: each token picks k distinct
experts of E, entries grouped expert-major in ascending t*k+j order):

  index      an expert index outside [0, E)
  duplicate  a token selects one expert twice
  offsets    a negative count, or offsets not the exclusive scan of counts
             (offsets[0] = 0, offsets[e+1] - offsets[e] = counts[e],
             offsets[E] = T*k)
  perm       perm, inv_perm not inverse bijections of [0, T*k): for every
             entry f, inv[f] in range and perm[inv[f]] = f; for every row r,
             perm[r] in range and inv[perm[r]] = r
  group      a row r whose entry f = perm[r] passes the perm test for r and
             has an in-range expert e, but r is outside
             [offsets[e], offsets[e] + counts[e])
  order      such a row r inside its range, whose next row r+1 is still
             inside it (and < T*k), holds an entry f2 = perm[r+1] in range of
             the same expert with f2 <= f
  weight     a routing weight that is not finite

Test infrastructure only.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import workloads as W

CHECK = {"index": 1, "duplicate": 2, "offsets": 4, "perm": 8, "group": 16, "order": 32, "weight": 64}


def record_faults(rec, T: int, E: int, k: int) -> int:
    """OR of the CHECK bits that ``rec`` (dict of tensors or arrays with the
    mrlmoe_routing field names; topk_w optional) violates."""
    def a(name):
        v = rec[name]
        return (v.cpu().numpy() if isinstance(v, torch.Tensor) else np.asarray(v)).reshape(-1).astype(np.int64)

    Tk = T * k
    idx, counts, offsets, perm, inv = a("topk_idx"), a("counts"), a("offsets"), a("perm"), a("inv_perm")
    bits = 0
    if np.any((idx < 0) | (idx >= E)):
        bits |= CHECK["index"]
    rows = np.sort(idx.reshape(T, k), axis=1)
    if k > 1 and np.any(rows[:, 1:] == rows[:, :-1]):
        bits |= CHECK["duplicate"]
    if (np.any(counts < 0) or np.any(offsets[1:] - offsets[:-1] != counts) or offsets[0] != 0
            or offsets[E] != Tk):
        bits |= CHECK["offsets"]
    ar = np.arange(Tk)
    inv_in = (inv >= 0) & (inv < Tk)
    perm_in = (perm >= 0) & (perm < Tk)
    entry_ok = inv_in & (perm[np.where(inv_in, inv, 0)] == ar)
    row_ok = perm_in & (inv[np.where(perm_in, perm, 0)] == ar)
    if not (entry_ok.all() and row_ok.all()):
        bits |= CHECK["perm"]
    f = np.where(row_ok, perm, 0)
    e = idx[f]
    e_in = row_ok & (e >= 0) & (e < E)
    ec = np.where(e_in, e, 0)
    lo = offsets[ec]
    hi = lo + counts[ec]
    if np.any(e_in & ((ar < lo) | (ar >= hi))):
        bits |= CHECK["group"]
    inside = e_in & (ar >= lo) & (ar < hi)
    nxt = inside & (ar + 1 < hi) & (ar + 1 < Tk)
    r = ar[nxt]
    f2 = perm[r + 1]
    f2_in = (f2 >= 0) & (f2 < Tk)
    same = f2_in & (idx[np.where(f2_in, f2, 0)] == e[nxt])
    if np.any(same & (f2 <= f[nxt])):
        bits |= CHECK["order"]
    w = rec.get("topk_w")
    if w is not None:
        wv = w.cpu().numpy() if isinstance(w, torch.Tensor) else np.asarray(w)
        if not np.all(np.isfinite(wv)):
            bits |= CHECK["weight"]
    return bits


def oracle_record(T: int, E: int, k: int, seed: int, hot: int = 0):
    """A valid record from the oracle: scores U(0, 1) from the seeded
    generator, selection and weights by the oracle's top-k, dispatch by its
    stable sort.  ``hot`` > 0 adds +10 to the bias of experts 0..hot-1, so
    every token picks them (long segments, many empty experts)."""
    s = W.uniform((T, E), 0.0, 1.0, seed, 1, "cpu")
    bias = torch.zeros(E, dtype=torch.float32)
    bias[:hot] = 10.0
    idx = O.select_topk(s, bias, k)
    w, _ = O.route_weights(s, idx, torch.ones(E))
    counts, offsets, perm, inv = O.permutation(idx, E)
    i32 = lambda t: t.reshape(-1).to(torch.int32).contiguous()
    return {"topk_idx": i32(idx), "topk_w": w.reshape(-1).to(torch.float32).contiguous(),
            "counts": i32(counts), "offsets": i32(offsets), "perm": i32(perm), "inv_perm": i32(inv)}


def _segment_with_two_rows(rec, E):
    c = rec["counts"].long()
    e = int(torch.nonzero(c >= 2)[0])
    return e, int(rec["offsets"][e])


def corrupt(rec, kind: str, T: int, E: int, k: int):
    """(corrupted copy, expected bits): one host-side corruption of a valid
    record, with the invariants it breaks by the definitions above."""
    r = {n: v.clone() for n, v in rec.items()}
    Tk = T * k
    t = T // 2
    if kind == "index_high":
        r["topk_idx"][t * k] = E
        return r, CHECK["index"]
    if kind == "index_negative":
        r["topk_idx"][t * k + k - 1] = -1
        return r, CHECK["index"]
    if kind == "weight_nan":
        r["topk_w"][3 % Tk] = float("nan")
        return r, CHECK["weight"]
    if kind == "weight_inf":
        r["topk_w"][Tk - 1] = float("inf")
        return r, CHECK["weight"]
    if kind == "duplicate":
        # (t, 1) now names the expert of (t, 0); its row stays in the old segment
        r["topk_idx"][t * k + 1] = r["topk_idx"][t * k]
        return r, CHECK["duplicate"] | CHECK["group"]
    if kind == "order_swap":
        # two adjacent rows of one expert swapped consistently in perm and inv_perm
        e, r0 = _segment_with_two_rows(rec, E)
        a, b = int(r["perm"][r0]), int(r["perm"][r0 + 1])
        r["perm"][r0], r["perm"][r0 + 1] = b, a
        r["inv_perm"][a], r["inv_perm"][b] = r0 + 1, r0
        return r, CHECK["order"]
    if kind == "group_swap":
        # the first rows of two different non-empty experts swapped consistently
        ne = torch.nonzero(rec["counts"].long() > 0).flatten()
        e1, e2 = int(ne[0]), int(ne[1])
        r1, r2 = int(rec["offsets"][e1]), int(rec["offsets"][e2])
        a, b = int(r["perm"][r1]), int(r["perm"][r2])
        r["perm"][r1], r["perm"][r2] = b, a
        r["inv_perm"][a], r["inv_perm"][b] = r2, r1
        return r, CHECK["group"]
    if kind == "perm_only_swap":
        # perm changed, inv_perm not: no longer inverse
        r["perm"][0], r["perm"][Tk - 1] = rec["perm"][Tk - 1], rec["perm"][0]
        return r, CHECK["perm"]
    if kind == "inv_shift":
        f = int(rec["perm"][0])
        r["inv_perm"][f] = (int(rec["inv_perm"][f]) + 1) % Tk
        return r, CHECK["perm"]
    if kind == "perm_out_of_range":
        r["perm"][Tk // 3] = Tk + 5
        return r, CHECK["perm"]
    if kind == "offset_bump":
        # a non-empty expert's range starts one row late: its first row is outside
        ne = torch.nonzero(rec["counts"].long() > 0).flatten()
        e = int(ne[ne > 0][0])
        r["offsets"][e] += 1
        return r, CHECK["offsets"] | CHECK["group"]
    if kind == "offset_total":
        r["offsets"][E] = Tk - 1
        return r, CHECK["offsets"]
    if kind == "count_negative":
        ne = torch.nonzero(rec["counts"].long() > 0).flatten()
        r["counts"][int(ne[0])] = -1
        return r, CHECK["offsets"] | CHECK["group"]
    raise ValueError(kind)


KINDS = ("index_high", "index_negative", "weight_nan", "weight_inf", "duplicate", "order_swap", "group_swap",
         "perm_only_swap", "inv_shift", "perm_out_of_range", "offset_bump", "offset_total", "count_negative")
