"""Expert-parallel form of the layer: the data plane around the library's
three phases (include/mrlmoe.h, "expert parallelism").

Rank d owns the routed experts [d E/n, (d+1) E/n).  Every rank routes its own
tokens (mrlmoe_ep_dispatch), sends each owner the contiguous slice of its
dispatched latent rows that belongs to the owner's experts together with
those experts' row counts, runs its own experts on what it received
(mrlmoe_ep_experts), returns the unweighted outputs to their sources in the
order they came, and combines (mrlmoe_ep_combine).  The pages motivate this
layout by the latent width of what crosses between GPUs (blog.derekhsu.net,
"ERNIE-5.5-Flash-Base", section "多路由潛在 MoE (Multi-Router Latent MoE)").

Two data planes share the same plan:

* ``DistributedExchange``: torch.distributed all-to-alls (NCCL between GPUs;
  gloo on CPU for the tests of this host logic).  The counts travel first (a
  fixed-size all-to-all), then the rows with uneven splits, then the outputs
  back with the splits reversed.
* ``emulate_forward``: all ranks in one process on one GPU.  The exchanges are
  plain device copies of the slices, and no rank touches another's memory.

The compute is the library's; this module only moves tensors and computes the
split sizes from the dispatch record.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

from . import _native as N


def owned_range(E: int, n_ranks: int, d: int):
    """Routed experts [lo, hi) of rank d."""
    if E % n_ranks:
        raise ValueError("the expert count must divide by the number of ranks")
    per = E // n_ranks
    return d * per, (d + 1) * per


def send_splits(offsets: Sequence[int], E: int, n_ranks: int) -> List[int]:
    """Rows this rank sends to each rank: the dispatch record's offsets at the
    owners' expert boundaries (offsets has E + 1 entries)."""
    per = E // n_ranks
    return [int(offsets[(d + 1) * per]) - int(offsets[d * per]) for d in range(n_ranks)]


def counts_by_destination(counts, n_ranks: int):
    """[n_ranks, E/n] view of the per-expert counts: row d goes to rank d."""
    return counts.view(n_ranks, -1)


@dataclass
class Dispatched:
    send_rows: object        # [T k, d_lat] bf16, expert-major
    counts: object           # [E] int32 (device)
    offsets_host: List[int]  # E + 1 offsets on the host (split sizes)


class ExpertParallelRank:
    """One rank's share of the layer: the replicated weights, its own routed
    experts (views of ``weights``' routed tensors, rows [lo, hi)), and one
    workspace for the three phases.  ``T`` is the largest token count any
    rank routes (it sizes what this rank can receive)."""

    def __init__(self, shape, weights: Dict[str, object], rank: int, n_ranks: int, device="cuda"):
        import torch
        self.shape, self.rank, self.n = shape, rank, n_ranks
        self.E = shape.n_experts
        self.lo, self.hi = owned_range(self.E, n_ranks, rank)
        self.w = weights
        self.cw = N.make_weights(weights)
        local = {k: weights[k][self.lo:self.hi] for k in ("w_gate", "w_up_e", "w_down_e")}
        self.w_local = local
        self.cw_local = N.make_weights(local)
        self.device = device
        self.cfg_max = N.make_config(shape)
        self.ws_bytes = N.mrlmoe_ep_workspace_size(self.cfg_max, n_ranks)
        if self.ws_bytes == 0:
            raise N.MrlmoeError(1, "mrlmoe_ep_workspace_size")
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)

    def _cfg(self, T: int):
        if T > self.cfg_max.T:
            raise ValueError(f"{T} tokens on a rank sized for {self.cfg_max.T}")
        return N.make_config(self.shape, T=T)

    def dispatch(self, x, bias, stream=None) -> Dispatched:
        """Phase 1: route this rank's tokens; the offsets come to the host (the
        split sizes of the all-to-alls)."""
        import torch
        T = x.shape[0]
        self.T = T
        cfg = self._cfg(T)
        k, L = self.shape.top_k, self.shape.d_lat
        i32 = dict(dtype=torch.int32, device=x.device)
        r = {"counts": torch.empty(self.E, **i32), "offsets": torch.empty(self.E + 1, **i32)}
        send = torch.empty(T * k, L, dtype=torch.bfloat16, device=x.device)
        N.mrlmoe_ep_dispatch(cfg, self.cw, bias, x, self.n, N.make_routing(r), send, self.workspace,
                             self.ws_bytes, stream)
        return Dispatched(send, r["counts"], r["offsets"].cpu().tolist())

    def experts(self, recv_rows, recv_counts, n_recv: int, stream=None):
        """Phase 3: this rank's experts on the received rows (recv_counts
        [n, E/n] int32 on the device); unweighted fp32 outputs in arrival order."""
        import torch
        cfg = self._cfg(self.T)
        out = torch.empty(max(n_recv, 1), self.shape.d_lat, dtype=torch.float32, device=recv_counts.device)[:n_recv]
        N.mrlmoe_ep_experts(cfg, self.cw_local, self.n, recv_rows if n_recv else None, recv_counts, n_recv,
                            out if n_recv else None, self.workspace, self.ws_bytes, stream)
        return out

    def combine(self, ret_rows, stream=None):
        """Phase 5: y [T, d_model] bf16 from the returned rows (dispatch order)."""
        import torch
        cfg = self._cfg(self.T)
        y = torch.empty(self.T, self.shape.d_model, dtype=torch.bfloat16, device=ret_rows.device)
        N.mrlmoe_ep_combine(cfg, self.cw, ret_rows, y, self.workspace, self.ws_bytes, stream)
        return y

    def status(self, stream=None) -> int:
        return N.mrlmoe_get_device_status(self.workspace, stream)


class DistributedExchange:
    """The two exchanges of the layer over a torch.distributed process group
    (one rank per process).  Every rank takes the same collective steps in
    the same order."""

    def __init__(self, n_ranks: int, E: int, group=None):
        self.n, self.E, self.group = n_ranks, E, group

    def counts(self, counts):
        """counts [E] -> [n, E/n]: row s = source s's counts for this rank's experts."""
        import torch.distributed as dist
        send = counts_by_destination(counts, self.n).contiguous()
        recv = send.new_empty(send.shape)
        dist.all_to_all_single(recv, send, group=self.group)
        return recv

    def rows(self, send_rows, send_split: List[int], recv_split: List[int]):
        """The dispatched rows: each destination its slice (uneven splits)."""
        import torch.distributed as dist
        recv = send_rows.new_empty((sum(recv_split),) + tuple(send_rows.shape[1:]))
        dist.all_to_all_single(recv, send_rows, output_split_sizes=recv_split, input_split_sizes=send_split,
                               group=self.group)
        return recv

    def back(self, out_rows, send_split: List[int], recv_split: List[int]):
        """The outputs back to their sources, in the order they came: what a
        source receives is its own rows in dispatch order."""
        import torch.distributed as dist
        ret = out_rows.new_empty((sum(send_split),) + tuple(out_rows.shape[1:]))
        dist.all_to_all_single(ret, out_rows, output_split_sizes=send_split, input_split_sizes=recv_split,
                               group=self.group)
        return ret


def forward_distributed(rank: ExpertParallelRank, x, bias, exchange: Optional[DistributedExchange] = None):
    """The layer on this rank's tokens, experts on their owners (one process
    per rank).  Returns y."""
    ex = exchange or DistributedExchange(rank.n, rank.E)
    d = rank.dispatch(x, bias)
    s_split = send_splits(d.offsets_host, rank.E, rank.n)
    rc = ex.counts(d.counts)
    r_split = [int(v) for v in rc.sum(1).tolist()]
    recv = ex.rows(d.send_rows, s_split, r_split)
    out = rank.experts(recv, rc, sum(r_split))
    ret = ex.back(out, s_split, r_split)
    return rank.combine(ret)


def emulate_forward(ranks: Sequence[ExpertParallelRank], xs: Sequence[object], bias, events: Optional[dict] = None):
    """All ranks in one process on one GPU: each exchange is a device copy of
    every (source, destination) slice into the destination's receive buffer.
    Returns the list of y, one per rank.  With ``events`` (a dict), CUDA
    events are recorded around each rank's phases on the current stream:
    events[phase] is a list of (start, end) pairs, phase one of "dispatch"
    and "combine" (per source rank), "experts" (per owner), "rows" and
    "back" (the two exchanges, all ranks' copies together); events["splits"]
    holds the rows each rank sent each rank."""
    import torch
    n = len(ranks)
    E = ranks[0].E
    per = E // n

    def mark(phase):
        if events is None:
            return None
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        events.setdefault(phase, []).append((a, b))
        a.record()
        return b

    disp = []
    for rk, x in zip(ranks, xs):
        e = mark("dispatch")
        disp.append(rk.dispatch(x, bias))
        if e is not None:
            e.record()
    splits = [send_splits(d.offsets_host, E, n) for d in disp]       # splits[s][d]
    if events is not None:
        events["splits"] = splits
    starts = [[0] * n for _ in range(n)]
    for s in range(n):
        for d in range(1, n):
            starts[s][d] = starts[s][d - 1] + splits[s][d - 1]
    recvs, rcs = [], []
    e = mark("rows")
    for d in range(n):
        rc = torch.stack([counts_by_destination(disp[s].counts, n)[d] for s in range(n)]).contiguous()
        n_in = sum(splits[s][d] for s in range(n))
        recv = torch.empty(n_in, ranks[d].shape.d_lat, dtype=torch.bfloat16, device=rc.device)
        a = 0
        for s in range(n):
            m = splits[s][d]
            recv[a:a + m].copy_(disp[s].send_rows[starts[s][d]:starts[s][d] + m])
            a += m
        assert rc.shape == (n, per)
        recvs.append(recv)
        rcs.append(rc)
    if e is not None:
        e.record()
    outs = []
    for d in range(n):
        e = mark("experts")
        outs.append(ranks[d].experts(recvs[d], rcs[d], recvs[d].shape[0]))
        if e is not None:
            e.record()
    rets = []
    e = mark("back")
    for s in range(n):
        ret = torch.empty(disp[s].send_rows.shape[0], ranks[s].shape.d_lat, dtype=torch.float32,
                          device=disp[s].send_rows.device)
        for d in range(n):
            # where source s's rows sit in owner d's arrival order
            a = sum(splits[q][d] for q in range(s))
            m = splits[s][d]
            ret[starts[s][d]:starts[s][d] + m].copy_(outs[d][a:a + m])
        rets.append(ret)
    if e is not None:
        e.record()
    ys = []
    for s in range(n):
        e = mark("combine")
        ys.append(ranks[s].combine(rets[s]))
        if e is not None:
            e.record()
    return ys
