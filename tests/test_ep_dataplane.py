"""Host logic of the expert-parallel data plane (sparse_moe_layer_mean_b200/ep.py)
on CPU: gloo ranks in separate processes run the product's exchange steps
(counts, rows, and outputs back, with the split sizes it derives from the
dispatch record), with the oracle's phases as the compute on each rank.  The
result must equal the in-process expert-parallel oracle bit for bit, and the
single-GPU oracle within rounding."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import workloads as W
from oracle import mrlmoe_ep as OEP
from sparse_moe_layer_mean_b200 import ep as EP

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOKENS = [64, 37, 1, 50]


def _setup(n):
    s = W.CONFIGS["c0_tiny"]
    w = W.make_weights(s, "cpu")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, 900, "cpu")
    xs = [W.make_x(s, "cpu", seed=11 + r, T=TOKENS[r % len(TOKENS)]) for r in range(n)]
    return s, w, bias, xs


def test_send_splits_and_counts_view():
    offsets = [0, 3, 3, 7, 10, 10, 12, 15, 20]                     # E = 8
    assert EP.send_splits(offsets, 8, 2) == [10, 10]
    assert EP.send_splits(offsets, 8, 4) == [3, 7, 2, 8]
    assert EP.send_splits(offsets, 8, 1) == [20]
    c = torch.arange(8)
    assert EP.counts_by_destination(c, 4).tolist() == [[0, 1], [2, 3], [4, 5], [6, 7]]
    assert EP.owned_range(8, 4, 3) == (6, 8)
    with pytest.raises(ValueError):
        EP.owned_range(10, 4, 0)


def _free_port():
    so = socket.socket()
    so.bind(("127.0.0.1", 0))
    p = so.getsockname()[1]
    so.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    s, w, bias, xs = _setup(world)
    ex = EP.DistributedExchange(world, s.n_experts)
    # phase 1 (oracle compute on this rank's tokens)
    rec = OEP.route_and_dispatch(xs[rank], w, bias, s.top_k)
    s_split = EP.send_splits(rec.offsets.tolist(), s.n_experts, world)
    # exchange 1: counts, then the rows
    rc = ex.counts(rec.counts)
    r_split = [int(v) for v in rc.sum(1).tolist()]
    recv = ex.rows(rec.rows.contiguous(), s_split, r_split)
    # phase 3 (oracle compute on what arrived, source by source)
    pieces, a = [], 0
    for src in range(world):
        pieces.append((recv[a:a + r_split[src]], rc[src]))
        a += r_split[src]
    outs = OEP.run_local_experts(rank, world, pieces, w)
    # exchange 2: outputs back, then the combine on the source
    ret = ex.back(torch.cat(outs).contiguous(), s_split, r_split)
    returned, a = [], 0
    for n in s_split:
        returned.append(ret[a:a + n])
        a += n
    out = OEP.combine(rec, returned, w, s.top_k, s.rms_eps)
    q.put((rank, out["c"], out["y"], s_split, r_split))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_data_plane_over_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r, c, y, s_split, r_split = q.get(timeout=300)
        got[r] = (c, y, s_split, r_split)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    s, w, bias, xs = _setup(world)
    outs, recs = OEP.ep_forward(xs, w, bias, s.top_k, s.rms_eps)
    for r in range(world):
        c, y, s_split, r_split = got[r]
        assert torch.equal(c, outs[r]["c"]) and torch.equal(y, outs[r]["y"])
        ref = O.forward(xs[r], w, bias, s.top_k, s.rms_eps)
        assert (c - ref.c).abs().max().item() <= 1e-12 * max(1.0, ref.c.abs().max().item())
        # what rank r sent each rank is what that rank received from r
        assert s_split == [got[d][3][r] for d in range(world)]
        assert sum(s_split) == xs[r].shape[0] * s.top_k
