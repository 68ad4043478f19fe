"""The expert-parallel form of the layer (oracle/mrlmoe_ep.py) against the
single-GPU oracle, on CPU: every rank routes its own tokens, ships the
dispatched latent rows of each expert to the rank that owns it, gets the
expert outputs back and combines.  In process (the all-to-alls as list
transposes) and as separate gloo processes with real all-to-alls."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import workloads as W
from oracle import mrlmoe_ep as EP

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOKENS = [64, 37, 1, 50]   # a different batch on each rank


def _setup(n):
    s = W.CONFIGS["c0_tiny"]
    w = W.make_weights(s, "cpu")
    bias = W.uniform((s.n_experts,), -0.01, 0.01, 4, 900, "cpu")
    xs = [W.make_x(s, "cpu", seed=11 + r, T=TOKENS[r % len(TOKENS)]) for r in range(n)]
    return s, w, bias, xs


def _check_against_single_gpu(s, w, bias, xs, outs):
    for x, out in zip(xs, outs):
        ref = O.forward(x, w, bias, s.top_k, s.rms_eps)
        d = (out["c"] - ref.c).abs().max().item()
        assert d <= 1e-12 * max(1.0, ref.c.abs().max().item()), d
        # y is bf16: at most one step where c's last bits moved a rounding
        dy = (out["y"] - ref.y).abs()
        assert torch.all(dy <= ref.y.abs() * 2.0 ** -7 + 1e-30), dy.max()


@pytest.mark.parametrize("n", [1, 2, 4, 16])
def test_expert_parallel_equals_single_gpu(n):
    s, w, bias, xs = _setup(n)
    outs, recs = EP.ep_forward(xs, w, bias, s.top_k, s.rms_eps)
    _check_against_single_gpu(s, w, bias, xs, outs)


def test_send_slices_partition_the_dispatch_record():
    s, w, bias, xs = _setup(4)
    rec = EP.route_and_dispatch(xs[0], w, bias, s.top_k)
    bufs = EP.send_buffers(rec, 4)
    # the slices, in rank order, are the dispatched rows; each carries its experts' counts
    assert torch.equal(torch.cat([b for b, _ in bufs]), rec.rows)
    assert torch.equal(torch.cat([c for _, c in bufs]), rec.counts)
    assert sum(b.shape[0] for b, _ in bufs) == xs[0].shape[0] * s.top_k


def test_exchange_counts_and_latent_width():
    # every (token, slot) pair is a row that stays local or crosses once; in
    # the latent the bytes per row are d_lat / d_model of the hidden width
    s, w, bias, xs = _setup(4)
    _, recs = EP.ep_forward(xs, w, bias, s.top_k, s.rms_eps)
    lat = EP.exchange_bytes(recs, 4, s.d_lat)
    hid = EP.exchange_bytes(recs, 4, s.d_model)
    assert lat["remote_rows"] + lat["local_rows"] == sum(x.shape[0] for x in xs) * s.top_k
    assert lat["bytes"] * s.d_model == hid["bytes"] * s.d_lat
    assert lat["remote_rows"] > 0


def _free_port():
    so = socket.socket()
    so.bind(("127.0.0.1", 0))
    p = so.getsockname()[1]
    so.close()
    return p


def _ep_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    s, w, bias, xs = _setup(world)
    rec = EP.route_and_dispatch(xs[rank], w, bias, s.top_k)
    sends = EP.send_buffers(rec, world)
    L = s.d_lat
    per = s.n_experts // world
    # 1) row counts and per-expert counts, one fixed-size record per destination
    meta = torch.stack([torch.cat([torch.tensor([b.shape[0]]), c]) for b, c in sends]).to(torch.int64)
    meta_in = torch.empty_like(meta)
    dist.all_to_all_single(meta_in.view(-1), meta.view(-1))
    n_in = meta_in[:, 0].tolist()
    # 2) the rows themselves (latent width), uneven splits
    send_rows = torch.cat([b for b, _ in sends]).contiguous()
    recv_rows = torch.empty(sum(n_in), L, dtype=torch.float64)
    dist.all_to_all_single(recv_rows.view(-1), send_rows.view(-1),
                           output_split_sizes=[n * L for n in n_in],
                           input_split_sizes=[b.shape[0] * L for b, _ in sends])
    recv, a = [], 0
    for src in range(world):
        recv.append((recv_rows[a:a + n_in[src]], meta_in[src, 1:1 + per]))
        a += n_in[src]
    outs = EP.run_local_experts(rank, world, recv, w)
    # 3) the outputs back to their sources, in the order they came
    back = torch.empty_like(send_rows)
    dist.all_to_all_single(back.view(-1), torch.cat(outs).contiguous().view(-1),
                           output_split_sizes=[b.shape[0] * L for b, _ in sends],
                           input_split_sizes=[n * L for n in n_in])
    returned, a = [], 0
    for b, _ in sends:
        returned.append(back[a:a + b.shape[0]])
        a += b.shape[0]
    out = EP.combine(rec, returned, w, s.top_k, s.rms_eps)
    q.put((rank, out["c"], out["y"]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_over_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, c, y = q.get(timeout=300)
        got[r] = (c, y)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    s, w, bias, xs = _setup(world)
    outs, _ = EP.ep_forward(xs, w, bias, s.top_k, s.rms_eps)
    for r in range(world):
        # the same operations on the same rows as in one process: bit for bit
        assert torch.equal(got[r][0], outs[r]["c"]) and torch.equal(got[r][1], outs[r]["y"]), r
    _check_against_single_gpu(s, w, bias, xs, outs)


@pytest.mark.parametrize("n,agg", [(1, "mean"), (2, "mean"), (4, "sum"), (4, "max")])
def test_expert_parallel_backward_equals_single_gpu(n, agg):
    # the owners see only the rows they received; summed over ranks the
    # gradients are the single-GPU ones of the whole batch
    import dataclasses
    from oracle import mrlmoe_backward as B
    s, w, bias, xs = _setup(n)
    s = dataclasses.replace(s, aggregation=agg)
    dys = [W.make_dy(s, "cpu", seed=31 + r, T=x.shape[0]) for r, x in enumerate(xs)]
    dxs, grads = EP.ep_backward(xs, dys, w, bias, s.top_k, s.rms_eps, agg)
    fc = B.forward_for_grad(torch.cat(xs), w, bias, s.top_k, rms_eps=s.rms_eps, aggregation=agg)
    ref = B.backward(fc, w, torch.cat(dys), s.top_k, aggregation=agg)
    d = (torch.cat(dxs) - ref["x"]).abs().max().item()
    assert d <= 1e-10 * ref["x"].abs().max().item(), d
    for name, g in grads.items():
        d = (g - ref[name]).abs().max().item()
        assert d <= 1e-10 * max(1e-30, ref[name].abs().max().item()), (name, d)
