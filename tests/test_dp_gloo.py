"""Data-parallel decomposition on CPU (gloo, world size 2).

Each rank holds the same NF4 weight and adapters and its own tokens; the
adapter gradients are the only exchange (a sum over ranks).  This checks, with
the oracle on the host, that the per-rank gradients summed by an all-reduce
equal the gradients of the concatenated global batch, and that every rank
sees the same frozen weight — the host-side logic `bench.py --gpus N` uses —
and that an 8-bit AdamW step after the all-reduce leaves the adapter replicas
and their optimizer states bit-identical across ranks.
"""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from oracle import linear as ol
from oracle import nf4

LIN = synth.Linear("dp", 128, 192)
M_PER_RANK, R, S = 24, 16, 0.5


def _bits(t):
    return synth.bf16_bits(t)


def _wd(d):
    codes, c8, s2 = nf4.quantize(_bits(d["W"]).reshape(-1))
    return nf4.dequantize(codes, c8, s2, d["W"].numel()).reshape(d["W"].shape)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = synth.dp_shard_inputs(LIN, M_PER_RANK, R, rank)
        wsum = torch.tensor([float(np.sum(_bits(d["W"]).astype(np.int64)))], dtype=torch.float64)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, wsum)
        _, dA, dB, _ = ol.linear_bwd(_bits(d["dY"]), _bits(d["X"]), _wd(d), _bits(d["A"]), _bits(d["B"]), S)
        tA, tB = torch.from_numpy(dA), torch.from_numpy(dB)
        dist.all_reduce(tA)
        dist.all_reduce(tB)
        if rank == 0:
            q.put((len({float(x) for x in sums}), tA.numpy(), tB.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_gradient_sum_equals_global_batch():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    n_distinct_w, dA, dB = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert n_distinct_w == 1, "ranks hold different frozen weights"
    shards = [synth.dp_shard_inputs(LIN, M_PER_RANK, R, r) for r in range(world)]
    X = np.concatenate([_bits(s["X"]) for s in shards])
    dY = np.concatenate([_bits(s["dY"]) for s in shards])
    d0 = shards[0]
    _, dA_ref, dB_ref, _ = ol.linear_bwd(dY, X, _wd(d0), _bits(d0["A"]), _bits(d0["B"]), S)
    assert np.allclose(dA, dA_ref, rtol=1e-12, atol=1e-14)
    assert np.allclose(dB, dB_ref, rtol=1e-12, atol=1e-14)


def _opt_worker(rank, world, port, q):
    """All-reduce the fp32 adapter gradients, then take one 8-bit AdamW step on
    this rank's replica of A and B (oracle): the replicas must stay identical."""
    from oracle import optim
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = synth.dp_shard_inputs(LIN, M_PER_RANK, R, rank)
        _, dA, dB, _ = ol.linear_bwd(_bits(d["dY"]), _bits(d["X"]), _wd(d), _bits(d["A"]), _bits(d["B"]), S)
        out = []
        for p, g in ((_bits(d["A"]), dA), (_bits(d["B"]), dB)):
            t = torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32).reshape(-1))
            dist.all_reduce(t)
            p1, st1 = optim.adamw8_step(p.reshape(-1), t.numpy(), optim.init_state(t.numel()), 2e-4, 0.9, 0.999,
                                        1e-8, 0.0, 1)
            out.append((p1, st1, t.numpy().copy()))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_rank_optimizer_step_keeps_replicas_identical():
    from oracle import optim
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_opt_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d0 = synth.dp_shard_inputs(LIN, M_PER_RANK, R, 0)
    for k, p0 in enumerate((_bits(d0["A"]), _bits(d0["B"]))):
        (pa, sa, ga), (pb, sb, gb) = res[0][k], res[1][k]
        assert np.array_equal(ga, gb)                        # same summed gradient on both ranks
        assert np.array_equal(pa, pb)                        # replicas identical after the step
        assert all(np.array_equal(x, y) for x, y in zip(sa, sb))
        p1, _ = optim.adamw8_step(p0.reshape(-1), ga, optim.init_state(ga.size), 2e-4, 0.9, 0.999, 1e-8, 0.0, 1)
        assert np.array_equal(pa, p1)                        # equals the single-process step on the sum
