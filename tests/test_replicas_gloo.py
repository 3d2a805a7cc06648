"""Multi-rank host logic of the benchmark, on CPU with gloo (world size 2):
replicas draw independent batches, compute independently, and the job's step
time is the slowest rank's.  The layer itself has no exchange step on one
device, so there is nothing else to reduce across ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle.moe_oracle as O
from expert_dispatch_router_b200 import synth

SHAPE = synth.GSHARD_TOP2.replace(name="replica", T=96, H=16, F=24, E=6, k=2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica_result(rank):
    inp = synth.make_inputs(SHAPE, seed=bench.replica_seed(0, rank), device="cpu")
    d = lambda t: None if t is None else t.double().numpy()
    layer = O.OracleLayer.from_mapping(SHAPE.as_dict())
    out = O.layer_forward(layer, d(inp["x"]), d(inp["wg"]), d(inp["w1"]), d(inp["w2"]))
    return out["y"], out["aux"]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        y, aux = _replica_result(rank)
        ms = 1.0 + 0.5 * rank                       # a per-rank step time
        worst = bench.max_over_ranks(ms, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, (rank, float(aux), float(np.abs(y).sum()), worst))
        if rank == 0:
            q.put(gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res = sorted(res)
    # the slowest rank's time on every rank
    assert all(r[3] == 1.5 for r in res)
    # replicas are independent: each equals a single-process run of its own seed
    for rank, aux, ysum, _ in res:
        y, a = _replica_result(rank)
        assert abs(aux - a) < 1e-12 and abs(ysum - float(np.abs(y).sum())) < 1e-9
    assert res[0][1] != res[1][1]
    assert bench.job_tokens_per_s(SHAPE.T, world, 1.5) == pytest.approx(2 * 96 / 1.5e-3)
