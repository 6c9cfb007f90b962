"""Multi-GPU host logic on CPU: two gloo ranks run the replica plumbing the
benchmark uses (rank discovery, per-rank token seeds, identical weights, the
max-over-ranks time and the whole-job throughput)."""
import os
import socket
from dataclasses import replace

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_63_b200 import replicas
from mixture_experts_layer_63_b200.inputs import WORKLOADS, make_inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        info = replicas.rank_info()
        w = replace(WORKLOADS["gshard"], T=64, d_model=64, d_ff=64)
        inp = make_inputs(w, seed=0, device="cpu")
        g = torch.Generator().manual_seed(replicas.token_seed(0, info.rank, info.world))
        x = torch.randn(w.T, w.d_model, generator=g)
        # per-rank elapsed times: rank 1 is the slow one
        t_max = replicas.max_over_ranks(10.0 + 5.0 * info.rank, dist)
        w_all = [torch.zeros_like(inp.w1) for _ in range(world)]
        dist.all_gather(w_all, inp.w1)
        x_all = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(x_all, x)
        q.put((info.rank, info.world, t_max,
               all(torch.equal(w_all[0], wi) for wi in w_all),
               not torch.equal(x_all[0], x_all[1]),
               replicas.throughput(info.world, w.T, 3, t_max)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, t_max, same_w, diff_x, tput in out:
        assert w == world
        assert t_max == 15.0                       # the slowest rank's time on every rank
        assert same_w                              # every replica holds the same layer
        assert diff_x                              # each rank its own tokens
        assert abs(tput - 2 * 64 * 3 / 0.015) < 1e-6


def test_single_process_defaults():
    info = replicas.rank_info({})
    assert (info.rank, info.world, info.local_rank) == (0, 1, 0)
    assert replicas.token_seed(7, 0, 1) == 7
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.throughput(1, 4096, 20, 4.0) == 4096 * 20 / 0.004
