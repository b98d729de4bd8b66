"""Data-parallel replicas: the host-side exchange of the per-expert load.

Two gloo ranks on CPU each route their own token shard (with the oracle,
since no GPU is needed to check the exchange), all-reduce the load through
mixture_experts_layer_60_b200.parallel_load, and apply the bias rule.  Every
rank must end with the same bias, equal to one process routing the whole
batch; a rank that leaves early must make the others fail, not hang."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as O


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _batch(T, d, N_r, seed=0):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((T, d))
    E = rng.standard_normal((N_r, d)) / np.sqrt(d)
    b = rng.uniform(-0.01, 0.01, N_r).astype(np.float32)
    return u, E, b


def _worker(rank, world, port, T, d, N_r, K, steps, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from mixture_experts_layer_60_b200.parallel_load import allreduce_load
    u, E, b = _batch(T * world, d, N_r)
    shard = u[rank * T:(rank + 1) * T]
    for s in range(steps):
        r = O.route(shard, E, b, K)
        counts, T_total = allreduce_load(torch.from_numpy(r["counts"]), T)
        assert T_total == T * world
        b = O.bias_update(b, counts.numpy(), T_total, K)
        # the same exchange with the token total known in advance
        counts2, T2 = allreduce_load(torch.from_numpy(r["counts"]), T, T_total=T * world)
        assert torch.equal(counts, counts2) and T2 == T_total
    out_q.put((rank, b.tobytes()))
    dist.destroy_process_group()


def test_two_rank_load_allreduce_matches_single_process():
    world, T, d, N_r, K, steps = 2, 96, 32, 16, 4, 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, d, N_r, K, steps, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    b0 = np.frombuffer(res[0], np.float32)
    b1 = np.frombuffer(res[1], np.float32)
    np.testing.assert_array_equal(b0, b1)
    # single process over the whole batch
    u, E, b = _batch(T * world, d, N_r)
    for _ in range(steps):
        r = O.route(u, E, b, K)
        b = O.bias_update(b, r["counts"], T * world, K)
    np.testing.assert_array_equal(b0, b)


def _leaver(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    from mixture_experts_layer_60_b200.parallel_load import allreduce_load
    c = torch.ones(8, dtype=torch.int32)
    allreduce_load(c, 10, T_total=20)          # one good step on every rank
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()                          # flush the message before leaving
        os._exit(0)                              # leaves between steps, nothing in flight
    try:
        allreduce_load(c, 10, T_total=20)
        q.put((rank, "no error"))
    except Exception as e:                       # the survivor sees an error, not a hang
        q.put((rank, "error:" + type(e).__name__))


def test_rank_leaving_between_steps_is_an_error_not_a_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_leaver, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=90) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert res[1] == "left"
    assert res[0].startswith("error:"), res[0]
