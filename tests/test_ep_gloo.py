"""Host side of expert parallelism on CPU (gloo, 2 ranks): the loads of all
ranks are gathered in rank order on every rank, and the receive totals they
imply cover every routed row exactly once."""
import os
import socket
import traceback

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from mixture_experts_layer_60_b200.parallel_ep import gather_counts
        N_r, T, K = 16, 50 + 7 * rank, 4
        g = torch.Generator().manual_seed(100 + rank)
        idx = torch.stack([torch.randperm(N_r, generator=g)[:K] for _ in range(T)])
        counts = torch.bincount(idx.reshape(-1), minlength=N_r).to(torch.int32)
        allc = gather_counts(counts)
        E_loc = N_r // world
        recv = [int(allc[:, d * E_loc:(d + 1) * E_loc].sum()) for d in range(world)]
        q.put((rank, allc.tolist(), counts.tolist(), recv, T * K))
    except Exception:
        q.put((rank, "error", traceback.format_exc(), None, None))
    finally:
        dist.destroy_process_group()


def test_gather_counts_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        r, allc, counts, recv, rows = q.get(timeout=120)
        assert allc != "error", counts
        out[r] = (allc, counts, recv, rows)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0]                         # same gathered table everywhere
    assert out[0][0] == [out[0][1], out[1][1]]            # in rank order
    assert sum(out[0][2]) == out[0][3] + out[1][3]        # every routed row received once
