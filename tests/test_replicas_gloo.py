"""Multi-process host logic of the replica scheme on CPU (gloo, world size 2).

The drafter shards by request: each rank holds a replica of the weights and runs its own
requests, with no collective on the data path.  These tests run two CPU processes that
(1) shard a batch of requests, run the oracle step on their share and check that the union
equals a single-process run, and (2) exercise the benchmark's barrier and max-over-ranks timing.
"""
import os
import socket

import numpy as np
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


def _init(rank, ws, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=120))


def _shard_worker(rank, ws, port, out):
    import dataclasses
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    from block_diffusion_drafter_dflash2_b200 import inputs
    from tests.parity import snapshot_request
    _init(rank, ws, port)
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=4, ctx_lo=10, ctx_hi=200)
    w = inputs.make_weights(wl.dims, wl.wseed)
    hw = oracle.HostWeights(w)
    st = inputs.make_state(wl)
    mine = [b for b in range(wl.batch) if b % ws == rank]   # request sharding, no data exchange
    paths = torch.full((wl.batch, wl.dims.block - 1), -1, dtype=torch.int32)
    for b in mine:
        sn = snapshot_request(wl, st, b)
        err, path, *_ = oracle.draft_request(wl.dims, hw, sn["taps"], sn["n"], sn["btok"], sn["kc"], sn["vc"], sn["pt"],
                                             sn["L0"])
        assert err == 0
        paths[b] = torch.from_numpy(path)
    # gather only to check the test's result (not part of the drafting path)
    gathered = [torch.zeros_like(paths) for _ in range(ws)]
    dist.all_gather(gathered, paths)
    if rank == 0:
        merged = torch.stack(gathered).max(0).values
        out.put(merged.numpy())
    dist.destroy_process_group()


def _timing_worker(rank, ws, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    _init(rank, ws, port)
    bench.barrier(ws)
    ms = 1.0 + rank  # rank-local step times
    m = bench.all_max(ms, ws)
    out.put((rank, m))
    dist.destroy_process_group()


def _run(fn, ws=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0, p.exitcode
    res = []
    while not q.empty():
        res.append(q.get())
    return res


def test_request_sharding_matches_single_process():
    import dataclasses
    import oracle
    from block_diffusion_drafter_dflash2_b200 import inputs
    from tests.parity import snapshot_request
    (merged,) = _run(_shard_worker)
    wl = dataclasses.replace(inputs.WORKLOADS["tiny"], batch=4, ctx_lo=10, ctx_hi=200)
    w = inputs.make_weights(wl.dims, wl.wseed)
    hw = oracle.HostWeights(w)
    st = inputs.make_state(wl)
    for b in range(wl.batch):
        sn = snapshot_request(wl, st, b)
        err, path, *_ = oracle.draft_request(wl.dims, hw, sn["taps"], sn["n"], sn["btok"], sn["kc"], sn["vc"], sn["pt"],
                                             sn["L0"])
        assert err == 0 and np.array_equal(merged[b], path)


def test_benchmark_timing_is_max_over_ranks():
    res = _run(_timing_worker)
    assert sorted(r for r, _ in res) == [0, 1]
    assert all(m == 2.0 for _, m in res)
