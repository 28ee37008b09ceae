"""The N > 1 benchmark path on CPU: two gloo ranks run bench.py's
aggregation (the job time is the slowest rank's device time, the value
counts every rank's units) and get different replica seeds.  The GPU path
itself needs one GPU per rank and no data-path collective (replicas)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from lut_logits_serving_b200 import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = [12.5, 20.0][rank]
    job = bench.aggregate(local_ms, world)
    value = bench.throughput(1000, world, job)
    w = synth.WORKLOADS["tiny"]
    d = synth.make(w, seed=bench.rank_seed(rank))
    q.put((rank, job, value, int(d["codes"][0, 0, 0]), float(d["h"][0, 0])))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, job0, v0, c0, h0), (r1, job1, v1, c1, h1) = res
    assert job0 == job1 == 20.0                       # max over ranks
    assert v0 == v1 == pytest.approx(2 * 1000 / 0.020)
    assert (c0, h0) != (c1, h1)                       # each replica its own inputs


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(7.0, 1) == 7.0
    assert bench.throughput(256000, 1, 0.1) == pytest.approx(2.56e9)


def _shard_worker(rank, world, port, q):
    """The exchange of the vocabulary-sharded pick: shard_rows covers the rows
    once, and all_gather_into_tensor lays the ranks' per-token winners out
    rank-major, [world][B], as rq_argmax_merge reads them."""
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import lut_logits_serving_b200 as rq
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    V, B = 1001, 5
    r0, r1 = rq.shard_rows(V, rank, world)
    val = torch.arange(B, dtype=torch.float32) + 100 * rank
    gidx = torch.full((B,), r0, dtype=torch.int32)
    vals = torch.empty((world * B,), dtype=torch.float32)   # flat, as rq_sharded_logits
    idxs = torch.empty((world * B,), dtype=torch.int32)
    dist.all_gather_into_tensor(vals, val)
    dist.all_gather_into_tensor(idxs, gidx)
    q.put((rank, r0, r1, vals.view(world, B).tolist(), idxs.view(world, B).tolist()))
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_pick_exchange_layout_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    bounds = [(r0, r1) for _, r0, r1, _, _ in res]
    assert bounds[0][0] == 0 and bounds[-1][1] == 1001
    assert all(bounds[i][1] == bounds[i + 1][0] for i in range(world - 1))
    for _, _, _, vals, idxs in res:
        assert vals == [[b + 100.0 * k for b in range(5)] for k in range(world)]
        assert idxs == [[bounds[k][0]] * 5 for k in range(world)]


def _sharded_call_worker(rank, world, port, q):
    """rq_sharded_logits itself over gloo, its three device calls replaced by
    CPU stand-ins that read a fixed full logits matrix: what is checked is the
    glue -- process-group size, the flat all-gathers, the [world][B] layout
    handed to the merge -- against the argmax of the full matrix."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import lut_logits_serving_b200 as rq
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    V, B = 1003, 4
    full = torch.from_numpy(np.random.default_rng(7).standard_normal((B, V)).astype(np.float32))
    r0, r1 = rq.shard_rows(V, rank, world)

    def logits_from_hidden(h, C, codes, fmt, d, softcap, want_argmax, ws, stream):
        part = full[:, r0:r1].contiguous()
        return part, part.argmax(dim=1).to(torch.int32), ws

    def candidates(logits, am, row0, stream=None):
        b = torch.arange(logits.shape[0])
        return logits[b, am.long()], am + row0

    def merge(vals, idxs, stream=None):
        n, nb = vals.shape
        out = torch.empty(nb, dtype=torch.int32)
        for b in range(nb):
            best = max(range(n), key=lambda k: (float(vals[k, b]), -int(idxs[k, b])))
            out[b] = idxs[best, b]
        return out

    rq.rq_logits_from_hidden = logits_from_hidden
    rq.rq_argmax_candidates = candidates
    rq.rq_argmax_merge = merge
    d = rq.dims(r1 - r0, 12, 2, 2, 4)
    logits, pick, _ = rq.rq_sharded_logits(None, None, None, rq.U16, d, r0)
    q.put((rank, logits.shape[1] == r1 - r0, pick.tolist(),
           full.argmax(dim=1).tolist()))
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_logits_glue_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_sharded_call_worker, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, own_rows, pick, want in res:
        assert own_rows and pick == want
