"""The N > 1 host path on CPU: two gloo ranks (spawned processes, 127.0.0.1).
Streams are partitioned by rank with no data-path exchange; the job time is
the max over ranks; the whole-job rate counts every rank's units. Sharding by
stream is exact: each rank's per-stream results equal the single-process
results for the same global stream ids. A rank that dies before the
collective makes the other rank's collective fail instead of hanging."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch.multiprocessing as mp

from rolling_kv_cache_sa_b200.dist import aggregate_rate, max_over_ranks, rank_stream_ids

B_PER_RANK = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=20))
    return dist


def _rows_for(streams):
    import oracle as O
    from inputgen import spec_for
    from inputgen.workloads import TINY_F32
    w = TINY_F32.with_(B=B_PER_RANK)
    cfg = O.cfg_for(w)
    toks = np.repeat(np.arange(w.Lc), w.H).astype(np.int32)
    heads = np.tile(np.arange(w.H), w.Lc).astype(np.int32)
    return [O.attend_rows(cfg, spec_for(w), s, 2, toks, heads) for s in streams]


def _worker_ok(rank, world, port, q):
    try:
        dist = _init(rank, world, port)
        ids = rank_stream_ids(rank, B_PER_RANK)
        t = max_over_ranks(10.0 + 5.0 * rank)
        rows = _rows_for(ids)
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        dist.barrier()
        dist.destroy_process_group()
        q.put(("ok", rank, ids, t, [r.tolist() for r in rows], gathered))
    except Exception as e:  # reported to the parent
        q.put(("err", rank, repr(e)))


def _worker_dies(rank, world, port, q):
    try:
        dist = _init(rank, world, port)
        if rank == 1:
            os._exit(3)  # leaves between steps: no collective in flight
        try:
            max_over_ranks(1.0)
            q.put(("no-error", rank))
        except Exception as e:
            q.put(("raised", rank, type(e).__name__))
    except Exception as e:
        q.put(("err", rank, repr(e)))


def _spawn(fn, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    return procs, q


def test_two_gloo_ranks_partition_streams_and_reduce_time():
    procs, q = _spawn(_worker_ok, 2)
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    assert all(r[0] == "ok" for r in res), res
    res.sort(key=lambda r: r[1])
    ids0, ids1 = res[0][2], res[1][2]
    assert ids0 == [0, 1] and ids1 == [2, 3]          # disjoint, covering 0..3
    assert res[0][5] == [ids0, ids1] == res[1][5]
    assert res[0][3] == res[1][3] == 15.0              # max over ranks
    # sharding by stream is exact: same rows as one process computing those streams
    single = _rows_for([0, 1, 2, 3])
    for r in res:
        for s, rows in zip(r[2], r[4]):
            np.testing.assert_array_equal(np.asarray(rows), single[s])
    assert aggregate_rate(64, 2, 15.0) == pytest.approx(64 * 2 / 0.015)


def test_dead_rank_fails_the_collective_instead_of_hanging():
    procs, q = _spawn(_worker_dies, 2)
    r = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert r[0] == "raised" and r[1] == 0, r


def test_single_process_helpers():
    assert rank_stream_ids(3, 4) == [12, 13, 14, 15]
    assert max_over_ranks(2.5) == 2.5  # no process group: identity
    with pytest.raises(ValueError):
        aggregate_rate(1, 1, 0.0)
