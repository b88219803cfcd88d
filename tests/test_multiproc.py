"""The N > 1 host path on CPU: two gloo ranks (one process each), batch sharding and the
max-over-ranks timing reduction used by the benchmark."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rank_quantized_kv_decode_b200 import dist as D


def test_rank_batch_covers_every_sequence_once():
    for gb in [1, 7, 8, 33]:
        for world in [1, 2, 3, 8]:
            seen = []
            for r in range(world):
                s, n = D.rank_batch(gb, r, world)
                seen.extend(range(s, s + n))
            assert seen == list(range(gb))
    with pytest.raises(ValueError):
        D.rank_batch(8, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # each rank measured a different time; every rank must see the slowest one
        seconds = [0.25, 0.75][rank]
        mx = D.max_over_ranks(seconds)
        start, count = D.rank_batch(16, rank, world)
        rate = D.aggregate_rate(count * 4096, world, mx)
        # the data path needs no collective: each rank's shard is disjoint and complete
        got = torch.zeros(16, dtype=torch.int64)
        got[start:start + count] = 1
        dist.all_reduce(got)
        q.put((rank, mx, rate, got.tolist()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, rate, got in res:
        assert mx == 0.75
        assert rate == pytest.approx(8 * 4096 * 2 / 0.75)
        assert got == [1] * 16


def _leaving_worker(rank, world, port, q):
    """Rank 1 leaves between steps (it raises before the timing reduction, with nothing in
    flight); rank 0 must learn of it from its next collective, as an error, not a hang."""
    import time
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=5))
    D.max_over_ranks(1.0)  # one step that both ranks complete
    if rank == 1:
        q.put((rank, "left", 0.0))
        raise SystemExit(3)
    t0 = time.monotonic()
    try:
        D.max_over_ranks(2.0)
        q.put((rank, "no error", time.monotonic() - t0))
    except Exception as e:  # noqa: BLE001 -- the backend's error type is not part of its API
        q.put((rank, "error: " + type(e).__name__, time.monotonic() - t0))


def test_a_rank_that_leaves_ends_the_others_next_collective_with_an_error():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_leaving_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (what, dt)) for r, what, dt in [q.get(timeout=120) for _ in range(world)])
    for p in procs:
        p.join(timeout=60)
    assert procs[1].exitcode == 3
    what, dt = res[0]
    assert what.startswith("error"), what
    assert dt < 30.0  # bounded by the process group's 5 s timeout, not a hang
