"""Multi-rank host logic of bench.py on CPU (world size 2, gloo): sequence
sharding covers every batch row exactly once, the timed region is reduced as a
max over ranks, and a rank that never joins a collective ends the other rank's
wait with an error instead of a hang (short process-group timeout)."""
import datetime
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=30):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _shard_and_max(rank, world, port, out):
    _init(rank, world, port)
    import bench
    rows = list(bench.shard_rows(10, rank, world))
    gathered = [None] * world
    dist.all_gather_object(gathered, rows)
    m = bench.max_over_ranks(1.5 + rank, world)
    out.put((rank, gathered, m))
    dist.barrier()
    dist.destroy_process_group()


def _missing_peer(rank, world, port, out):
    _init(rank, world, port, timeout_s=3)
    if rank == 1:
        out.put((rank, "left"))  # leaves between steps without joining the collective
        return
    import bench
    try:
        bench.max_over_ranks(1.0, world)
        out.put((rank, "no error"))
    except Exception as e:  # noqa: BLE001
        out.put((rank, "error: " + type(e).__name__))


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return sorted(res, key=lambda x: x[0])


def test_sharding_and_max_over_ranks():
    res = _run(_shard_and_max)
    (_, gathered, m0), (_, _, m1) = res
    flat = [r for part in gathered for r in part]
    assert sorted(flat) == list(range(10)) and len(flat) == 10
    assert [len(p) for p in gathered] == [5, 5]
    assert m0 == m1 == 2.5


def test_shard_rows_uneven():
    sys.path.insert(0, ROOT)
    import bench
    for world in (1, 2, 3, 4, 8):
        parts = [list(bench.shard_rows(13, r, world)) for r in range(world)]
        assert sorted(x for p in parts for x in p) == list(range(13))
        assert max(map(len, parts)) - min(map(len, parts)) <= 1


def test_missing_rank_ends_collective_with_error():
    res = _run(_missing_peer)
    assert res[1][1] == "left"
    assert res[0][1].startswith("error"), res[0]
