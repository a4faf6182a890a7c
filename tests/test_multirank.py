"""Multi-rank host logic of bench.py on CPU with gloo (world size 2).

The path partitions into independent (b, h) problems, so N ranks run N
independent batches with no data-path collective; what crosses ranks is the
timing barrier and the max-over-ranks reduction.  These tests exercise that
logic and the failure mode of a rank that leaves early.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=30):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _worker_max(rank, world, port, q):
    import bench
    _init(rank, world, port)
    ms = [3.0, 7.5][rank]
    got = bench.max_over_ranks(ms, world, torch.device("cpu"))
    r, w, lr = bench.dist_env()
    # per-rank shards: same config, distinct seeds -> distinct inputs
    from linear_attention_video_chunk_b200 import inputs
    c = bench.CONFIGS["wan13b"]
    x = inputs.head_array(c["seed"] + 1000 * rank, "q", 0, 0, 16, 8)
    t = torch.from_numpy(x).float()
    others = [torch.zeros_like(t) for _ in range(world)]
    dist.all_gather(others, t)
    tokens = bench.work(c)["tokens"] * world
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, (r, w, lr), not torch.equal(others[0], others[1]), tokens / (got / 1e3)))


def test_max_over_ranks_and_weak_scaling_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_max, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, env, distinct, value in res:
        assert got == 7.5                      # every rank sees the slowest rank's time
        assert env == (rank, world, rank)
        assert distinct                        # the two shards differ
        assert value == pytest.approx(2 * 32760 / 7.5e-3)


def _worker_leaver(rank, world, port, q):
    _init(rank, world, port, timeout_s=5)
    dist.barrier()                             # both ranks joined
    if rank == 1:
        os._exit(0)                            # leaves between steps, nothing in flight
    try:
        dist.barrier()
        q.put("no error")
    except Exception as e:  # noqa: BLE001 - any error means the loss was detected
        q.put("error: " + type(e).__name__)


def test_rank_that_leaves_is_detected_not_hung():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker_leaver, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    msg = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert msg.startswith("error"), msg
