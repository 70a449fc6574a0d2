"""The multi-rank plumbing on the CPU: two gloo processes run the same
helpers bench.py runs over NCCL (process group from the environment,
barrier, max over ranks, per-rank batches, whole-job rate), and a rank
that never arrives ends the others' wait with an error instead of a hang."""

import os
import socket
import time

import pytest
import torch.multiprocessing as mp

from exact_attention_147_b200 import ranks


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))


def _worker(rank, world, port, out):
    _env(rank, world, port)
    r, w, local = ranks.init("gloo", timeout_s=30.0)
    assert (r, w, local) == (rank, world, rank)
    # each rank "takes" a different time; every rank must see the maximum
    mx = ranks.max_over_ranks(0.5 + rank, w, "cpu")
    ranks.barrier(w)
    out.put((rank, mx, ranks.batch_seed(1000, rank)))
    ranks.finalize(w)


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r for r, _, _ in res) == [0, 1]
    assert all(mx == 1.5 for _, mx, _ in res)
    seeds = {s for _, _, s in res}
    assert len(seeds) == world          # every rank draws its own batch


def _late_worker(rank, world, port, out):
    _env(rank, world, port)
    if rank == 1:
        return                          # never joins the group
    t0 = time.time()
    try:
        ranks.init("gloo", timeout_s=5.0)
        ranks.barrier(world)
        out.put(("no error", time.time() - t0))
    except Exception as e:              # the missing rank surfaces as an error
        out.put((type(e).__name__, time.time() - t0))


def test_missing_rank_ends_in_an_error_not_a_hang():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_late_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    what, took = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert what != "no error"
    assert took < 60


def test_single_process_needs_no_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert ranks.rank_env() == (0, 1, 0)
    assert ranks.init("gloo") == (0, 1, 0)
    assert ranks.max_over_ranks(2.5, 1) == 2.5
    ranks.barrier(1)
    ranks.finalize(1)


@pytest.mark.parametrize("world", [1, 2, 8])
def test_whole_job_rate_is_weak_scaling(world):
    # each rank processes 10 units; the slowest rank took 2 s
    assert ranks.whole_job_rate(10.0, world, 2.0) == 5.0 * world
