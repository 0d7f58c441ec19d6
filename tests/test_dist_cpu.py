"""The multi-rank path of the benchmark on CPU: two gloo ranks exchange the
timing maximum, take distinct replica seeds and compute the aggregate rate."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from rank_key_top_b200 import dist as rdist


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w, _ = rdist.init_from_env("gloo", timeout_s=30)
    rdist.barrier(w)
    t = rdist.max_over_ranks(1.5 + r, w, device="cpu")
    seed = rdist.replica_seed(1004, r)
    seeds = [None] * w
    import torch.distributed as dist
    dist.all_gather_object(seeds, seed)
    out[r] = (r, w, t, tuple(seeds), rdist.aggregate_rate(100, w, t))
    rdist.finish(w)


@pytest.mark.parametrize("world", [2])
def test_two_ranks(world):
    port = free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        rank, w, t, seeds, rate = res[r]
        assert (rank, w) == (r, world)
        assert t == 2.5                        # the slowest rank's time, on every rank
        assert len(set(seeds)) == world        # replicas decode distinct batches
        assert rate == pytest.approx(world * 100 / 2.5)


def test_single_process_defaults(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert rdist.init_from_env("gloo")[1] == 1
    assert rdist.max_over_ranks(3.0, 1) == 3.0
    assert rdist.aggregate_rate(10, 1, 2.0) == 5.0


def leaving_worker(rank, world, port, out):
    """Rank 1 joins the group, then leaves between steps (exits without its
    next collective); rank 0's next collective must end with an error, not
    wait for ever."""
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w, _ = rdist.init_from_env("gloo", timeout_s=10)
    rdist.barrier(w)
    if r == 1:
        out[r] = "left"
        os._exit(0)
    try:
        rdist.max_over_ranks(1.0, w, device="cpu")
        out[r] = "no error"
    except Exception as e:  # the process group reports the missing peer
        out[r] = "error: " + type(e).__name__
    os._exit(0)


def test_rank_that_leaves_ends_the_others_collective():
    port = free_port()
    with mp.Manager() as m:
        out = m.dict()
        ctx = mp.spawn(leaving_worker, args=(2, port, out), nprocs=2, join=False)
        for p in ctx.processes:
            p.join(timeout=90)
        alive = [p.is_alive() for p in ctx.processes]
        for p in ctx.processes:
            if p.is_alive():
                p.kill()
        res = dict(out)
    assert not any(alive), "a rank was still waiting"
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]
