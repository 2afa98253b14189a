"""Multi-rank host logic on CPU with the gloo backend (world size 2): the
unit sharding covers every (layer, batch, head) unit exactly once, the timed
region's max-over-ranks is the slowest rank's time, and a rank that raises
ends the job with an error instead of hanging the others."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from channel_pruned_decode_b200 import dist as sd


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("n", [0, 1, 7, 8, 256, 1001])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_partitions_units(n, world):
    seen = []
    sizes = []
    for r in range(world):
        rg = sd.shard(n, r, world)
        seen.extend(rg)
        sizes.append(len(rg))
    assert seen == list(range(n))
    assert max(sizes) - min(sizes) <= 1


def test_shard_rejects_bad_args():
    with pytest.raises(ValueError):
        sd.shard(4, 2, 2)
    with pytest.raises(ValueError):
        sd.shard(-1, 0, 1)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    try:
        r, w = sd.init("gloo", timeout_s=30)
        units = sd.shard(256, r, w)
        sd.barrier()
        t = 1.0 + r  # stand-in for this rank's device time
        q.put((r, list(units), sd.max_over_ranks(t), sd.sum_over_ranks(len(units))))
        sd.finalize()
    except Exception as e:  # pragma: no cover - surfaced through the queue
        q.put((rank, "error", repr(e), None))


def test_gloo_two_ranks_max_and_cover():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    out.sort()
    assert all(o[1] != "error" for o in out), out
    assert out[0][1] + out[1][1] == list(range(256))
    assert out[0][2] == out[1][2] == 2.0
    assert out[0][3] == out[1][3] == 256


def _failing_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    try:
        sd.init("gloo", timeout_s=5)
    except Exception as e:
        # a peer too slow to reach the rendezvous on a loaded host ends the
        # same way: an error on this rank within the timeout, not a hang
        if rank == 1:
            raise SystemExit(3)
        q.put((rank, "init " + type(e).__name__))
        return
    if rank == 1:
        raise SystemExit(3)  # leaves between steps, nothing in flight
    try:
        sd.barrier()
        q.put((rank, "no error"))
    except Exception as e:
        q.put((rank, type(e).__name__))


def test_gloo_missing_rank_fails_fast():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    rank, what = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert rank == 0 and what != "no error"
    assert procs[1].exitcode == 3
