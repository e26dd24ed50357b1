"""The multi-GPU host logic on CPU: two gloo ranks (one process each) shard the
batch by seed, meet at barriers, and reduce the timed region with a max, so
the whole-job throughput is all ranks' units over the slowest rank's time."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from linear_rnn_sequence_wkv7_b200 import inputs
from linear_rnn_sequence_wkv7_b200.dist import Dist, aggregate_throughput, shard_seed


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    d = Dist("gloo").init(timeout_s=60)
    try:
        d.barrier()
        seed = shard_seed(1, d.rank)
        shard = inputs.gen_sequence(1, 8, 2, 64, seed=seed, dtype="bf16")["r"]
        elapsed = 0.5 + 0.25 * d.rank          # stand-in for a device-timed region
        slowest = d.max(elapsed)
        d.barrier()
        out.put((d.rank, seed, int(shard.view(np.uint16).astype(np.int64).sum()), slowest,
                 aggregate_throughput(1000.0, slowest, d.world)))
    finally:
        d.close()


def test_two_gloo_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, c0, m0, v0), (r1, s1, c1, m1, v1) = results
    assert (r0, r1) == (0, 1)
    assert s0 != s1 and c0 != c1                 # each rank draws its own batch shard
    assert m0 == m1 == 0.75                      # max over ranks, seen by every rank
    assert v0 == v1 == 1000.0 * 2 / 0.75         # units of all ranks over the slowest time


def test_single_process_is_identity():
    d = Dist("gloo")
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    if d.world == 1:
        d.init()
        assert d.max(3.5) == 3.5
        d.barrier()
        d.close()


def _failing_rank_main(rank, world, port, out):
    """Rank 1 fails between steps (an exception before the timing reduction);
    rank 0 must learn of it from its own collective, as an error, not a hang."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    d = Dist("gloo").init(timeout_s=5)
    d.barrier()
    if rank == 1:
        raise RuntimeError("rank 1 fails between steps")
    try:
        d.max(1.0)
        out.put(("no error", ""))
    except Exception as e:          # a closed connection or the process-group timeout
        out.put(("error", type(e).__name__))
    out.close()
    out.join_thread()
    os._exit(0)                     # no teardown collective with a dead peer


def test_a_failed_rank_ends_the_others_collective_with_an_error():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_failing_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    status, _ = out.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert status == "error"
    assert procs[0].exitcode == 0
    assert procs[1].exitcode != 0
