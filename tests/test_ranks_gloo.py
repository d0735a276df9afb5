"""The multi-rank host logic of bench.py on CPU with two gloo ranks: each rank
draws different sequences (the path shards by sequence, no data-path
collective), the timing is the maximum over ranks, and the throughput counts
the tokens of every rank over that time."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import synth
        prompt = synth.prompt_ids(synth.TINY, 2, 16, seed=bench.rank_prompt_seed(rank))
        ms = 100.0 + 50.0 * rank                       # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world)
        value = bench.whole_job_tokens_per_s(world, 2, 64, 3, ms_max)
        out[rank] = (prompt.tolist(), ms_max, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_sequences_and_reduce_time():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    p0, m0, v0 = out[0]
    p1, m1, v1 = out[1]
    assert not np.array_equal(np.array(p0), np.array(p1))   # different sequences per rank
    assert m0 == m1 == 150.0                                  # the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 2 * 64 * 3 / 0.150)  # every rank's tokens
