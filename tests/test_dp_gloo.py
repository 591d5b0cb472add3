"""The data-parallel host logic with two gloo ranks on CPU: rank environment,
per-rank shard seeds, the max-over-ranks reduction of the step time, the
whole-job throughput, and that every rank's shard is computed independently
(the fp64 oracle on each rank's shard equals the same shard computed alone)."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from chunkwise_linear_rnn_gla_b200 import dp
from chunkwise_linear_rnn_gla_b200.inputs import make_inputs, to_f64_numpy

import oracle

WORLD = 2
STEP_MS = [3.0, 5.0]  # per-rank device times fed to the reduction
UNITS = 1000.0         # tokens per rank and step


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(rank):
    inp = make_inputs(1, 2, 40, 8, 8, "f32", seed=dp.shard_seed(0, rank), h0=True, with_grad=False)
    f = {k: to_f64_numpy(v) for k, v in inp.items() if v is not None}
    o, hT = oracle.fwd(f["q"], f["k"], f["v"], f["log_a"], f["h0"])
    return o, hT


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD),
                      LOCAL_RANK=str(rank))
    try:
        dist.init_process_group("gloo", init_method="env://", timeout=timedelta(seconds=60))
        env = dp.rank_env()
        m = dp.max_over_ranks(STEP_MS[env.rank])
        thr = dp.job_throughput(UNITS, env.world, m)
        o, hT = _shard(env.rank)
        got = [None] * env.world
        dist.all_gather_object(got, (env.rank, o, hT))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, env.world, m, thr, got))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e), None, None))


def test_two_rank_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda r: r[0])
    for rank, world, m, thr, got in res:
        assert world == WORLD, (rank, m)
        assert m == max(STEP_MS)
        assert thr == pytest.approx(UNITS * WORLD / (max(STEP_MS) / 1e3))
        for r, o, hT in got:
            o_ref, hT_ref = _shard(r)  # the same shard computed alone, in this process
            np.testing.assert_array_equal(o, o_ref)
            np.testing.assert_array_equal(hT, hT_ref)
    # different ranks see different shards
    o0, o1 = res[0][4][0][1], res[0][4][1][1]
    assert not np.array_equal(o0, o1)


def test_rank_env_and_seeds():
    assert dp.rank_env({}) == dp.RankEnv(0, 1, 0)
    assert dp.rank_env({"RANK": "1", "WORLD_SIZE": "4", "LOCAL_RANK": "1"}) == dp.RankEnv(1, 4, 1)
    with pytest.raises(ValueError):
        dp.rank_env({"RANK": "4", "WORLD_SIZE": "4"})
    seeds = {dp.shard_seed(7, r) for r in range(8)}
    assert len(seeds) == 8
    assert dp.global_batch(4, 8) == 32
    assert dp.max_over_ranks(2.5) == 2.5  # no process group: the local value
    with pytest.raises(ValueError):
        dp.job_throughput(1.0, 1, 0.0)
