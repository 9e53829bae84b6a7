"""The multi-GPU path of bench.py, on CPU with two gloo ranks.

The KDA core shards by (sequence, head): every rank runs its own batch with no collective on the
data path, and the benchmark's only cross-rank steps are a barrier and a MAX reduction of the
timed region.  These tests run those steps with world size 2 on the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from linear_attention_serving_rule_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = bench.dist_setup(world, backend="gloo")
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    # each rank "times" a different amount; everyone must report the slowest
    mx = bench.max_over_ranks(10.0 + rank * 5.0, w, torch.device("cpu"))
    # each rank draws its own batch
    seed = bench.rank_seed(synth.WORKLOADS["prefill_bf16"]["seed"], rank)
    inp = synth.make_prefill(H=2, dk=16, dv=16, dtype="f32", seed=seed, B=1, T=8)
    fp = float(inp.q.sum())
    fps = [None] * w
    dist.all_gather_object(fps, fp)
    rate = bench.whole_job_rate(w, 4 * 4096, 20, mx)
    dist.destroy_process_group()
    q.put((rank, mx, fps, rate))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks(world):
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
    res.sort()
    for rank, mx, fps, rate in res:
        assert mx == 15.0                      # MAX over ranks
        assert fps[0] != fps[1]                # different batches per rank
        assert rate == pytest.approx(world * 4 * 4096 * 20 / 0.015)


def test_single_process_defaults():
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.rank_seed(1, 0) == 1 and bench.rank_seed(1, 3) == 3001
