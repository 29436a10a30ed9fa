"""The N > 1 path of the benchmark on CPU: two gloo ranks (world size 2) run the host-side logic that the
GPU ranks run over NCCL — each rank draws its own seeded inputs, the per-rank timings are reduced to
the max over ranks, and the whole-job rate counts every rank's units over the slowest rank's time.
There is no data-path collective: each rank's work is independent (replicas over sequences)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from mla_latent_kv_31_b200 import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank inputs: the bench seeds each rank's cache and hidden states with its rank
        cache = synth.latent_cache(synth.TINY, 8, seed=rank)
        # per-rank timings (ms): rank 1 is the slow one for the first, rank 0 for the second
        ms = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 3.0])
        out[rank] = (float(cache.sum()), ms)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_to_the_max_and_draw_their_own_inputs():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    # both ranks see the same reduced timings: the max over ranks, element by element
    assert res[0][1] == res[1][1] == [2.0, 5.0, 3.0]
    # different seeds, different inputs (independent replicas)
    assert res[0][0] != res[1][0]


def test_max_over_ranks_is_identity_on_one_process():
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_whole_job_rate_counts_all_ranks_units_over_the_slowest_time(world):
    # weak scaling: each rank processes 75.5 MB of cache per step; the slowest rank takes 0.2 ms
    rate = bench.whole_job_rate(world, 75_497_472, 0.2e-3)
    assert rate == pytest.approx(world * 75_497_472 / 0.2e-3)
    assert np.isclose(rate / world, 75_497_472 / 0.2e-3)
