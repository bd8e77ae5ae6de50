"""The bench's multi-rank host logic on CPU: two gloo ranks (spawned
processes) get distinct users, agree on the slowest rank's time, and report
whole-job throughput over all ranks' work."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import bench
import synth


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 5.0 * rank                        # rank 1 is the slow one
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        batch = synth.workload_attention("layer_bf16", seed=bench.rank_seed(rank))
        out[rank] = (got, int(batch.total_tokens), float(batch.q.float().sum()))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_share_the_max_and_draw_distinct_users():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(worker, args=(world, free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][2] != res[1][2]                       # different users on each rank


def test_whole_job_counts_every_rank():
    v1, t1 = bench.whole_job(2e12, 1e6, 1, 10.0)
    v2, t2 = bench.whole_job(2e12, 1e6, 2, 10.0)
    assert np.isclose(v1, 200.0) and np.isclose(v2, 2 * v1) and np.isclose(t2, 2 * t1)


def test_rank_seeds():
    assert bench.rank_seed(0) is None
    assert len({bench.rank_seed(r) for r in range(8)}) == 8


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def test_peak_follows_the_clock_the_region_ran_at():
    """The burst bf16 peak applies whenever the median SM clock held within 5%
    of its maximum, power-cap flags or not; a region the cap slowed takes the
    sustained peak; both fractions are reported by tensor_roofline."""
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    hot = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped_hot = {"sm_mhz": 1942.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    slowed = {"sm_mhz": 1342.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.pick_bf16_peak(peaks, hot)[0] == 1600.0
    assert bench.pick_bf16_peak(peaks, capped_hot)[0] == 1600.0
    assert "sw_power_cap seen" in bench.pick_bf16_peak(peaks, capped_hot)[1]
    assert bench.pick_bf16_peak(peaks, slowed)[0] == 1400.0
    assert bench.pick_bf16_peak(peaks, None)[0] == 1600.0
