"""The multi-GPU bench path is N independent replicas (the decode path does
not shard): each rank times its own steps, the job's step time is the max
over ranks, and the job's throughput counts every rank's bytes.  Checked
here with two gloo ranks on the CPU (no GPU)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = 1.0 + 0.5 * rank                       # rank 1 is the slow one
        job_ms = bench.max_over_ranks(ms, world, device="cpu")
        out[rank] = (job_ms, bench.whole_job_gbs(world, 2.78e9, job_ms))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_time_and_whole_job_value():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 1.5            # every rank sees the slowest time
    assert res[0][1] == pytest.approx(2 * 2.78e9 / 1.5e-3 / 1e9)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.whole_job_gbs(1, 1e9, 1.0) == pytest.approx(1000.0)


def test_traffic_record_matches_current_decode_sources():
    """The decode kernel's committed DRAM-traffic ratio applies only while its
    sources hash to the profiled version; the committed record does."""
    import bench
    r = bench.traffic_for("qmv_mma_kernel", "decode-stack-batched")
    assert r is not None and 0.9 < r < 1.1
    assert bench.traffic_for("qmv_mma_kernel", "another-workload") is None
    assert bench.traffic_for("no_such_kernel", "decode-stack-batched") is None
