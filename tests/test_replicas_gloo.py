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


def test_traffic_record_applies_only_to_the_profiled_sources(tmp_path, monkeypatch):
    """A kernel's DRAM-traffic ratio (profiles/traffic.json) is used only while
    its sources hash to the profiled version and the workload matches."""
    import hashlib
    import json
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    rec = {"k": {"workload": "w", "sources": ["k.cu"],
                 "sources_sha256_16": hashlib.sha256(b"kernel v1").hexdigest()[:16],
                 "dram_bytes_per_algorithmic_byte": 0.99}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("k", "w") == 0.99
    assert bench.traffic_for("k", "other") is None
    assert bench.traffic_for("missing", "w") is None
    src.write_text("kernel v2")                         # the kernel changed since the capture
    assert bench.traffic_for("k", "w") is None
