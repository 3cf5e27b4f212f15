"""Multi-process host logic of bench.py with two gloo ranks on CPU: each rank
draws its own batch, the job's time is the slowest rank's, and the whole-job
throughput counts every rank's units (weak scaling, no data exchange)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 1.0 + rank  # rank 1 is the slow one
        t = bench.max_over_ranks(ms, dist)
        value, tmax = bench.aggregate([t] * world, 100.0)
        # the end-to-end record: rank 1 is the slow one again
        rec = {"value": 0.0, "unit": "TFLOP/s", "ms_per_step": 0.0, "ms_raw": 4.0 + rank,
               "h2d_bytes_per_step": 10, "d2h_bytes_per_step": 3, "pipelined": "x"}
        e2e = bench.whole_job_e2e(rec, 1e12, world, dist)
        q.put((rank, t, value, tmax, bench.shard_seed(0, rank), e2e))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_gloo_max_over_ranks_and_weak_aggregate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value, tmax, seed, e2e in res:
        assert t == 2.0 and tmax == 2.0
        assert abs(value - world * 100.0 / 2e-3) < 1e-6
        # whole job: every rank's work over the slowest rank's step (5 ms)
        assert e2e["ms_per_step"] == 5.0 and abs(e2e["value"] - world * 1.0 / 5e-3) < 1e-9
        assert e2e["h2d_bytes_per_step"] == 10 * world and e2e["d2h_bytes_per_step"] == 3 * world
        assert "ms_raw" not in e2e
    assert len({r[4] for r in res}) == world  # each rank its own batch


def test_single_rank_needs_no_collective():
    import bench

    assert bench.max_over_ranks(3.5, None) == 3.5
    v, t = bench.aggregate([2.0], 10.0)
    assert t == 2.0 and abs(v - 5000.0) < 1e-9


def test_single_rank_e2e_record():
    import bench

    rec = {"value": 0.0, "unit": "TFLOP/s", "ms_per_step": 4.3624, "ms_raw": 4.36237,
           "h2d_bytes_per_step": 201326592, "d2h_bytes_per_step": 134217728, "pipelined": "x"}
    e2e = bench.whole_job_e2e(rec, 824.7e9, 1, None)
    assert e2e["ms_per_step"] == 4.3624 and abs(e2e["value"] - round(824.7e9 / 4.36237e-3 / 1e12, 3)) < 1e-9
    assert e2e["h2d_bytes_per_step"] == 201326592 and e2e["d2h_bytes_per_step"] == 134217728
    assert "ms_raw" not in e2e and e2e["unit"] == "TFLOP/s"


def test_launches_per_step():
    import bench
    from differential_attention_swa_b200.inputs import WORKLOADS

    # one persistent prefill kernel; the backward's row statistics, stride
    # pass (local + strided only), dK/dV and dQ kernels
    assert bench.launches_per_step(WORKLOADS["mistral_swa_prefill"]) == 1
    assert bench.launches_per_step(WORKLOADS["local_strided_prefill"]) == 1
    assert bench.launches_per_step(WORKLOADS["mistral_swa_backward"]) == 3
    assert bench.launches_per_step(WORKLOADS["local_strided_backward"]) == 4


def test_profiled_traffic_tracks_sources(tmp_path, monkeypatch):
    import bench

    # a summary counts only while the kernel's sources hash to what it records
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash(["k.cu"])
    (tmp_path / "profiles" / "k.md").write_text(f"dram_bytes_per_launch: 12345\nsource_sha256_16: {h}\n")
    assert bench.profiled_traffic("k.md", ["k.cu"]) == 12345
    src.write_text("kernel v2")
    assert bench.profiled_traffic("k.md", ["k.cu"]) is None
    assert bench.profiled_traffic("missing.md", ["k.cu"]) is None
    for name, (summary, sources) in bench.PROFILES.items():  # every listed summary exists
        assert os.path.exists(os.path.join(os.path.dirname(os.path.dirname(__file__)), "profiles", summary)), name


def test_reference_arm_line(monkeypatch):
    import bench

    # the oracle arm prints the GPU arm's metric and config (one bounded step)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    d = bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "3"]))
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["higher_is_better"] is True and d["value"] > 0
    assert d["config"] == {"workload": "mistral_swa_prefill", "B": 2, "Hq": 32, "Hkv": 8, "N": 8192, "d": 128,
                           "W": 4096, "S": 0, "parallelism": "dp1 (independent batches)",
                           "l2": "flushed between steps"}
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
