"""bench.py's multi-GPU path on the CPU: replicas timed by the slowest rank.

The step has no exchange, so N GPUs run N independent replicas; the only
collective is the max of the per-rank timings.  Two gloo ranks check that
reduction and the whole-job aggregation, and the reference arm's rank rule
(rank 0 runs and prints, the others exit without work).
"""
import json
import os
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 5.0 - rank, 1.0]
        got = bench.max_over_ranks(local, "cpu")
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(got, f)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks(tmp_path):
    port = 29500 + os.getpid() % 1000
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert json.load(open(tmp_path / f"rank{r}.json")) == [11.0, 5.0, 1.0]


def test_replica_aggregation():
    sys.path.insert(0, ROOT)
    import bench
    # 4 replicas each doing 3e12 flop; the slowest took 2 s -> 6 TFLOP/s whole-job.
    assert bench.replica_throughput(3e12, 4, 2.0) == 6.0
    assert bench.max_over_ranks([1.5, 2.5], "cpu") == [1.5, 2.5]      # single process: identity


def test_reference_arm_rank_rule():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "single_256",
           "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env["RANK"] = "0"
    r = subprocess.run(cmd, capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_peaks_file_read_per_key(tmp_path):
    import bench
    full = tmp_path / "full.json"
    full.write_text('{"hbm_gbs": 6546.6, "bf16_tflops": 1648.7, "bf16_tflops_sustained": 1352.3}')
    peaks, src = bench.load_peaks(str(full))
    assert peaks == {"hbm_gbs": 6546.6, "bf16_tflops": 1648.7, "bf16_tflops_sustained": 1352.3}
    assert set(src.values()) == {"measured"}
    part = tmp_path / "part.json"       # records with a value field; one key missing
    part.write_text('{"hbm_gbs": {"value": 6546.6}, "bf16_tflops": {"median": 1648.7}}')
    peaks, src = bench.load_peaks(str(part))
    assert peaks["hbm_gbs"] == 6546.6 and peaks["bf16_tflops"] == 1648.7
    assert peaks["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert src == {"hbm_gbs": "measured", "bf16_tflops": "measured", "bf16_tflops_sustained": "fallback"}
    bad = tmp_path / "bad.json"
    bad.write_text("not json")
    peaks, src = bench.load_peaks(str(bad))
    assert peaks == bench.FALLBACK_PEAKS and set(src.values()) == {"fallback"}
    peaks, src = bench.load_peaks(str(tmp_path / "absent.json"))
    assert peaks == bench.FALLBACK_PEAKS and set(src.values()) == {"fallback"}
