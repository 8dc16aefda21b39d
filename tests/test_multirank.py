"""The N > 1 host path of bench.py on CPU: two gloo ranks run the same barrier,
max-over-ranks timing and whole-job aggregation that NCCL ranks run on GPUs
(replicas exchange no data, so this is the whole multi-GPU protocol).  The
reference arm under torchrun prints from rank 0 only and other ranks exit 0."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(world, backend="gloo")
    bench.barrier(w)
    local_ms = [1.5, 4.0][r]                      # rank 1 is the slow replica
    ms = bench.dist_max(local_ms, w)
    value = bench.whole_job_tflops(w, 4.0e11, ms)
    bench.barrier(w)
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"world": w, "rank": r, "local": local, "ms": ms, "value": value,
                   "backend": dist.get_backend()}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time(tmp_path):
    port = _free_port()
    mp.start_processes(_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, d in enumerate(res):
        assert d["world"] == 2 and d["rank"] == r and d["local"] == r and d["backend"] == "gloo"
        assert d["ms"] == 4.0                      # max over ranks, seen identically by both
        assert abs(d["value"] - 2 * 4.0e11 / 4.0e-3 / 1e12) < 1e-9


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_max(2.5, 1) == 2.5
    assert bench.whole_job_tflops(1, 1e12, 1.0) == 1000.0


def test_reference_arm_prints_from_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_keeps_the_contract():
    # rank 0 of the reference arm prints one JSON line with the contract's keys (CPU, seconds)
    import json
    env = dict(os.environ)
    for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(key, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-500:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["workload"] == "n8192_causal"
    assert set(line["cpu_baseline"]) >= {"value", "unit", "cores", "kind", "sample"}
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_launch_percentiles():
    sys.path.insert(0, ROOT)
    import bench
    p = bench.launch_percentiles([float(x) for x in range(1, 12)])   # 1..11
    assert p == {"p10": 2.0, "p50": 6.0, "p90": 10.0}
    assert bench.launch_percentiles([0.5]) == {"p10": 0.5, "p50": 0.5, "p90": 0.5}


def test_traffic_is_reported_only_for_the_captured_kernel(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    h = bench.kernel_source_hash()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "ncu_traffic.json").write_text(json.dumps({
        "a": {"kernel_source_sha": h, "dram_bytes_per_launch": 123},
        "b": {"kernel_source_sha": "0" * 16, "dram_bytes_per_launch": 456}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: h)
    assert bench.load_traffic("a") == 123
    assert bench.load_traffic("b") is None          # captured on another kernel source
    assert bench.load_traffic("missing") is None
