"""Host-side logic of bench.py, on CPU: the reference (oracle) arm's JSON
line, rank handling under a multi-rank launch, the max-over-ranks timing
reduction over a world-size-2 gloo group, and clock-log parsing."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

REQUIRED = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")


def _run_bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_json_line():
    r = _run_bench({}, "--impl", "reference", "--workload", "single_linear_16x1024x1024",
                   "--decode-workload", "single_linear_16x1024x1024", "--steps", "3", "--warmup", "1")
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in REQUIRED:
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TOPS"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "single_linear_16x1024x1024"
    dec = d["decode"]
    assert dec["value"] > 0 and dec["cpu_baseline"]["kind"] == "oracle" and dec["config"]["T"] == 16


def test_reference_arm_nonzero_rank_exits_silently():
    env = {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}
    r = _run_bench(env, "--impl", "reference", "--workload", "single_linear_16x1024x1024",
                   "--decode-workload", "none", "--steps", "2", "--warmup", "1")
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    bench.barrier(dist)
    # each rank reports its own elapsed time; every rank must see the max
    m = bench.max_over_ranks(dist, 10.0 + rank, "cpu")
    out[rank] = m
    dist.destroy_process_group()


def test_max_over_ranks_world2_gloo():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert dict(out) == {0: 11.0, 1: 11.0}


def test_single_process_helpers_are_identity():
    assert bench.max_over_ranks(None, 3.5, "cpu") == 3.5
    bench.barrier(None)


def test_clock_log_parsing():
    text = ("0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
            "0, 1890, 1965, 950.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n")
    d = bench.parse_clock_csv(text)
    assert d["sm_mhz"] == 1890.0 and d["sm_max_mhz"] == 1965.0 and d["samples"] == 3
    assert d["reasons"] == ["sw_power_cap"]
    assert bench.parse_clock_csv("")["sm_mhz"] is None


def test_workload_registry_covers_every_config():
    cfgs = bench.all_configs()
    assert bench.DEFAULT_WORKLOAD in cfgs
    assert len([n for n in cfgs if n.startswith("b175_sweep_")]) == 96
    for name in ("single_linear_16x1024x1024", "b175_fc1_decode_t1_12288x49152",
                 "b175_fc1_decode_t16_12288x49152", "b175_qkv_prefill_4096x12288x36864"):
        assert name in cfgs


def test_work_counts():
    ops, wbytes = bench.work({"T": 2, "K": 32, "N": 16}, 3)
    assert ops == 2 * 2 * 32 * 16
    assert wbytes == 32 * 16 + 4 * 16 + 2 * 3 * 16


def test_default_workloads_are_the_largest_prefill_and_a_decode_point():
    cfgs = bench.all_configs()
    single_gpu = [c for n, c in wl_configs().items()]
    biggest = max(single_gpu, key=lambda c: 2 * c["T"] * c["K"] * c["N"])
    assert cfgs[bench.DEFAULT_WORKLOAD] == biggest
    d = cfgs[bench.DECODE_WORKLOAD]
    assert d["T"] <= 16 and d["K"] == 12288 and d["N"] == 49152


def wl_configs():
    from int8_quantized_row_b200 import workloads as wl
    return wl.CONFIGS


def test_nvml_clock_summary():
    samples = [(1965.0, 700.0, 0x0), (1800.0, 990.0, 0x4), (1890.0, 950.0, 0x4 | 0x1)]
    d = bench.summarise_clock_samples(samples, 1965.0, "test")
    assert d["sm_mhz"] == 1890.0 and d["sm_max_mhz"] == 1965.0 and d["samples"] == 3
    assert d["reasons"] == ["sw_power_cap"] and d["power_w_max"] == 990.0
    d = bench.summarise_clock_samples([(1500.0, 1.0, 0x8 | 0x40)], 1965.0, "test")
    assert d["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert bench.summarise_clock_samples([], 1965.0, "test")["sm_mhz"] is None


def test_tensor_peak_follows_the_timed_region():
    pk = dict(hbm_gbs=1.0, bf16_tflops=1687.0, bf16_tflops_sustained=1436.0, src="measured")
    burst, src = bench.tensor_peak(pk, 0.03)
    assert burst == 2 * 1687.0 and "burst" in src
    sus, src = bench.tensor_peak(pk, 5.0)
    assert sus == 2 * 1436.0 and "sustained" in src


def test_traffic_is_keyed_on_the_kernel_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    sha = bench.kernel_source_sha("gemm_decode_kernel")
    assert sha != bench.kernel_source_sha("gemm_prefill_pair_kernel")
    rec = {"captures": {"w": {"kernel": "gemm_decode_kernel", "source_sha": sha, "bytes_per_launch": 123}}}
    (tmp_path / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("w", "gemm_decode_kernel") == 123
    assert bench.ncu_traffic("w", "gemm_prefill_pair_kernel") is None
    rec["captures"]["w"]["source_sha"] = "stale"
    (tmp_path / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("w", "gemm_decode_kernel") is None


def test_oracle_thread_count_follows_openmp():
    """`cores` in the CPU baseline is the thread count the oracle's OpenMP loops
    run with: OMP_NUM_THREADS when set (torchrun sets 1 per rank), and every
    core of the process once the reference arm raises it on rank 0."""
    import subprocess
    import sys
    code = ("import bench, oracle; oracle.default(); a = bench.cpu_threads(); bench.use_all_cores(); "
            "print(a, bench.cpu_threads(), bench.host_cores())")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                         check=True).stdout.split()
    before, after, host = map(int, out)
    assert before == 1 and after == host >= 1
