"""Host-side logic of the multi-GPU bench on CPU: two `gloo` ranks take the
max over ranks of their step times and report whole-job throughput; the
reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 17.25][rank]            # the slower rank sets the step time
        ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        out[rank] = (ms, bench.job_tflops(world, 1e12, ms / 10))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_with_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 17.25
    # 2 replicas x 1e12 flop per step, 1.725 ms per step
    assert res[0][1] == pytest.approx(2 * 1e12 / 1.725e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.job_tflops(1, 2e12, 2.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun, a rank other than 0 of `--impl reference` exits 0
    without work or output."""
    import subprocess
    import sys
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_json_line():
    """`--impl reference` (the oracle on the host cores, in the GPU arm's
    two-level configuration) prints one JSON line with the contract's keys."""
    import json
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                        "--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "layer"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["config"]["scales"].startswith("E4M3")          # the GPU arm's default scales
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["quantize_GBps"] > 0 and line["cpu_baseline"]["gemm_GFLOPs"] > 0
    assert line["config"]["M"] == 8192 and line["config"]["N"] == 8192


def test_oracle_step_model_units():
    """The oracle's whole-step figure: elements / rate + flops / rate, in the
    GPU arm's unit; a doubled GEMM rate can at most halve the step time."""
    from fp4_quantized_gemms_b200 import workloads as wl
    s = wl.LARGE
    a = bench.oracle_step_figures(s, True, 1e8, 1e10)
    elems = 2 * (s.M * s.K + s.N * s.K + s.M * s.N)
    flops = 6 * s.M * s.N * s.K
    assert a["step_s"] == pytest.approx(elems / 1e8 + flops / 1e10)
    assert a["value"] == pytest.approx(flops / a["step_s"] / 1e12)
    assert a["quantize_GBps"] == pytest.approx(1e8 * (2.5 + 1 / 16) / 1e9)
    b = bench.oracle_step_figures(s, True, 1e8, 2e10)
    assert a["step_s"] / 2 < b["step_s"] < a["step_s"]
