"""Host-side parts of bench.py on CPU (gloo ranks, no GPU): the timed region
is the slowest rank's, every rank receives it, the whole-job value counts every rank's
steps, the reference arm runs on rank 0 only, and the oracle baselines run."""
import argparse
import os
import socket

import numpy as np
import pytest
import torch

import bench


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, tmpdir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 2.5 + 1.5 * rank  # this rank's time of the timed region
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        np.save(os.path.join(tmpdir, f"ms{rank}.npy"), np.array([mine, got]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_every_rank_gets_the_slowest_time(world, tmp_path):
    import torch.multiprocessing as mp
    mp.spawn(_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [np.load(tmp_path / f"ms{r}.npy") for r in range(world)]
    slowest = max(r[0] for r in res)
    assert all(r[1] == slowest for r in res)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(1.25, 1, torch.device("cpu")) == 1.25


def test_whole_job_rate_counts_every_rank():
    # 3 ranks x 10 steps x 2e12 flops in 40 ms -> 1500 TFLOP/s for the job, 500 per rank
    assert bench.whole_job_rate(3, 2e12, 10, 40.0) == pytest.approx(1500.0)
    assert bench.whole_job_rate(1, 2e12, 10, 40.0) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    args = argparse.Namespace(steps=1, warmup=0, gpus=2, workload="crop768", op="attention")
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_gate_cpu_baseline_times_the_oracle():
    line = bench.gate_cpu_baseline(target_s=0.2)
    assert line["kind"] == "oracle" and line["unit"] == "GB/s"
    assert line["value"] > 0 and line["cores"] >= 1 and line["seconds"] > 0


@pytest.mark.parametrize("B,N,H", [(1, 768, 4), (1, 384, 4), (2, 256, 4), (2, 128, 4), (1, 64, 2), (2, 1024, 4)])
def test_launch_count_follows_the_library_chunk_rule(B, N, H):
    """The bench's per-step kernel count includes the dBias reduce exactly when the
    library's workspace holds row-chunk partials (its size beyond the rows-only part)."""
    from triangle_attention_biomolecular_b200 import _binding as Bd
    has_partials = Bd.tri_attn_bwd_workspace_bytes(B, N, H, 32) > Bd.tri_attn_bwd_rows_workspace_bytes(B, N, N, H, 32)
    assert bench.attn_launches_per_step(B, N, H) == 5 + int(has_partials)


def test_l2_note_follows_the_input_size():
    assert bench.l2_note(604_000_000).startswith("inputs (604 MB) larger than the 126 MB L2")
    assert "fit in the 126 MB L2" in bench.l2_note(50_000_000)


def test_json_line_carries_every_contract_key(monkeypatch, capsys):
    """The line's assembly from a measured step (the GPU part replaced by fixed
    numbers): every key of the output contract is present, the whole-job value
    follows from the step time, and the roofline fraction is achieved / peak."""
    import json
    import sys
    ms_step = 2.6
    fake = {"ms": 20 * ms_step,
            "kern_ms": {"fwd": 0.78, "bwd_prep": 0.10, "bwd_main": 1.14, "bwd_dbias": 0.61},
            "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5},
            "e2e": {"value": 55.0, "unit": "TFLOP/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1},
            "shape": (1, 768, 4, 32), "step_stats": {"median": ms_step}, "lengths": [768],
            "memory": {"peak_allocated_bytes": 1}, "mask": "zeros", "bias_std": 2.0}
    monkeypatch.setattr(bench, "run_ours", lambda *a: fake)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "20", "--warmup", "5", "--no-cpu-baseline"])
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    bench.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == 20 and line["warmup"] == 5
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert abs(line["ms_per_step"] - ms_step) < 1e-9
    flops = 14.0 * 4 * 768 ** 3 * 32
    assert abs(line["value"] - flops / (ms_step * 1e-3) / 1e12) < 1e-2
    r = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in r, key
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    assert line["config"]["workload"].startswith("crop768")
    assert line["gpu_launches"] == 5 * 20


def test_reference_arm_line_on_rank_zero(capsys):
    """The reference arm (the FP64 oracle on host cores) prints one line with the
    same metric and unit as ours, marked as the reference, with its CPU baseline
    and an end-to-end entry that moves no device bytes."""
    import json
    args = argparse.Namespace(steps=1, warmup=0, gpus=1, workload="crop768", op="attention")
    bench.run_reference(args, rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["higher_is_better"] is True and line["dtype"] == "f64" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
