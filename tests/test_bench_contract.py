"""bench.py's host side on CPU: the reference arm's JSON line and the L2 statement.

The reference arm times the fp64 oracle on the host cores in the same metric as the GPU
arm, so it runs here; the GPU arm's line is checked by the GPU runs themselves.
"""
import json
import os
import subprocess
import sys

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps",
           "1", "--warmup", "3", "--cpu-seconds", "1", "--workload", "layer-4k"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["config"]["workload"] == "layer-4k"
    assert line["config"]["T"] == 4096 and line["config"]["L"] == 24
    assert line["value"] > 0
    # ms_per_step is the whole step's algorithmic FLOPs at the measured rate
    flops = workloads.forward_flops(**workloads.CONFIGS["layer-4k"]) * (1 + bench.BWD_FLOP_FACTOR)
    assert abs(line["ms_per_step"] - flops / (line["value"] * 1e12) * 1e3) <= \
        1e-3 * line["ms_per_step"] + 1e-3
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1
    # the backward shares the sample's tokens out among the host's threads
    assert cpu["cores"] == min(cpu["sample_tokens"], cpu["host_threads"])
    assert cpu["value_1_thread"] > 0 and cpu["sample_1_thread_tokens"] >= 1
    assert cpu["unit"] == "TFLOP/s" and cpu["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == "TFLOP/s"
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_l2_statement_follows_the_workload_size():
    assert bench.l2_note(workloads.CONFIGS["long-64k"]) == "inputs larger than L2 (no flush)"
    assert bench.l2_note(workloads.CONFIGS["fwd-bwd-16k"]) == "inputs larger than L2 (no flush)"
    note = bench.l2_note(workloads.CONFIGS["tiny"])
    assert "fit in L2" in note and "not a headline figure" in note


def test_reference_arm_under_two_ranks_prints_on_rank_zero_only():
    """As under torchrun --nproc-per-node 2: rank 1 exits 0 without work or output,
    rank 0 prints the line for the whole job (n_gpus = 2)."""
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus",
            "2", "--steps", "1", "--warmup", "3", "--cpu-seconds", "1", "--workload", "tiny"]
    outs = {}
    for rank in (1, 0):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT="29533")
        r = subprocess.run(base, cwd=ROOT, env=env, capture_output=True, text=True,
                           timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        outs[rank] = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert outs[1] == []
    assert len(outs[0]) == 1
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def test_clock_summary_reads_nvidia_smi_samples():
    """The clocks object of the bench line: median SM clock under load, the maximum, and
    every throttle reason seen active in any sample."""
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1612, 1965, 950.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1590, 1965, 990.00, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 700.00, 0x0000000000000000, Not Active, Active, Not Active, Not Active",
        "[N/A], [N/A]",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1612.0, "sm_max_mhz": 1965.0, "samples": 3,
                 "reasons": ["hw_thermal_slowdown", "sw_power_cap"]}
    assert bench.ClockSampler(0).summary()["reasons"] == ["unsampled"]
