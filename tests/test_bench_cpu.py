"""bench.py on the host: the reference arm (the fp64 oracle timed on the host
cores) prints one JSON line with the keys the driver reads, ranks other than 0
stay silent, and both arms name the same workload.  No GPU is needed."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from rnn_joint_network_02_b200 import synth  # noqa: E402


def _run(*argv, env_extra=None, timeout=600):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv], capture_output=True, text=True,
                          env=env, cwd=ROOT, timeout=timeout)


def test_reference_arm_prints_one_complete_line():
    r = _run("--impl", "reference", "--workload", "short", "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True and line["unit"] == "cells/s"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == "short" and line["config"]["mode"] == "untiled"


def test_reference_arm_other_ranks_do_no_work():
    r = _run("--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
             env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("gpus", [1, 4])
def test_both_arms_name_the_same_config(gpus):
    """The reference line's config is built by the same function as ours, for
    the same number of GPUs, with the headline (first measured) mode."""
    args = bench.parse(["--gpus", str(gpus)])
    batch = synth.workload(args.workload)
    cfg = bench.config_of(batch, args, gpus)
    assert cfg["parallelism"] == f"dp{gpus}" and cfg["global_batch"] == batch.dims["B"] * gpus
    assert cfg["mode"] == bench.modes_of(args)[0] == "untiled"


def test_stage_work_is_the_algorithmic_work():
    """2HV flops per valid cell for each joint contraction; 4V bytes per cell
    for the untiled dz pass (bf16 z read, bf16 dz written)."""
    batch = synth.workload("medium")
    d, cells = batch.dims, batch.valid_cells()
    H, V = d["H"], d["V"]
    for stage in ("joint_fwd", "bwd_dWo", "bwd_dh"):
        assert bench.stage_work(batch, stage, "untiled") == ("tensor", 2.0 * H * V * cells)
    assert bench.stage_work(batch, "joint_bwd_dz", "untiled") == ("hbm", 4.0 * V * cells)
    assert bench.stage_work(batch, "joint_bwd_dz", "tiled") == ("tensor", 2.0 * H * V * cells)
    kind, work = bench.stage_work(batch, "joint_fwd", "untiled", n_dur=5)
    assert work == 2.0 * H * (V + 5) * cells
