#!/usr/bin/env python
"""Benchmark of one fused RNN-T joint + transducer-loss forward+backward call
per batch (lattice-vocab cells/s = B*T*(U+1)*V / step time, and peak GB).

    python bench.py [--gpus N --steps K --warmup W] [--workload medium] [--mode tiled|untiled]
    python bench.py --impl reference ...      # the fp64 CPU oracle on a bounded sample

A step is one frnnt_fwd_bwd call over one synthetic batch (all steps of the
path: projections, forward joint, lattice DP, backward joint, projection
backward).  With N > 1 (torchrun, one process per GPU) every rank runs its
own batch of the same shape (weak scaling) and the step time is the max over
ranks.  Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rnn_joint_network_02_b200 import dist as rdist  # noqa: E402
from rnn_joint_network_02_b200 import frnnt, synth  # noqa: E402

METRIC = "RNN-T joint+loss fwd+bwd lattice-vocab cells/sec (B·T·(U+1)·V) and peak GB"
UNIT = "cells/s"
L2_BYTES = 126 * 1024 * 1024


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="medium", choices=list(synth.WORKLOADS))
    p.add_argument("--mode", default="both", choices=["both", "tiled", "untiled"],
                   help="both: untiled is the headline value, tiled is reported alongside")
    p.add_argument("--path", default="auto", choices=["auto", "simt"])
    p.add_argument("--chunk-cells", type=int, default=0)
    p.add_argument("--loss", default="marginal", choices=["marginal", "viterbi", "tdt"],
                   help="training criterion: every alignment (default), the best one, or the token-and-duration "
                        "transducer (durations 0..4 frames, a duration head beside the label head)")
    p.add_argument("--prune", type=int, default=0,
                   help="pruned lattice: S label positions per frame on a band along the diagonal (0: whole lattice)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args(argv)


# DRAM bytes (read + write) per launch of a stage's kernel, from one ncu
# capture of that kernel in the bench's own launch configuration (the file
# under profiles/ gives the command), keyed by (workload, mode, stage, loss).
# An entry is removed whenever its kernel changes, so the roofline's traffic is
# null rather than stale.
MEASURED_TRAFFIC = {
    ("medium", "untiled", "bwd_dWo", "marginal"): (1.204969e9 + 0.008939e9,
                                                   "profiles/ncu_gemm2_backward_medium_untiled.md"),
    ("medium", "untiled", "bwd_dh", "marginal"): (0.628156e9 + 0.015830e9,
                                                  "profiles/ncu_gemm2_backward_medium_untiled.md"),
    ("medium", "untiled", "joint_fwd", "marginal"): (0.009181e9 + 0.556763e9,
                                                     "profiles/ncu_joint_tc_medium_untiled.md"),
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=d["hbm_gbs"], tensor=d["bf16_tflops"], tensor_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, tensor=1590.0, tensor_sustained=1400.0, source="fallback")


def modes_of(args):
    """Modes a run measures; the first is the headline."""
    return ["untiled", "tiled"] if args.mode == "both" else [args.mode]


def config_of(batch, args, n_gpus):
    """The workload as both arms' JSON lines name it (the headline mode)."""
    d = batch.dims
    return {"workload": args.workload, "B": d["B"], "T": d["T"], "U": d["U"], "D_enc": d["D_enc"],
            "D_pred": d["D_pred"], "H": d["H"], "V": d["V"], "mode": modes_of(args)[0], "path": args.path,
            "loss": args.loss, "prune_S": args.prune,
            "durations": list(synth.TDT_DURATIONS) if args.loss == "tdt" else None,
            "valid_cells": batch.valid_cells(), "padded_cells": batch.padded_cells(),
            "l2": "flushed between timed steps (256 MiB write)", "parallelism": f"dp{n_gpus}",
            "global_batch": d["B"] * n_gpus}


# ------------------------------------------------------------------ algorithmic work per stage

def stage_work(batch, stage, mode, cells=None, n_dur=0):
    """(kind, amount per call): tensor flops or HBM bytes that the stage must
    do by definition (recomputation and tile padding excluded); ``cells`` = the
    valid cells of the lattice computed (default: the whole lattice's);
    ``n_dur`` = outputs of a duration head beside the V label logits."""
    d = batch.dims
    H, V = d["H"], d["V"] + n_dur
    cells = batch.valid_cells() if cells is None else cells
    if stage in ("joint_fwd", "bwd_dWo", "bwd_dh"):
        return "tensor", 2.0 * H * V * cells
    if stage == "joint_bwd_dz":
        # tiled: the logits are recomputed (2HV per cell); untiled: elementwise over the stored logits
        return ("tensor", 2.0 * H * V * cells) if mode == "tiled" else ("hbm", 4.0 * V * cells)
    if stage == "joint_bwd":
        return "tensor", 4.0 * H * V * cells
    if stage == "lattice_dp":
        return "hbm", (8 + 4 + 8 + 4) * cells
    if stage == "projection":
        return "tensor", 2.0 * (d["B"] * d["T"] * d["D_enc"] * H + d["B"] * (d["U"] + 1) * d["D_pred"] * H)
    if stage == "projection_bwd":
        return "tensor", 4.0 * (d["B"] * d["T"] * d["D_enc"] * H + d["B"] * (d["U"] + 1) * d["D_pred"] * H)
    return None, 0.0


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples every 20 ms; only samples inside [mark_start, mark_end]
    (host wall clock) are reported."""

    def __init__(self, index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.t0 = self.t1 = None
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-i", str(index), "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        self.lines_at = []
        time.sleep(0.3)

    def mark_start(self):
        self.f.flush()
        self.t0 = self._count()

    def mark_end(self):
        time.sleep(0.05)
        self.t1 = self._count()

    def _count(self):
        try:
            return sum(1 for _ in open(self.f.name))
        except OSError:
            return 0

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = []
        lines = open(self.f.name).read().splitlines()
        lo = self.t0 or 0
        hi = self.t1 if self.t1 is not None else len(lines)
        window = lines[max(0, lo - 1):hi] if hi > lo else lines[max(0, lo - 2):lo + 1]
        for line in window:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        for r in rows:
            for name, col in (("hw_slowdown", 5), ("hw_thermal_slowdown", 6), ("sw_thermal_slowdown", 7),
                              ("sw_power_cap", 8)):
                if r[col].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ oracle (CPU) leg

def duration_head(batch):
    """The token-and-duration workloads' duration head (seeded, like the other inputs)."""
    return synth.duration_head(batch, len(synth.TDT_DURATIONS), seed=5)


def oracle_sample(batch, utterance=0, loss="marginal"):
    """Times the fp64 oracle on one utterance; returns (seconds, metric units)."""
    import numpy as np

    import oracle
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    w = np.zeros(batch.f.shape[0])
    w[utterance] = 1.0
    t0 = time.perf_counter()
    if loss == "tdt":
        W_d, b_d = (t.double().numpy() for t in duration_head(batch))
        oracle.tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d, b_d, batch.labels.numpy(), batch.T_len.numpy(),
                           batch.U_len.numpy(), synth.TDT_DURATIONS, grad_loss=w, utterances=[utterance])
    else:
        oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(),
                       grad_loss=w, utterances=[utterance], loss=loss)
    dt = time.perf_counter() - t0
    d = batch.dims
    units = d["T"] * (d["U"] + 1) * d["V"]      # this utterance's share of B*T*(U+1)*V
    return dt, units


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    batch = synth.workload(args.workload)
    for _ in range(args.warmup):
        oracle_sample(batch, loss=args.loss)
    times = []
    units = 0
    for _ in range(args.steps):
        dt, units = oracle_sample(batch, loss=args.loss)
        times.append(dt)
    sec = sum(times) / len(times)
    value = units / sec
    Tb, Ub = int(batch.T_len[0]), int(batch.U_len[0])
    sample = (f"utterance 0 of {args.workload} (T_len={Tb}, U_len={Ub}) per step; "
              f"units = T*(U+1)*V of one utterance")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(batch, args, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores(), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def measure_mode(args, mode, batch, d, dev, world, rank, local, flush):
    """Times one mode: warm-up, K timed steps (each after an L2 flush), the
    end-to-end variant with host buffers, per-stage device times."""
    dtype = "bf16" if batch.dtype == "bf16" else "f32"
    tdt = args.loss == "tdt"
    durations = tuple(synth.TDT_DURATIONS) if tdt else ()
    dims = frnnt.dims_of(d["f"], d["g"], d["W_o"], dtype, mode, args.path, args.chunk_cells, batch.blank,
                         "marginal" if tdt else args.loss, args.prune, durations)
    bounds = None
    valid = batch.valid_cells()
    if args.prune:
        hb = synth.diagonal_bounds(batch.T_len, batch.U_len, batch.f.shape[1], args.prune)
        valid = sum(min(args.prune, int(batch.U_len[b]) - int(hb[b, t]) + 1)
                    for b in range(batch.dims["B"]) for t in range(int(batch.T_len[b])))
        bounds = hb.to(dev)
    out = frnnt.Outputs(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], dims, W_d=d.get("W_d"),
                        b_d=d.get("b_d"))
    stream = torch.cuda.current_stream(dev)

    def call(check=False):
        if tdt:
            res = frnnt.fwd_bwd_tdt(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["W_d"], d["b_d"],
                                    d["labels"], d["T_len"], d["U_len"], durations, mode=mode,
                                    chunk_cells=args.chunk_cells, blank=batch.blank, out=out, check=check,
                                    stream=stream)
        elif bounds is not None:
            res = frnnt.fwd_bwd_pruned(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"],
                                       d["T_len"], d["U_len"], bounds, args.prune, mode=mode, path=args.path,
                                       chunk_cells=args.chunk_cells, loss=args.loss, blank=batch.blank, out=out,
                                       check=check, stream=stream)
        else:
            res = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                                d["U_len"], mode=mode, path=args.path, chunk_cells=args.chunk_cells, loss=args.loss,
                                blank=batch.blank, out=out, check=check, stream=stream)
        if world > 1:
            # the data-parallel exchange: weight gradients summed over ranks
            rdist.allreduce_weight_grads(res[1])
        return res

    # peak device memory of one call: the library allocates nothing, so the
    # peak is inputs + outputs + workspace (measured before other buffers exist)
    call(check=True)
    torch.cuda.synchronize()
    flush_bytes = flush.numel()           # the L2-flush buffer is the bench's, not the call's
    torch.cuda.reset_peak_memory_stats(dev)
    call(check=True)
    torch.cuda.synchronize()
    peak_bytes = torch.cuda.max_memory_allocated(dev) - flush_bytes

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    frnnt.profile_read()
    frnnt.profile(True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if sampler:
        sampler.mark_start()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        call()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_end()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    frnnt.profile(False)
    stages = frnnt.profile_read()
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())

    # end to end through the public API with host buffers: pinned H2D of the
    # step's inputs, the call, D2H of the loss and status word
    host = {k: v.cpu().pin_memory() for k, v in d.items()}
    loss_h = torch.empty(batch.f.shape[0], dtype=torch.float32).pin_memory()
    status_h = torch.empty(4, dtype=torch.int32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = loss_h.numel() * 4 + status_h.numel() * 4
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for k, v in host.items():
            d[k].copy_(v, non_blocking=True)
        call()
        loss_h.copy_(out.loss, non_blocking=True)
        status_h.copy_(out.status, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if int(status_h[0]) != 0:
            raise RuntimeError(f"device status {int(status_h[0])}")
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e = sum(e2e_ms) / len(e2e_ms)
    if world > 1:
        t = torch.tensor([e2e], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e = float(t.item())

    # cells of the lattice that is computed: B*T*(U+1), or B*T*S when pruned
    units = (batch.dims["B"] * batch.dims["T"] * args.prune if args.prune else batch.padded_cells()) * batch.dims["V"]
    launches = sum(v["launches"] for v in stages.values())
    roofline = None
    pk = peaks()
    if stages:
        dom = max(stages, key=lambda k: stages[k]["ms"])
        kind, work = stage_work(batch, dom, mode, valid, len(durations))
        per_call_ms = stages[dom]["ms"] / args.steps
        tr = None if args.prune else MEASURED_TRAFFIC.get((args.workload, mode, dom, args.loss))
        if kind == "tensor":
            achieved = work / (per_call_ms / 1e3) / 1e12
            roofline = {"bound": "tensor", "achieved": achieved, "peak": pk["tensor_sustained"], "unit": "TFLOP/s",
                        "frac": achieved / pk["tensor_sustained"], "traffic": tr[0] if tr else None,
                        "traffic_source": tr[1] if tr else None, "stage": dom,
                        "launches_per_step": stages[dom]["launches"] / args.steps,
                        "peak_source": pk["source"] + " sustained dense bf16 (the stage runs inside a long step)"}
        elif kind == "hbm":
            achieved = work / (per_call_ms / 1e3) / 1e9
            roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                        "frac": achieved / pk["hbm"], "traffic": tr[0] if tr else None,
                        "traffic_source": tr[1] if tr else None, "stage": dom, "peak_source": pk["source"]}
    return {"ms": ms, "value": world * units / (ms / 1e3), "peak_bytes": peak_bytes,
            "valid_cells_per_s": world * valid * batch.dims["V"] / (ms / 1e3),
            "e2e": {"value": world * units / (e2e / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e},
            "launches": launches, "roofline": roofline, "clocks": clocks,
            "stages": {k: {"ms_per_step": v["ms"] / args.steps, "launches_per_step": v["launches"] / args.steps}
                       for k, v in stages.items()}}


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    idx = synth.WORKLOADS[args.workload]["index"]
    batch = synth.workload(args.workload, seed=1000 + idx + 7919 * rank)
    d = {k: getattr(batch, k).to(dev).contiguous()
         for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")}
    if args.loss == "tdt":
        W_d, b_d = duration_head(batch)
        d["W_d"], d["b_d"] = W_d.to(dev).contiguous(), b_d.to(dev).contiguous()
    dtype = "bf16" if batch.dtype == "bf16" else "f32"
    elt = 2 if dtype == "bf16" else 4
    footprint = (2 * sum(getattr(batch, k).numel() for k in ("f", "g", "W_f", "W_g", "W_o", "b_o")) * elt +
                 4 * (batch.labels.numel() + 2 * batch.T_len.numel()) + 4 * batch.T_len.numel())

    modes = modes_of(args)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    results = {}
    for m in modes:
        results[m] = measure_mode(args, m, batch, d, dev, world, rank, local, flush)
    head = results[modes[0]]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, u = oracle_sample(batch, loss=args.loss)
        Tb, Ub = int(batch.T_len[0]), int(batch.U_len[0])
        cpu = {"value": u / dt, "unit": UNIT, "cores": cores(), "kind": "oracle",
               "sample": f"utterance 0 of {args.workload} (T_len={Tb}, U_len={Ub}); units = T*(U+1)*V of one "
                         f"utterance; numpy fp64, BLAS threads = all cores"}

    if rank == 0:
        cfg = config_of(batch, args, world)
        line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": dtype, "data": "synthetic (seeded; shapes of the workload)",
                "config": cfg,
                "peak_gb": head["peak_bytes"] / 1e9, "footprint_gb": footprint / 1e9,
                "peak_over_footprint": head["peak_bytes"] / footprint,
                "valid_cells_per_s": head["valid_cells_per_s"], "e2e": head["e2e"], "gpu_launches": head["launches"],
                "stages": head["stages"], "roofline": head["roofline"], "cpu_baseline": cpu,
                "clocks": head["clocks"],
                "modes": {m: {"value": r["value"], "ms_per_step": r["ms"], "peak_gb": r["peak_bytes"] / 1e9,
                              "peak_over_footprint": r["peak_bytes"] / footprint, "e2e_value": r["e2e"]["value"],
                              "roofline": r["roofline"], "stages": r["stages"], "clocks": r["clocks"]}
                          for m, r in results.items()}}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
