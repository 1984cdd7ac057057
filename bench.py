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
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the per-workload block (short, medium, long, large in both modes) and the "
                        "chunk-size protocol that a one-GPU run adds after the headline")
    return p.parse_args(argv)


# DRAM bytes (read + write) per launch of a stage's kernel, from one ncu
# capture of that kernel in the bench's own launch configuration (the file
# under profiles/ gives the command), keyed by (workload, mode, stage, loss).
# An entry is removed whenever its kernel changes, so the roofline's traffic is
# null rather than stale.
MEASURED_TRAFFIC = {
    ("medium", "untiled", "bwd_dWo", "marginal"): (1.111446e9 + 0.003530e9,
                                                   "profiles/ncu_gemm2_backward_medium_untiled.md"),
    ("medium", "untiled", "bwd_dh", "marginal"): (0.628257e9 + 0.015802e9,
                                                  "profiles/ncu_gemm2_backward_medium_untiled.md"),
    ("medium", "untiled", "joint_fwd", "marginal"): (0.009422e9 + 0.555290e9,
                                                     "profiles/ncu_joint_tc_medium_untiled.md"),
    # one full 592-tile chunk launch (the stage has four real launches per call)
    ("medium", "tiled", "joint_bwd_dz", "marginal"): (0.007356e9 + 0.200818e9,
                                                      "profiles/ncu_joint_bwd_dz_medium_tiled.md (per 592-tile launch)"),
}


# Nominal dense bf16 tensor throughput of one B200 (NVIDIA's B200 datasheet
# figure without 2:4 sparsity), for context beside the measured peaks.
DATASHEET_BF16_TFLOPS = 2250.0
# MUFU (tanh, exp2) results per clock per SM; 148 SMs.
MUFU_PER_CLK_SM = 16
SMS = 148


def peaks():
    """Roofline denominators: the measured copy bandwidth and the measured
    dense bf16 GEMM throughput of this machine's B200s (burst: a GEMM timed alone
    at full clocks, the right denominator for a stage of a millisecond-scale
    step; sustained: seconds back to back under the power cap)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=d["hbm_gbs"], tensor=d["bf16_tflops"], tensor_sustained=d["bf16_tflops_sustained"],
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm=6650.0, tensor=1590.0, tensor_sustained=1400.0, sm_max_mhz=1965.0, source="fallback")


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


def oracle_sample(batch, budget_s=10.0, loss="marginal", first=0):
    """Times the fp64 oracle on utterances first, first+1, ... until ``budget_s``
    seconds of CPU work (at least one utterance).  The metric's unit is the
    batch's padded cells B*T*(U+1)*V per second; the oracle computes only
    valid cells, so the sample stands for the batch in proportion to its valid
    cells: value = padded units of the batch / (sample time * batch valid cells
    / sample valid cells).  Also returns the plain valid-cell rate."""
    import numpy as np

    import oracle
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    B = batch.f.shape[0]
    d = batch.dims
    W_d = b_d = None
    if loss == "tdt":
        W_d, b_d = (t.double().numpy() for t in duration_head(batch))
    done, secs, valid = [], 0.0, 0
    for k in range(B):
        b = (first + k) % B
        w = np.zeros(B)
        w[b] = 1.0
        t0 = time.perf_counter()
        if loss == "tdt":
            oracle.tdt_fwd_bwd(f, g, W_f, W_g, W_o, b_o, W_d, b_d, batch.labels.numpy(), batch.T_len.numpy(),
                               batch.U_len.numpy(), synth.TDT_DURATIONS, grad_loss=w, utterances=[b])
        else:
            oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(), batch.U_len.numpy(),
                           grad_loss=w, utterances=[b], loss=loss)
        secs += time.perf_counter() - t0
        done.append(b)
        valid += int(batch.T_len[b]) * (int(batch.U_len[b]) + 1)
        if secs >= budget_s:
            break
    batch_secs = secs * batch.valid_cells() / valid
    return {"seconds": secs, "utterances": done, "valid_cells": valid, "batch_seconds_est": batch_secs,
            "value": batch.padded_cells() * d["V"] / batch_secs, "valid_cells_per_s": valid * d["V"] / secs}


def oracle_line(batch, name, sample):
    """The cpu_baseline object of a JSON line from one oracle sample."""
    return {"value": sample["value"], "unit": UNIT, "cores": cores(), "kind": "oracle",
            "valid_cells_per_s": sample["valid_cells_per_s"],
            "sample": (f"{name}: utterances {sample['utterances']} ({sample['valid_cells']} valid cells of the "
                       f"batch's {batch.valid_cells()}) in {sample['seconds']:.2f} s; value = the batch's "
                       f"B*T*(U+1)*V over the sample time scaled to the batch's valid cells "
                       f"({sample['batch_seconds_est']:.1f} s per batch); valid_cells_per_s = the sample's "
                       f"T_len*(U_len+1)*V per second; numpy fp64, BLAS threads = all cores")}


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
    # each step: the oracle on utterance 0 of the workload (a bounded sample,
    # scaled to the batch by its valid cells; see oracle_sample)
    for _ in range(args.warmup):
        oracle_sample(batch, budget_s=0.0, loss=args.loss)
    samples = [oracle_sample(batch, budget_s=0.0, loss=args.loss) for _ in range(args.steps)]
    secs = sum(x["batch_seconds_est"] for x in samples) / len(samples)
    value = batch.padded_cells() * batch.dims["V"] / secs
    cpu = oracle_line(batch, args.workload, samples[-1])
    cpu["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(batch, args, args.gpus), "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def stage_rooflines(batch, mode, stages, steps, valid, n_dur, workload, loss, prune):
    """Per stage: its algorithmic work over its device time against the peak
    of its bound (tensor: measured burst dense bf16, also shown against the
    sustained and datasheet figures; hbm: measured copy bandwidth)."""
    pk = peaks()
    out = {}
    for name, st in stages.items():
        kind, work = stage_work(batch, name, mode, valid, n_dur)
        if kind is None or st["ms"] <= 0:
            continue
        per_call_ms = st["ms"] / steps
        tr = None if prune else MEASURED_TRAFFIC.get((workload, mode, name, loss))
        if kind == "tensor":
            achieved = work / (per_call_ms / 1e3) / 1e12
            out[name] = {"bound": "tensor", "achieved": achieved, "peak": pk["tensor"], "unit": "TFLOP/s",
                         "frac": achieved / pk["tensor"], "traffic": tr[0] if tr else None,
                         "traffic_source": tr[1] if tr else None, "stage": name,
                         "ms_per_step": per_call_ms, "launches_per_step": st["launches"] / steps,
                         "frac_sustained": achieved / pk["tensor_sustained"],
                         "frac_datasheet": achieved / DATASHEET_BF16_TFLOPS,
                         "peak_source": pk["source"] + " burst dense bf16 (cuBLAS GEMM timed alone at full "
                                                       "clocks); frac_sustained: against the power-capped "
                                                       "sustained figure; frac_datasheet: against 2250 TFLOP/s"}
        else:
            achieved = work / (per_call_ms / 1e3) / 1e9
            out[name] = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": achieved / pk["hbm"], "traffic": tr[0] if tr else None,
                         "traffic_source": tr[1] if tr else None, "stage": name,
                         "ms_per_step": per_call_ms, "launches_per_step": st["launches"] / steps,
                         "peak_source": pk["source"] + " copy bandwidth"}
    return out


def mufu_roofline(batch, valid, ms, clocks):
    """MUFU work of the path, 2H tanh + 2V exp per valid cell (forward and
    backward), over the whole step against 16 results/clock/SM on 148 SMs at
    the SM clock seen under load."""
    d = batch.dims
    ops = (2.0 * d["H"] + 2.0 * d["V"]) * valid
    mhz = (clocks or {}).get("sm_mhz") or peaks()["sm_max_mhz"]
    peak = MUFU_PER_CLK_SM * SMS * mhz * 1e6
    achieved = ops / (ms / 1e3)
    return {"bound": "alu", "unit": "MUFU results/s", "achieved": achieved, "peak": peak, "frac": achieved / peak,
            "per_cell": "2H tanh + 2V exp", "peak_source": f"16/clk/SM x 148 SMs x {mhz:.0f} MHz"}


def measure_mode(args, mode, batch, d, dev, world, rank, local, flush, workload=None, chunk_cells=None,
                 steps=None, warmup=None, e2e=True):
    """Times one mode: warm-up, K timed steps (each after an L2 flush), the
    end-to-end variant with host buffers, per-stage device times."""
    workload = args.workload if workload is None else workload
    chunk_cells = args.chunk_cells if chunk_cells is None else chunk_cells
    steps = args.steps if steps is None else steps
    warmup = args.warmup if warmup is None else warmup
    dtype = "bf16" if batch.dtype == "bf16" else "f32"
    tdt = args.loss == "tdt"
    durations = tuple(synth.TDT_DURATIONS) if tdt else ()
    # data parallelism: the weight gradients come back as fp32 accumulators
    # (views of one flat buffer) so the exchange is one fp32 all-reduce
    wf32 = world > 1
    dims = frnnt.dims_of(d["f"], d["g"], d["W_o"], dtype, mode, args.path, chunk_cells, batch.blank,
                         "marginal" if tdt else args.loss, args.prune, durations, wgrad_f32=wf32)
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
                                    chunk_cells=chunk_cells, blank=batch.blank, out=out, check=check,
                                    stream=stream, wgrad_f32=wf32)
        elif bounds is not None:
            res = frnnt.fwd_bwd_pruned(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"],
                                       d["T_len"], d["U_len"], bounds, args.prune, mode=mode, path=args.path,
                                       chunk_cells=chunk_cells, loss=args.loss, blank=batch.blank, out=out,
                                       check=check, stream=stream, wgrad_f32=wf32)
        else:
            res = frnnt.fwd_bwd(d["f"], d["g"], d["W_f"], d["W_g"], d["W_o"], d["b_o"], d["labels"], d["T_len"],
                                d["U_len"], mode=mode, path=args.path, chunk_cells=chunk_cells, loss=args.loss,
                                blank=batch.blank, out=out, check=check, stream=stream, wgrad_f32=wf32)
        if world > 1:
            # the data-parallel exchange: one all-reduce of the flat fp32 weight
            # gradients, each sum rounded once to the input dtype
            rdist.allreduce_weight_grads(res[1], out_dtype=d["W_o"].dtype)
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

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    frnnt.profile_read()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if sampler:
        sampler.mark_start()
    for i in range(steps):
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
    launches = frnnt.profile_read()           # launch counts of the timed steps (always kept)
    # per-stage device times from separate steps: the library's stage events
    # sit between kernels that otherwise start while the previous one drains,
    # so they are kept out of the timed steps
    prof_steps = min(steps, 5)
    frnnt.profile(True)
    for _ in range(prof_steps):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    frnnt.profile(False)
    stages = frnnt.profile_read()
    for k, v in stages.items():           # as totals over the timed steps, like the launch counts
        v["ms"] *= steps / prof_steps
        v["launches"] = launches[k]["launches"] if k in launches else v["launches"] * steps / prof_steps
    ms = sum(a.elapsed_time(b) for a, b in evs) / steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())

    # cells of the lattice that is computed: B*T*(U+1), or B*T*S when pruned
    units = (batch.dims["B"] * batch.dims["T"] * args.prune if args.prune else batch.padded_cells()) * batch.dims["V"]
    res = {"ms": ms, "value": world * units / (ms / 1e3), "peak_bytes": peak_bytes,
           "valid_cells_per_s": world * valid * batch.dims["V"] / (ms / 1e3), "clocks": clocks,
           "launches": sum(v["launches"] for v in stages.values()),
           "stages": {k: {"ms_per_step": v["ms"] / steps, "launches_per_step": v["launches"] / steps}
                      for k, v in stages.items()}}
    rl = stage_rooflines(batch, mode, stages, steps, valid, len(durations), workload, args.loss, args.prune)
    res["rooflines"] = rl
    res["roofline"] = rl[max(rl, key=lambda k: rl[k]["ms_per_step"])] if rl else None
    res["mufu"] = mufu_roofline(batch, valid, ms, clocks)

    if e2e:
        # end to end through the public API with host buffers, as a training
        # loop feeds it: every step's inputs come from pinned host memory (one
        # packed H2D copy into one of two device buffers, on a copy stream, so
        # that step i+1's inputs arrive while step i computes), then the call,
        # then the D2H of its loss and status word.  The steps are queued back to
        # back; the time per step is the device time from the end of the last
        # warm-up step to the end of the last step, over the timed steps, so
        # every timed step's copies lie inside it.  Results are checked after
        # the last step.
        d = dict(d)   # the call's inputs become views of the device buffers (the caller's dict is kept)
        keys = list(d.keys())
        sizes = [(d[k].numel() * d[k].element_size() + 255) // 256 * 256 for k in keys]
        host_buf = torch.empty(sum(sizes), dtype=torch.uint8).pin_memory()
        dev_bufs = [torch.empty(sum(sizes), dtype=torch.uint8, device=dev) for _ in range(2)]
        views = [{}, {}]
        off = 0
        for k, n in zip(keys, sizes):
            nb = d[k].numel() * d[k].element_size()
            host_buf[off:off + nb].copy_(d[k].cpu().contiguous().view(-1).view(torch.uint8))
            for b in range(2):
                views[b][k] = dev_bufs[b][off:off + nb].view(d[k].dtype).view(d[k].shape)
            off += n
        n = warmup + steps
        loss_h = torch.empty(n, batch.f.shape[0], dtype=torch.float32).pin_memory()
        status_h = torch.zeros(n, 4, dtype=torch.int32).pin_memory()
        h2d = sum(d[k].numel() * d[k].element_size() for k in keys)
        d2h = loss_h[0].numel() * 4 + status_h[0].numel() * 4
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(n)]
        used = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        torch.cuda.synchronize()
        t_host = time.perf_counter()
        for i in range(n):
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(used[i - 2])   # the buffer's previous step is done with it
                dev_bufs[i % 2].copy_(host_buf, non_blocking=True)
                copied[i].record(copy_stream)
            flush.zero_()
            stream.wait_event(copied[i])
            d.update(views[i % 2])
            call()
            used[i].record(stream)
            loss_h[i].copy_(out.loss, non_blocking=True)
            status_h[i].copy_(out.status, non_blocking=True)
            done[i].record(stream)
        t_host = (time.perf_counter() - t_host) / n
        torch.cuda.synchronize()
        if int(status_h[:, 0].abs().sum()) != 0:
            raise RuntimeError(f"device status {status_h[:, 0].tolist()}")
        w0 = max(warmup, 1)   # the first step has no predecessor to be timed from
        e2e_t = done[w0 - 1].elapsed_time(done[n - 1]) / (n - w0)
        if world > 1:
            t = torch.tensor([e2e_t], device=dev)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            e2e_t = float(t.item())
        res["e2e"] = {"value": world * units / (e2e_t / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "ms_per_step": e2e_t,
                      "host_queue_ms_per_step": t_host * 1e3,
                      "how": "per step: pinned H2D of the inputs (one packed copy, on a copy stream into one of two "
                             "device buffers, so the next step's inputs arrive during this step), the public call, "
                             "D2H of loss and status; steps queued back to back; device time from the end of the "
                             "warm-up to the end of the last step, per step"}
    del out
    return res


def inputs_on(batch, dev, loss):
    d = {k: getattr(batch, k).to(dev).contiguous()
         for k in ("f", "g", "W_f", "W_g", "W_o", "b_o", "labels", "T_len", "U_len")}
    if loss == "tdt":
        W_d, b_d = duration_head(batch)
        d["W_d"], d["b_d"] = W_d.to(dev).contiguous(), b_d.to(dev).contiguous()
    return d


def footprint_bytes(batch):
    """Inputs + weights + gradients (gradients in the input dtype) + the int arrays."""
    elt = 2 if batch.dtype == "bf16" else 4
    return (2 * sum(getattr(batch, k).numel() for k in ("f", "g", "W_f", "W_g", "W_o", "b_o")) * elt +
            4 * (batch.labels.numel() + 2 * batch.T_len.numel()) + 4 * batch.T_len.numel())


def mode_entry(r, footprint):
    return {"value": r["value"], "ms_per_step": r["ms"], "valid_cells_per_s": r["valid_cells_per_s"],
            "peak_gb": r["peak_bytes"] / 1e9, "peak_over_footprint": r["peak_bytes"] / footprint,
            "e2e_value": r["e2e"]["value"] if "e2e" in r else None, "roofline": r["roofline"],
            "rooflines": r["rooflines"], "mufu": r["mufu"], "stages": r["stages"], "clocks": r["clocks"]}


WORKLOAD_BLOCK = ("short", "medium", "long", "large")
PROTOCOL_CHUNKS = (8192, 16384, 32768, 65536, 131072, 262144)
PROTOCOL_WORKLOADS = ("medium", "long")


def protocol(args, name, batch, d, dev, flush, footprint, untiled):
    """The comparison protocol of "Flash RNN-T" (abstract): each mode at its
    lowest-memory setting whose throughput is within 95 % of that mode's peak.
    Tiled mode's memory knob is the backward chunk (cells per chunk); untiled
    mode has none (one setting)."""
    pts = []
    for c in PROTOCOL_CHUNKS:
        r = measure_mode(args, "tiled", batch, d, dev, 1, 0, 0, flush, workload=name, chunk_cells=c,
                         steps=min(args.steps, 5), warmup=3, e2e=False)
        pts.append({"chunk_cells": c, "ms_per_step": r["ms"], "value": r["value"], "peak_gb": r["peak_bytes"] / 1e9,
                    "peak_over_footprint": r["peak_bytes"] / footprint})
    best = max(p["value"] for p in pts)
    ok = [p for p in pts if p["value"] >= 0.95 * best]
    pick = min(ok, key=lambda p: p["peak_gb"])
    return {"tiled": {"points": pts, "peak_value": best, "lowest_memory_within_95pct": pick},
            "untiled": {"points": [{"chunk_cells": None, "ms_per_step": untiled["ms"], "value": untiled["value"],
                                    "peak_gb": untiled["peak_bytes"] / 1e9,
                                    "peak_over_footprint": untiled["peak_bytes"] / footprint}],
                        "note": "no memory knob: the logits of the whole lattice are stored"}}


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
    d = inputs_on(batch, dev, args.loss)
    dtype = "bf16" if batch.dtype == "bf16" else "f32"
    footprint = footprint_bytes(batch)

    modes = modes_of(args)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    results = {}
    for m in modes:
        results[m] = measure_mode(args, m, batch, d, dev, world, rank, local, flush)
    head = results[modes[0]]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_line(batch, args.workload, oracle_sample(batch, budget_s=10.0, loss=args.loss))

    # one GPU, default criterion: every workload in both modes, and the
    # chunk-size protocol, after the headline
    workloads, proto = None, None
    if world == 1 and not args.no_workloads and args.loss == "marginal" and not args.prune and args.path == "auto":
        del d
        workloads, proto = {}, {}
        for name in WORKLOAD_BLOCK:
            wb = batch if name == args.workload else synth.workload(name)
            wd = inputs_on(wb, dev, args.loss)
            fp = footprint_bytes(wb)
            entry = {"footprint_gb": fp / 1e9, "valid_cells": wb.valid_cells(), "padded_cells": wb.padded_cells()}
            measured = {}
            for m in ("untiled", "tiled"):
                r = results[m] if name == args.workload and m in results else measure_mode(
                    args, m, wb, wd, dev, 1, 0, local, flush, workload=name, e2e=False)
                measured[m] = r
                entry[m] = mode_entry(r, fp)
                torch.cuda.empty_cache()
            if name in PROTOCOL_WORKLOADS:
                proto[name] = protocol(args, name, wb, wd, dev, flush, fp, measured["untiled"])
            if not args.no_cpu_baseline:
                entry["oracle"] = oracle_line(wb, name, oracle_sample(wb, budget_s=3.0))
            workloads[name] = entry
            del wd
            torch.cuda.empty_cache()

    if rank == 0:
        cfg = config_of(batch, args, world)
        line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": head["ms"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": dtype, "data": "synthetic (seeded; shapes of the workload)",
                "config": cfg,
                "peak_gb": head["peak_bytes"] / 1e9, "footprint_gb": footprint / 1e9,
                "peak_over_footprint": head["peak_bytes"] / footprint,
                "valid_cells_per_s": head["valid_cells_per_s"], "e2e": head["e2e"], "gpu_launches": head["launches"],
                "stages": head["stages"], "roofline": head["roofline"], "rooflines": head["rooflines"],
                "mufu": head["mufu"], "cpu_baseline": cpu, "clocks": head["clocks"],
                "modes": {m: mode_entry(r, footprint) for m, r in results.items()}}
        if workloads is not None:
            line["workloads"] = workloads
            line["protocol"] = proto
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
