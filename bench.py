#!/usr/bin/env python3
"""Benchmark: W8A8 / power-of-two Mamba2 prefill tokens/s on one B200 per rank.

Workload (default): the Mamba2-130M-shaped stack -- 24 pre-normed residual
mixer layers (d_model 768, d_inner 1536, 24 heads of 64, d_state 128),
batch 1, 2048 tokens, outlier-injected N(0,1) inputs, random-init weights,
activation scales dynamic per token, PoT exponents calibrated on the GPU
from 16 seeded sequences of 512 tokens.  One step = one prefill of the whole
stack over the batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--mode dynamic|static]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

Under torchrun each rank runs an independent replica on its own GPU (the
prefill of independent sequences needs no collective): weak scaling; the
step time is the max over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from quantized_state_space_mamba2_b200 import synth as S  # noqa: E402

WORKLOAD = "stack130m_24l_b1_t2048"
OUTLIER_SEED = 4242
L2_FLUSH_BYTES = 512 << 20
SCAN_OPS_PER_CELL = 6  # decay multiply, rounding shift, dt*x*B multiply-add, clamp (2), C*h MAC


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--mode", default="dynamic", choices=["dynamic", "static"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scan-tile", default=None,
                    help="npt,pc,tch of the sequential scan kernel (a compiled variant)")
    return ap.parse_args()


def workload():
    w = S.WORKLOADS[WORKLOAD]
    return w["shape"], w["layers"], w["batch"], w["seqlen"], w["n_outliers"], w["outlier_scale"]


def layer_params(n_layers, shape):
    return [S.layer_params(shape, 1000 + l) for l in range(n_layers)]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return json.load(f)
    except OSError:
        return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle baseline
class OracleSample:
    """The oracle as it stands (single-threaded C, composed by numpy) on a
    bounded sample of the workload: one stack layer (pre-norm + mixer +
    residual) over the full batch, scaled to the stack's token rate
    (tokens / (layers x one layer's time))."""

    def __init__(self, shape, n_layers, mode: str):
        import oracle as O
        _, _, B, T, n_out, scale = workload()
        self.O, self.B, self.T, self.n_layers = O, B, T, n_layers
        P = S.layer_params(shape, 1000)
        self.L = O.prepare_layer(P, shape, rotate=1,
                                 mode=O.DYNAMIC if mode == "dynamic" else O.STATIC, prenorm=True)
        xcal = S.calibration_batch(shape.d_model, 64, n_out, scale, OUTLIER_SEED, n_seqs=1)
        O.calibrate_layer(self.L, xcal, residual=True)
        self.x = S.activations(B, T, shape.d_model, seed=1, n_outliers=n_out, outlier_scale=scale,
                               outlier_seed=OUTLIER_SEED)

    def run(self) -> float:
        t0 = time.perf_counter()
        self.O.mixer_prefill(self.L, self.x, residual=True)
        return time.perf_counter() - t0

    def describe(self, seconds: float) -> dict:
        return {"value": self.B * self.T / (seconds * self.n_layers), "unit": "tokens/s",
                "cores": 1, "kind": "oracle",
                "sample": f"1 of {self.n_layers} stack layers over {self.B}x{self.T} tokens "
                          f"({seconds:.2f} s), scaled to {self.n_layers} layers"}


def cpu_oracle_sample(shape, n_layers, mode: str) -> dict:
    o = OracleSample(shape, n_layers, mode)
    return o.describe(o.run())


def run_reference(args):
    """--impl reference: the CPU oracle on this host's cores (rank 0 only);
    each step is the bounded sample above."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    shape, n_layers, B, T, _, _ = workload()
    o = OracleSample(shape, n_layers, args.mode)
    for _ in range(args.warmup):
        o.run()
    secs = [o.run() for _ in range(max(1, args.steps))]
    per_step = statistics.mean(secs) * n_layers      # one stack prefill
    value = B * T / per_step
    cb = o.describe(statistics.mean(secs))
    line = {"impl": "reference", "metric": "W8A8 Mamba2 prefill tokens/s", "value": value,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": len(secs), "warmup": args.warmup,
            "ms_per_step": 1000.0 * per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8+int32 fixed point (CPU oracle)",
            "data": "synthetic", "config": config_block(args, shape, n_layers, B, T),
            "cpu_baseline": dict(cb, value=value),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_block(args, shape, n_layers, B, T):
    return {"workload": WORKLOAD, "layers": n_layers, "batch": B, "seq_len": T,
            "d_model": shape.d_model, "d_inner": shape.d_inner, "nheads": shape.nheads,
            "d_state": shape.d_state, "act_quant": args.mode, "hadamard": True,
            "calibration": "16 seeded sequences x 512 tokens (GPU, stage by stage)",
            "l2": "flushed between timed steps (512 MiB write)", "parallelism": f"replica x{args.gpus}",
            "scan_tile": args.scan_tile or "4,4,16"}


# ---------------------------------------------------------------- the GPU arm
def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    from quantized_state_space_mamba2_b200 import build, lib
    from quantized_state_space_mamba2_b200.model import DeviceStack

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    lib.load()
    if args.scan_tile:
        lib.set_scan_tile(*[int(v) for v in args.scan_tile.split(",")])
    dev = torch.device("cuda", local)
    shape, n_layers, B, T, n_out, scale = workload()
    mode = lib.FM_DYNAMIC if args.mode == "dynamic" else lib.FM_STATIC

    stack = DeviceStack(layer_params(n_layers, shape), shape, rotate=1, mode=mode, device=dev)
    xcal = S.calibration_batch(shape.d_model, T, n_out, scale, OUTLIER_SEED)
    stack.calibrate(torch.from_numpy(xcal).to(dev))
    del xcal
    x_host = S.activations(B, T, shape.d_model, seed=1 + rank, n_outliers=n_out,
                           outlier_scale=scale, outlier_seed=OUTLIER_SEED)
    x0 = torch.from_numpy(x_host).to(dev)
    r = torch.empty_like(x0)
    M = B * T
    ws = stack.layers[0].workspace(B, T)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # stage buffers inside the workspace-equivalent set (same composition as fm_mixer_prefill)
    d = shape
    q_in = torch.empty((M, d.d_model), dtype=torch.int8, device=dev)
    sx_in = torch.empty(M, dtype=torch.float32, device=dev)
    z = torch.empty((M, d.d_inner), dtype=torch.float32, device=dev)
    xbc = torch.empty((M, d.conv_ch), dtype=torch.int8, device=dev)
    dtr = torch.empty((M, d.nheads), dtype=torch.float32, device=dev)
    xo = torch.empty((M, d.conv_ch), dtype=torch.int8, device=dev)
    y = torch.empty((M, d.d_inner), dtype=torch.int32, device=dev)
    q_out = torch.empty((M, d.d_inner), dtype=torch.int8, device=dev)
    sx_out = torch.empty(M, dtype=torch.float32, device=dev)
    sws = torch.empty(lib.scan_workspace_bytes(d, B, T), dtype=torch.uint8, device=dev)
    launches_per_step = 7 * n_layers  # FWHT+quant, in_proj, conv, scan prep, scan, gate, out_proj

    def step(scan_events=None):
        src = x0
        for i, Ly in enumerate(stack.layers):
            lib.hadamard_quant(src, d.d_model, Ly.prenorm_w, 1, mode, Ly.static_amax, q_in, sx_in)
            lib.in_proj(q_in, sx_in, Ly.w_in_q, Ly.w_in_s, d, Ly.exps, z, xbc, dtr)
            lib.conv1d_pot(xbc, B, T, d, Ly.conv_wq, Ly.conv_bq, Ly.exps, None, xo)
            if scan_events is not None:
                scan_events[i][0].record(stream)
            lib.ssm_scan_pot(xo, dtr, B, T, d, Ly.dt_bias, Ly.A_q, Ly.D_q, Ly.exps, None, y, sws)
            if scan_events is not None:
                scan_events[i][1].record(stream)
            lib.gate_norm_quant(y, z, d, Ly.exps, Ly.norm_w, 1, mode, Ly.static_amax[1:], q_out,
                                sx_out)
            lib.w8a8_gemm(q_out, sx_out, Ly.w_out_q, Ly.w_out_s, r, residual=src)
            src = r

    # the stage-by-stage step must equal the public fm_mixer_prefill path
    step()
    ref = x0.clone()
    stack.prefill_(ref, ws=ws)
    torch.cuda.synchronize()
    lib.sync_status()
    if not torch.equal(ref, r):
        raise SystemExit("bench: stage-by-stage step differs from fm_mixer_prefill")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(n_layers)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for k in range(args.steps):
        flush.zero_()
        torch.cuda.nvtx.range_push("bench_step")
        ev[k][0].record(stream)
        step(sev[k])
        ev[k][1].record(stream)
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    lib.sync_status()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    scan_ms = [a.elapsed_time(b) for row in sev for a, b in row]
    total_ms = sum(step_ms)
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * B * T * args.steps / (total_ms / 1000.0)

    # roofline of the dominant kernel (the sequential fixed-point scan, integer-ALU bound)
    peaks = measured_peaks()
    cells = B * d.nheads * d.headdim * d.d_state * T
    scan_avg_s = statistics.mean(scan_ms) / 1000.0
    achieved = cells * SCAN_OPS_PER_CELL / scan_avg_s / 1e12
    sm_mhz_peak = (peaks or {}).get("sm_max_mhz", 1965.0)
    alu_peak = 148 * 4 * 32 * sm_mhz_peak * 1e6 / 1e12
    roofline = {"bound": "alu", "kernel": "fm_ssm_scan_pot (k_scan_prep + k_scan_seq)",
                "achieved": achieved,
                "peak": alu_peak, "unit": "Tops/s (int32)", "frac": achieved / alu_peak,
                "traffic": None,
                "peak_basis": f"148 SMs x 4 SMSPs x 32 lanes x 1 int op/clk x {sm_mhz_peak:.0f} MHz",
                "avg_launch_us": 1e6 * scan_avg_s,
                "share_of_step": sum(scan_ms) / sum(step_ms)}

    # end to end through the public API: pinned host input -> device, 24 x
    # fm_mixer_prefill, device -> pinned host output, every step
    xh = torch.from_numpy(x_host).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(x0)

    def e2e_step():
        xd.copy_(xh, non_blocking=True)
        stack.prefill_(xd, ws=ws)
        oh.copy_(xd, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    lib.sync_status()
    if not torch.equal(oh, ref.cpu()):
        raise SystemExit("bench: end-to-end output differs from the device-resident step")
    e2e_t = torch.tensor([sum(e2e_ms)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
    e2e_value = world * B * T * args.steps / (float(e2e_t.item()) / 1000.0)
    nbytes = x_host.nbytes

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_oracle_sample(shape, n_layers, args.mode)
        line = {"metric": "W8A8 Mamba2 prefill tokens/s", "value": value, "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "int8 GEMM (int32 acc) + int32 fixed point",
                "data": "synthetic (seeded outlier-injected N(0,1), random-init weights)",
                "config": config_block(args, shape, n_layers, B, T),
                "roofline": roofline, "cpu_baseline": cpu, "clocks": clk,
                "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
                        "d2h_bytes_per_step": nbytes},
                "gpu_launches": launches_per_step * args.steps,
                "scan_ms_per_layer": statistics.mean(scan_ms)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
