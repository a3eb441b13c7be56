#!/usr/bin/env python3
"""Benchmark: W8A8 / power-of-two Mamba2 tokens/s on one B200 per rank.

Default workload (the headline line), stack130m_24l_b1_t2048: the
Mamba2-130M-shaped stack -- 24 pre-normed residual mixer layers (d_model 768,
d_inner 1536, 24 heads of 64, d_state 128), batch 1, 2048 tokens,
outlier-injected N(0,1) inputs, random-init weights, activation scales
dynamic per token (--mode static: calibrated), power-of-two exponents
calibrated on the GPU from 16 seeded sequences of 512 tokens.  One step = one
prefill of the whole stack over the batch.

Other workloads (--workload):
  mixer130m_b1_t256       one bare 130M mixer layer, batch 1, 256 tokens
  gemm2p7b_inproj         FWHT + int8 quantisation + the in_proj W8A8 GEMM at
                          the 2.7B shapes (K 2560, N 10576), M = --gemm-m
                          (2048 | 8192 | 32768), fp32 dequantised output
  stack2p7b_64l_b2_t4096  64 2.7B-shaped stack layers, batch 2, 4096 tokens
  decode2p7b_64l_b64      one decode step of 64 sequences through the 64
                          2.7B-shaped layers, states from a 512-token prefill

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload W] [--mode dynamic|static]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

Under torchrun each rank runs an independent replica on its own GPU (the
sequences of a batch are independent problems; no collective on the data
path): weak scaling; the step time is the max over ranks.  Prints one JSON
line on rank 0.
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

METRIC = "W8A8 Mamba2 prefill tokens/s (130M/2.7B shapes); int8 TOPS & HBM GB/s vs peak"
DEFAULT_WORKLOAD = "stack130m_24l_b1_t2048"
WORKLOAD_NAMES = ["mixer130m_b1_t256", "stack130m_24l_b1_t2048", "gemm2p7b_inproj",
                  "stack2p7b_64l_b2_t4096", "decode2p7b_64l_b64"]
OUTLIER_SEED = 4242
L2_FLUSH_BYTES = 512 << 20
# Algorithmic work of one state-cell update of the scan: decay multiply,
# rounding shift, dt*x*B multiply-add, clamp (2), C*h multiply-accumulate.
SCAN_OPS_PER_CELL = 6
SSD_CHUNK = 128  # tokens per chunk of the chunked scan mode
# fp32 work of one state-cell update of the LQ scan: (dt x) B, the decay
# multiply-add, the C h multiply-add
LQ_FLOPS_PER_CELL = 5
NOMINAL_INT8_OVER_BF16 = 2.0  # 4.5 / 2.25 PFLOP/s dense
CPU_SAMPLE_MIN_S = 10.0
# tokens of the all-core oracle sample (per process; one layer)
CPU_ALLCORE_TOKENS = 512


# DRAM bytes (read + write) per launch of a roofline kernel, from one-pass ncu
# captures of the current kernels (profiles/dram_traffic_roofline_kernels.md);
# None where no capture of the kernel in that configuration exists.
DRAM_TRAFFIC = {
    # 130M stack, B 1, T 2048, static exponents, the int32 state, the layer
    # loop the roofline is timed on: k_scan_prep 3,885,056 + 0 and
    # k_scan_seq<4, 4, 32> 19,665,920 + 0 (the x codes staged as int8)
    ("fm_ssm_scan_pot (k_scan_prep + k_scan_seq)", "stack130m_24l_b1_t2048", "31,0", "static"):
        23550976,
    # 2.7B decode, B 64: k_scan_step 168,172,672 + 108,671,744 (mean of the
    # two layers' launches; u evaluated once per lane)
    ("fm_ssm_scan_pot, T = 1 (k_scan_step)", "decode2p7b_64l_b64", "31,0", "static"): 276844416,
    # in_proj GEMM at M = 32768: 306,106,112 + 1,339,252,992
    ("fm_w8a8_gemm (k_gemm_i8_persist, tcgen05 kind::i8)", "gemm2p7b_inproj", 32768): 1645359104,
}


def dram_traffic(kernel: str, args):
    if args.workload == "gemm2p7b_inproj":
        return DRAM_TRAFFIC.get((kernel, args.workload, args.gemm_m))
    if getattr(args, "lq", False) or getattr(args, "scan_mode", "seq") != "seq":
        return None
    return DRAM_TRAFFIC.get((kernel, args.workload, args.state_spec,
                             getattr(args, "xbc_exponents", "static")))


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOAD_NAMES)
    ap.add_argument("--gemm-m", type=int, default=32768, choices=[2048, 8192, 32768])
    ap.add_argument("--mode", default="dynamic", choices=["dynamic", "static"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scan-tile", default=None,
                    help="npt,pc,tch of the sequential scan kernel (a compiled variant)")
    ap.add_argument("--scan-mode", default="seq", choices=["seq", "ssd"],
                    help="seq: the sequential fixed-point scan (the method); ssd: the chunked "
                         "tensor-core scan mode (its own error budget)")
    ap.add_argument("--state-spec", default="31,0", choices=["31,0", "16,7"],
                    help="scan state word and increment guard bits: 31,0 the method as built, "
                         "16,7 the narrow state with the guard-bit increment")
    ap.add_argument("--gemm-tile", type=int, default=0, choices=[0, 128, 256],
                    help="tile width of the persistent GEMM (0: chosen by the grid)")
    ap.add_argument("--lq-cpw", type=int, default=0, choices=[0, 1, 2, 4],
                    help="channels per warp of the LQ scan (0: chosen by the grid)")
    ap.add_argument("--gemm-cluster", default="off", choices=["on", "off"],
                    help="decode-size GEMMs with fewer tiles than SMs split K over a "
                         "thread-block cluster (off: the library's default)")
    ap.add_argument("--pdl", default="on", choices=["on", "off"],
                    help="programmatic dependent launch of the library's kernels (on: the "
                         "library's default)")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed steps one by one instead of replaying them as one "
                         "captured CUDA graph")
    ap.add_argument("--xbc-exponents", default="static", choices=["static", "token"],
                    help="conv-output exponents: static per head / B / C (as built) or per token")
    ap.add_argument("--lq", action="store_true",
                    help="the FastMamba-LQ variant of a prefill workload (fp32 conv, scan, gate)")
    ap.add_argument("--modes", default="auto",
                    help="comma list of sub-records measured after the headline, each a full "
                         "timed run of the same workload in another mode: static, ssd, state16, "
                         "lq; 'auto' = all four for the default workload, none otherwise; 'none'")
    ap.add_argument("--chunks", type=int, default=0,
                    help="runs per sequence of a stack prefill pipelined through the layers by "
                         "fm_stack_prefill (0: 4 for a single-sequence stack prefill with the "
                         "sequential scan, else 1; 1: the layer loop)")
    ap.add_argument("--layers", type=int, default=None,
                    help="profiling only: run the first N layers of a stack workload")
    return ap.parse_args(argv)


SUB_MODES = ("static", "ssd", "state16", "candidate", "lq")


def sub_modes(args) -> list:
    if args.modes == "none" or args.impl == "reference":
        return []
    if args.modes == "auto":
        return list(SUB_MODES) if args.workload == DEFAULT_WORKLOAD and not args.layers else []
    out = [m for m in args.modes.split(",") if m]
    bad = set(out) - set(SUB_MODES)
    if bad:
        raise SystemExit(f"bench: unknown --modes {sorted(bad)}")
    return out


def variant_args(args, mode: str):
    """The arguments of one sub-record: the headline's, with one mode changed."""
    v = argparse.Namespace(**vars(args))
    if mode == "static":
        v.mode = "static"
    elif mode == "ssd":
        v.scan_mode = "ssd"
    elif mode == "state16":
        v.state_spec = "16,7"
    elif mode == "candidate":  # per-token exponents, 16-bit state, guard-bit increment
        v.state_spec = "16,7"
        v.xbc_exponents = "token"
    elif mode == "lq":
        v.lq = True
    return v


def n_layers(args) -> int:
    w = S.WORKLOADS[args.workload]
    return args.layers if args.layers else w.get("layers", 1)


def stack_chunks(args) -> int:
    """Runs per sequence of the pipelined stack prefill (1: the layer loop).
    By default 4 for a single sequence, whose scan alone leaves SM
    sub-partitions idle (measured, 130M stack: 302.4 k tokens/s as the layer
    loop, 335.7 k with 2 runs, 340.3 k with 4 runs and the 16-step scan chunks
    the library then picks; at B = 2 the 2.7B scan fills the GPU and
    pipelining gained nothing).  The FastMamba-LQ variant,
    single-token steps and the chunked scan mode (whose state crosses a call
    boundary as int32, so a split prefill is not the one-pass result) run the
    layer loop."""
    w = S.WORKLOADS.get(args.workload, {})
    if (w.get("layers", 1) <= 1 or w.get("seqlen", 1) <= 1 or getattr(args, "lq", False) or
            getattr(args, "scan_mode", "seq") == "ssd"):
        return 1
    if getattr(args, "chunks", 0) > 0:
        return args.chunks
    return 4 if w.get("batch", 1) == 1 else 1


def stack_runs(T: int, n: int) -> tuple:
    """(runs, tokens per run) of one sequence of T tokens under
    fm_stack_prefill(n_chunks = n): ceil(T / n) tokens rounded up to a
    multiple of 32 per run, the last run the remainder."""
    tc = min(T, -(-(-(-T // n)) // 32) * 32)
    return -(-T // tc), tc


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return None


def workload_tokens(args) -> int:
    """Tokens one step processes on one rank."""
    w = S.WORKLOADS[args.workload]
    if args.workload == "gemm2p7b_inproj":
        return args.gemm_m
    return w["batch"] * w["seqlen"]


def config_block(args) -> dict:
    w = S.WORKLOADS[args.workload]
    d = w["shape"]
    c = {"workload": args.workload, "d_model": d.d_model, "d_inner": d.d_inner,
         "nheads": d.nheads, "headdim": d.headdim, "d_state": d.d_state, "act_quant": args.mode,
         "hadamard": "block 256", "l2": "flushed between timed steps (512 MiB write)",
         "parallelism": f"replica x{args.gpus}"}
    if args.workload == "gemm2p7b_inproj":
        c.update(M=args.gemm_m, N=d.n_in, K=d.d_model)
    else:
        c.update(layers=n_layers(args), batch=w["batch"], seq_len=w["seqlen"],
                 calibration=f"{S.CALIB_SEQS} seeded sequences x "
                             f"{min(w.get('prefill_len', w['seqlen']), S.CALIB_MAX_LEN)} tokens "
                             "(GPU, stage by stage)",
                 scan_tile=args.scan_tile or "4,auto,32", scan_mode=args.scan_mode,
                 state_spec=args.state_spec,
                 xbc_exponents=getattr(args, "xbc_exponents", "static"))
        ch = stack_chunks(args)
        if ch == 1 and w.get("layers", 1) > 1 and w["seqlen"] > 1:
            c.update(pipeline="none: the layer loop on one stream")
        if ch > 1:
            runs, tc = stack_runs(w["seqlen"], ch)
            c.update(pipeline=f"fm_stack_prefill, n_chunks {ch}: {runs} runs of up to {tc} "
                              "tokens per sequence, each on its own stream, waiting only for "
                              "the previous run's conv and scan of the same layer"
                              + ("; the runs' scans stage 16-step chunks where the grid is too "
                                 "small for 8 channels per CTA" if not args.scan_tile else ""))
        if getattr(args, "lq", False):
            c.update(variant="FastMamba-LQ (W8A8 linears; fp32 conv, scan, gate)")
        if "prefill_len" in w:
            c.update(prefill_len=w["prefill_len"], step="one decode token per sequence")
    return c


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
        return parse_clock_samples(out)


def parse_clock_samples(text: str) -> dict:
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in text.strip().splitlines():
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


# ---------------------------------------------------------------- CPU oracle samples
class OracleSample:
    """The oracle as it stands (single-threaded C composed by numpy) on a
    bounded sample of a workload: one layer over a slice of its tokens (the
    oracle's cost is linear in tokens and in layers), or a slice of the GEMM's
    rows.  value = sample tokens / (sample seconds x the workload's layers)."""

    def __init__(self, workload: str, mode: str, gemm_m: int = 32768, max_tokens: int = 0):
        import oracle as O
        self.O, self.workload = O, workload
        w = S.WORKLOADS[workload]
        shape = w["shape"]
        omode = O.DYNAMIC if mode == "dynamic" else O.STATIC
        n_out, scale = w["n_outliers"], w["outlier_scale"]
        self.layers = w.get("layers", 1)
        if workload == "gemm2p7b_inproj":
            rows = 128 if not max_tokens else min(128, max_tokens)
            self.x = S.activations(1, rows, shape.d_model, seed=11, n_outliers=n_out,
                                   outlier_scale=scale, outlier_seed=OUTLIER_SEED)[0]
            self.wq, self.sw = O.prepare_linear(S.layer_params(shape, 1000)["w_in"])
            self.tokens = rows
            self.desc = f"{rows} of the {gemm_m} rows (FWHT + quantisation + in_proj GEMM)"
            self.run_fn = self._gemm
            return
        prenorm = self.layers > 1
        L = O.prepare_layer(S.layer_params(shape, 1000), shape, rotate=1, mode=omode,
                            prenorm=prenorm)
        xcal = S.calibration_batch(shape.d_model, 64, n_out, scale, OUTLIER_SEED, n_seqs=1)
        O.calibrate_layer(L, xcal, residual=prenorm)
        self.L, self.prenorm = L, prenorm
        if workload == "decode2p7b_64l_b64":
            Bs = w["batch"]
            self.x = S.activations(Bs, 1, shape.d_model, seed=5, n_outliers=n_out,
                                   outlier_scale=scale, outlier_seed=OUTLIER_SEED)
            self.cs = np.zeros((Bs, 3, shape.conv_ch), np.int8)
            self.ss = np.zeros((Bs, shape.nheads, shape.headdim, shape.d_state), np.int32)
            self.tokens = Bs
            self.desc = f"one decode step of 1 of {self.layers} layers for all {Bs} sequences"
            self.run_fn = self._decode
            return
        B, T = w["batch"], w["seqlen"]
        Ts = min(B * T, 2048 if shape.d_model <= 1024 else 256)  # ~5-10 s a run
        if max_tokens:
            Ts = min(Ts, max_tokens)
        self.x = S.activations(1, Ts, shape.d_model, seed=1, n_outliers=n_out,
                               outlier_scale=scale, outlier_seed=OUTLIER_SEED)
        self.tokens = Ts
        self.desc = f"1 of {self.layers} layers over {Ts} of the {B}x{T} tokens"
        self.run_fn = self._prefill

    def _gemm(self):
        q, sx = self.O.hadamard_quant(self.x)
        self.O.dequant(self.O.gemm_i8(q, self.wq), sx, self.sw)

    def _prefill(self):
        self.O.mixer_prefill(self.L, self.x, residual=self.prenorm)

    def _decode(self):
        self.O.mixer_prefill(self.L, self.x, residual=True, conv_state=self.cs,
                             ssm_state=self.ss)

    def run(self) -> float:
        t0 = time.perf_counter()
        self.run_fn()
        return time.perf_counter() - t0

    def value(self, seconds: float) -> float:
        return self.tokens / (seconds * self.layers)

    def measure(self, min_seconds: float = CPU_SAMPLE_MIN_S, max_runs: int = 16) -> dict:
        secs = []
        while sum(secs) < min_seconds and len(secs) < max_runs:
            secs.append(self.run())
        return self.describe(statistics.mean(secs), len(secs))

    def describe(self, seconds: float, runs: int) -> dict:
        scaled = "" if self.layers == 1 else f", scaled to {self.layers} layers"
        return {"value": self.value(seconds), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": f"{self.desc}{scaled}; {runs} run(s), {seconds:.2f} s each"}


def _oracle_worker(workload, mode, gemm_m, max_tokens, runs, ready, go, out):
    """One host core's share of the all-core oracle baseline (a spawned
    process): set up the sample, wait for the common start, time `runs` runs."""
    o = OracleSample(workload, mode, gemm_m, max_tokens)
    o.run()
    ready.wait()
    go.wait()
    secs = [o.run() for _ in range(runs)]
    out.put((secs, o.tokens, o.layers, o.desc))


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_all_cores(workload, mode, gemm_m, max_tokens, runs, warmup=0):
    """The oracle as it stands, one single-threaded process per host core, all
    running the same bounded sample at once (spawned: no CUDA state is
    inherited).  Returns (tokens/s of the whole host, per-run wall seconds,
    cores, tokens of one process's sample, sample description)."""
    import multiprocessing as mp
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[v] = "1"
    n = host_cores()
    ctx = mp.get_context("spawn")
    ready, go, out = ctx.Barrier(n + 1), ctx.Event(), ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker,
                         args=(workload, mode, gemm_m, max_tokens, warmup + runs, ready, go, out))
             for _ in range(n)]
    for p in procs:
        p.start()
    ready.wait()
    t0 = time.perf_counter()
    go.set()
    res = [out.get() for _ in range(n)]
    wall = time.perf_counter() - t0
    for p in procs:
        p.join()
    _, tokens, layers, desc = res[0]
    # every process times its runs; the slowest process's timed runs set the
    # host's rate (the warm-up runs share the common window but are not counted)
    timed = max(sum(r[0][warmup:]) for r in res)
    value = n * runs * tokens / (timed * layers)
    return value, timed / runs, n, tokens, desc


def cpu_baseline(args) -> dict:
    """Rank 0, one GPU: the oracle on the host cores.  `value`/`cores` are
    the all-core figure (one oracle process per core); the single-threaded
    oracle's own figure is kept beside it."""
    one = OracleSample(args.workload, args.mode, args.gemm_m).measure()
    val, per_run, n, _, desc = oracle_all_cores(args.workload, args.mode, args.gemm_m,
                                                CPU_ALLCORE_TOKENS, runs=1)
    layers = S.WORKLOADS[args.workload].get("layers", 1)
    scaled = "" if layers == 1 else f", scaled to {layers} layers"
    return {"value": val, "unit": "tokens/s", "cores": n, "kind": "oracle",
            "sample": f"{n} processes (one per host core) each running {desc}{scaled}, "
                      f"concurrently; {per_run:.2f} s per run",
            "single_thread": one}


def run_reference(args):
    """--impl reference: the CPU oracle as it stands on this host's cores
    (rank 0 only).  One timed step = one bounded sample of the workload, run
    concurrently by one oracle process per core; `value` extrapolates the
    sample to the whole workload (the oracle's cost is linear in layers and
    tokens: factor `extrapolation`), and `ms_per_step` is the wall time of
    the sample that was actually timed."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    steps = max(1, args.steps)
    value, per_run, n, o_tokens, desc = oracle_all_cores(args.workload, args.mode, args.gemm_m,
                                                         CPU_ALLCORE_TOKENS, runs=steps,
                                                         warmup=args.warmup)
    layers = S.WORKLOADS[args.workload].get("layers", 1)
    factor = layers * workload_tokens(args) / (n * o_tokens)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * per_run, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8/int32 fixed point (CPU oracle)",
            "data": "synthetic", "config": config_block(args),
            "step": f"one sample per host core: {desc}, {n} cores",
            "extrapolation": {"factor": factor,
                              "basis": "value = sample tokens x cores / (sample wall x layers); "
                                       "one full workload step is `factor` times the timed "
                                       "sample's work"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": n, "kind": "oracle",
                             "sample": f"{desc}, one process per core, {steps} timed runs"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU workloads
def _stage_buffers(torch, d, M, dev):
    e = lambda *sh, dt: torch.empty(sh, dtype=dt, device=dev)
    return dict(q_in=e(M, d.d_model, dt=torch.int8), sx_in=e(M, dt=torch.float32),
                z=e(M, d.d_inner, dt=torch.float32), xbc=e(M, d.conv_ch, dt=torch.int8),
                dtr=e(M, d.nheads, dt=torch.float32), xo=e(M, d.conv_ch, dt=torch.int8),
                y=e(M, d.d_inner, dt=torch.int32), q_out=e(M, d.d_inner, dt=torch.int8),
                sx_out=e(M, dt=torch.float32), e_tok=e(M, d.nheads + 2, dt=torch.int32))


def _gemm_workspace(torch, lib, d, M, dev):
    """The split-K workspace of a layer's two GEMMs at M rows (None when neither
    splits) and the extra launches (one epilogue kernel per split GEMM)."""
    n_in = lib.gemm_workspace_bytes(M, d.n_in, d.d_model)
    n_out = lib.gemm_workspace_bytes(M, d.d_model, d.d_inner)
    n = max(n_in, n_out)
    ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    return ws, int(n_in > 0) + int(n_out > 0)


class StackWorkload:
    """Prefill of a stack (or of one bare mixer layer).  The timed step calls
    the stage entry points in the order fm_mixer_prefill composes them (checked
    bit for bit against it), with events around each layer's scan."""

    launches_per_layer = 7  # FWHT+quant, in_proj, conv, scan prep, scan, gate, out_proj
    chunks = 1  # runs per sequence of the pipelined stack prefill (1: the layer loop)

    def __init__(self, args, torch, lib, dev, rank):
        from quantized_state_space_mamba2_b200.model import DeviceLayer, DeviceStack
        self.torch, self.lib, self.dev = torch, lib, dev
        w = S.WORKLOADS[args.workload]
        self.shape = d = w["shape"]
        self.n_layers = n_layers(args)
        self.B, self.T = w["batch"], w["seqlen"]
        self.stack_mode = w.get("layers", 1) > 1
        self.mode = lib.FM_DYNAMIC if args.mode == "dynamic" else lib.FM_STATIC
        params = (S.layer_params(d, 1000 + l) for l in range(self.n_layers))
        xcal = torch.from_numpy(S.calibration_batch(d.d_model, self.T, w["n_outliers"],
                                                    w["outlier_scale"], OUTLIER_SEED)).to(dev)
        if self.stack_mode:
            self.stack = DeviceStack(list(params), d, rotate=1, mode=self.mode, device=dev)
            self.layers = self.stack.layers
            self.stack.calibrate(xcal)
        else:
            self.layers = [DeviceLayer(next(params), d, rotate=1, mode=self.mode, device=dev)]
            self.layers[0].calibrate(xcal)
        del xcal
        self.x_host = S.activations(self.B, self.T, d.d_model, seed=1 + rank,
                                    n_outliers=w["n_outliers"], outlier_scale=w["outlier_scale"],
                                    outlier_seed=OUTLIER_SEED)
        self.x0 = torch.from_numpy(self.x_host).to(dev)
        self.r = torch.empty_like(self.x0)
        M = self.B * self.T
        self.ws = self.layers[0].workspace(self.B, self.T)
        self.ssd = getattr(args, "scan_mode", "seq") == "ssd" and self.T > 1
        self.tok = getattr(args, "xbc_exponents", "static") == "token"
        nb = (lib.ssd_workspace_bytes if self.ssd else
              lib.scan_workspace_bytes_tok if self.tok else lib.scan_workspace_bytes)(d, self.B,
                                                                                     self.T)
        self.sws = torch.empty(nb, dtype=torch.uint8, device=dev)
        self.buf = _stage_buffers(torch, d, M, dev)
        self.tokens = M
        self.gws, extra = _gemm_workspace(torch, lib, d, M, dev)
        # the chunked scan is three kernels where the sequential one is two
        self.launches = (self.launches_per_layer + extra + (1 if self.ssd else 0)) * self.n_layers
        # the timed step: the stack pipelined over time by fm_stack_prefill
        # (chunks > 1), else the stage-by-stage layer loop below
        self.chunks = stack_chunks(args) if self.stack_mode else 1
        if self.chunks > 1:
            runs, tc = stack_runs(self.T, self.chunks)
            self.pws = self.stack.stack_workspace(self.B, self.T, self.chunks)
            _, extra_run = _gemm_workspace(torch, lib, d, tc, dev)
            # every run carries conv state, so a run of more than one token
            # adds the conv-state update; a one-token run's scan is the single
            # step (no prep) and its conv writes the state itself
            last = self.T - (runs - 1) * tc
            per_run = lambda tn: (self.launches_per_layer + extra_run +
                                  ((1 if self.ssd else 0) + 1 if tn > 1 else -1))
            self.launches = (per_run(tc) * (runs - 1) + per_run(last)) * self.n_layers * self.B

    def states(self, i):
        return None, None

    def step(self, ev=None, staged=False):
        """One step.  Pipelined (chunks > 1, unless staged): x0 copied to r, then
        one fm_stack_prefill call in place.  Staged: the stage entry points in
        fm_mixer_prefill's order, layer by layer, on the current stream, with
        the events ev[i] around layer i's scan."""
        if self.chunks > 1 and not staged:
            self.r.copy_(self.x0)
            self.stack.prefill_pipelined_(self.r, n_chunks=self.chunks, ws=self.pws)
            return
        lib, d, B, T, b = self.lib, self.shape, self.B, self.T, self.buf
        stream = self.torch.cuda.current_stream(self.dev)
        src = self.x0
        for i, Ly in enumerate(self.layers):
            cs, ss = self.states(i)
            lib.hadamard_quant(src, d.d_model, Ly.prenorm_w, 1, self.mode, Ly.static_amax,
                               b["q_in"], b["sx_in"])
            lib.in_proj(b["q_in"], b["sx_in"], Ly.w_in_q, Ly.w_in_s, d, Ly.exps, b["z"], b["xbc"],
                        b["dtr"], ws=self.gws)
            if self.tok:
                lib.conv1d_pot_tok(b["xbc"], B, T, d, Ly.conv_wq, Ly.conv_bq, Ly.exps, cs, b["xo"],
                                   b["e_tok"])
            else:
                lib.conv1d_pot(b["xbc"], B, T, d, Ly.conv_wq, Ly.conv_bq, Ly.exps, cs, b["xo"])
            if ev is not None:
                ev[i][0].record(stream)
            if self.tok:
                lib.ssm_scan_pot_tok(b["xo"], b["dtr"], B, T, d, Ly.dt_bias, Ly.A_q, Ly.D_q,
                                     Ly.exps, b["e_tok"], ss, b["y"], self.sws)
            else:
                scan = lib.ssd_scan if self.ssd else lib.ssm_scan_pot
                scan(b["xo"], b["dtr"], B, T, d, Ly.dt_bias, Ly.A_q, Ly.D_q, Ly.exps, ss, b["y"],
                     self.sws)
            if ev is not None:
                ev[i][1].record(stream)
            lib.gate_norm_quant(b["y"], b["z"], d, Ly.exps, Ly.norm_w, 1, self.mode,
                                Ly.static_amax[1:], b["q_out"], b["sx_out"])
            lib.w8a8_gemm(b["q_out"], b["sx_out"], Ly.w_out_q, Ly.w_out_s, self.r,
                          residual=src if self.stack_mode else None, ws=self.gws)
            src = self.r

    def output(self):
        return self.r

    def public_output(self):
        """The same input through the public per-layer entry point."""
        if self.stack_mode:
            out = self.x0.clone()
            self.stack.prefill_(out, ws=self.ws)
            return out
        return self.layers[0].prefill(self.x0, ws=self.ws)

    def e2e_setup(self):
        torch = self.torch
        self.xh = torch.from_numpy(self.x_host).pin_memory()
        self.oh = torch.empty_like(self.xh).pin_memory()
        self.xd = torch.empty_like(self.x0)
        self.od = torch.empty_like(self.x0)
        self.h2d_bytes = self.d2h_bytes = self.x_host.nbytes

    def e2e_step(self):
        if self.stack_mode and self.chunks > 1:
            # one call with the batch in host memory: each run's input and
            # output copies travel on the run's stream, overlapping the others
            self.stack.prefill_host(self.xh, self.oh, self.xd, n_chunks=self.chunks, ws=self.pws)
            return
        self.xd.copy_(self.xh, non_blocking=True)
        if self.stack_mode:
            self.stack.prefill_(self.xd, ws=self.ws)
            self.oh.copy_(self.xd, non_blocking=True)
        else:
            self.layers[0].prefill(self.xd, out=self.od, ws=self.ws)
            self.oh.copy_(self.od, non_blocking=True)

    def e2e_matches(self, ref) -> bool:
        return self.torch.equal(self.oh, ref.cpu())

    def roofline(self, dom_ms, peaks):
        d = self.shape
        if self.ssd:
            # per token and head: C.B^T Q ds, M.X Q hd, state hd ds, inter ds hd MACs
            macs = self.B * self.T * d.nheads * (SSD_CHUNK * d.d_state + SSD_CHUNK * d.headdim +
                                                 2 * d.headdim * d.d_state)
            achieved = 2 * macs / (dom_ms / 1e3) / 1e12
            peak = (peaks or {}).get("bf16_tflops", 1590.0)
            return {"bound": "tensor", "kernel": "fm_ssd_scan (k_ssd_state + k_ssd_pass + k_ssd_out)",
                    "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                    "traffic": None,
                    "peak_basis": "measured bf16 dense (burst); the C.B^T quarter runs as int8",
                    "algorithmic": f"2 x {macs} MACs per launch"}
        cells = self.B * d.nheads * d.headdim * d.d_state * self.T
        achieved = cells * SCAN_OPS_PER_CELL / (dom_ms / 1e3) / 1e12
        mhz = (peaks or {}).get("sm_max_mhz", 1965.0)
        peak = 148 * 4 * 32 * mhz * 1e6 / 1e12
        return {"bound": "alu", "kernel": "fm_ssm_scan_pot (k_scan_prep + k_scan_seq)",
                "achieved": achieved, "peak": peak, "unit": "Tops/s (int32)",
                "frac": achieved / peak, "traffic": None,
                "peak_basis": f"derived: 148 SMs x 4 SMSPs x 32 lanes x 1 int op/clk x "
                              f"{mhz:.0f} MHz (measured max SM clock)",
                "algorithmic": f"{SCAN_OPS_PER_CELL} int ops per state-cell update x {cells} "
                               "updates per launch"}


class DecodeWorkload(StackWorkload):
    """One decode step of B sequences through the whole stack; conv and SSM
    states come from a seeded prefill and advance by one token per step."""

    launches_per_layer = 6  # FWHT+quant, in_proj, conv (+ conv-state update), scan step, gate, out_proj

    def __init__(self, args, torch, lib, dev, rank):
        from quantized_state_space_mamba2_b200.model import DeviceStack
        self.torch, self.lib, self.dev = torch, lib, dev
        w = S.WORKLOADS[args.workload]
        self.shape = d = w["shape"]
        self.n_layers, self.B, self.T = n_layers(args), w["batch"], 1
        self.stack_mode = True
        self.ssd = False  # a single-token step always runs the sequential scan step
        self.tok = getattr(args, "xbc_exponents", "static") == "token"
        self.mode = lib.FM_DYNAMIC if args.mode == "dynamic" else lib.FM_STATIC
        P = w["prefill_len"]
        self.stack = DeviceStack([S.layer_params(d, 1000 + l) for l in range(self.n_layers)], d,
                                 rotate=1, mode=self.mode, device=dev)
        self.layers = self.stack.layers
        xcal = torch.from_numpy(S.calibration_batch(d.d_model, P, w["n_outliers"],
                                                    w["outlier_scale"], OUTLIER_SEED)).to(dev)
        self.stack.calibrate(xcal)
        del xcal
        self.st = [L.new_states(self.B) for L in self.layers]
        pre = torch.from_numpy(S.activations(self.B, P, d.d_model, seed=77 + rank,
                                             n_outliers=w["n_outliers"],
                                             outlier_scale=w["outlier_scale"],
                                             outlier_seed=OUTLIER_SEED)).to(dev)
        self.stack.prefill_(pre, states=self.st)
        del pre
        torch.cuda.synchronize()
        self.st0 = [(c.clone(), s.clone()) for c, s in self.st]
        self.x_host = S.activations(self.B, 1, d.d_model, seed=5 + rank,
                                    n_outliers=w["n_outliers"], outlier_scale=w["outlier_scale"],
                                    outlier_seed=OUTLIER_SEED)
        self.x0 = torch.from_numpy(self.x_host).to(dev)
        self.r = torch.empty_like(self.x0)
        self.ws = self.layers[0].workspace(self.B, 1)
        self.sws = torch.empty(lib.scan_workspace_bytes(d, self.B, 1), dtype=torch.uint8,
                               device=dev)
        self.buf = _stage_buffers(torch, d, self.B, dev)
        self.tokens = self.B
        self.gws, extra = _gemm_workspace(torch, lib, d, self.B, dev)
        self.launches = (self.launches_per_layer + extra) * self.n_layers

    def states(self, i):
        return self.st[i]

    def restore(self):
        for (c, s), (c0, s0) in zip(self.st, self.st0):
            c.copy_(c0)
            s.copy_(s0)

    def public_output(self):
        self.restore()
        out = self.x0.clone()
        for (cs, ss), Ly in zip(self.st, self.layers):
            Ly.decode(out, cs, ss, residual=True, out=out, ws=self.ws)
        self.torch.cuda.synchronize()
        self.restore()
        return out

    def e2e_step(self):
        self.xd.copy_(self.xh, non_blocking=True)
        for (cs, ss), Ly in zip(self.st, self.layers):
            Ly.decode(self.xd, cs, ss, residual=True, out=self.xd, ws=self.ws)
        self.oh.copy_(self.xd, non_blocking=True)

    def e2e_matches(self, ref) -> bool:
        return True  # the states have advanced; the public path was checked before timing

    def roofline(self, dom_ms, peaks):
        d = self.shape
        esz = 2 if self.lib.STATE_BITS == 16 else 4      # int16 state under the narrow spec
        state = self.B * d.nheads * d.headdim * d.d_state * esz
        io = self.B * (d.conv_ch + 4 * d.nheads + 4 * d.d_inner)
        achieved = (2 * state + io) / (dom_ms / 1e3) / 1e9
        peak = (peaks or {}).get("hbm_gbs", 6548.0)
        return {"bound": "hbm", "kernel": "fm_ssm_scan_pot, T = 1 (k_scan_step)",
                "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": None, "peak_basis": "measured copy bandwidth (hbm_gbs)",
                "algorithmic": f"state read + write {2 * state} B + x, B, C, dt, y {io} B "
                               "per launch"}


class GemmWorkload:
    """FWHT + quantisation of X [M, 2560] and the in_proj W8A8 GEMM
    (N = 10576) with an fp32 dequantised output, at the 2.7B shapes; events
    around the GEMM."""

    n_layers = 1

    def __init__(self, args, torch, lib, dev, rank):
        self.torch, self.lib, self.dev = torch, lib, dev
        w = S.WORKLOADS["gemm2p7b_inproj"]
        d = w["shape"]
        self.M, self.N, self.K = args.gemm_m, d.n_in, d.d_model
        self.x_host = S.activations(1, self.M, self.K, seed=11 + rank, n_outliers=w["n_outliers"],
                                    outlier_scale=w["outlier_scale"],
                                    outlier_seed=OUTLIER_SEED)[0]
        self.x0 = torch.from_numpy(self.x_host).to(dev)
        W = torch.from_numpy(S.layer_params(d, 1000)["w_in"]).to(dev)
        self.wq = torch.empty((self.N, self.K), dtype=torch.int8, device=dev)
        self.sw = torch.empty(self.N, dtype=torch.float32, device=dev)
        lib.prepare_linear(W, 1, self.wq, self.sw)
        del W
        self.q = torch.empty((self.M, self.K), dtype=torch.int8, device=dev)
        self.sx = torch.empty(self.M, dtype=torch.float32, device=dev)
        self.Y = torch.empty((self.M, self.N), dtype=torch.float32, device=dev)
        self.tokens = self.M
        self.launches = 2

    def _run(self, x, ev=None):
        lib = self.lib
        stream = self.torch.cuda.current_stream(self.dev)
        lib.hadamard_quant(x, self.K, None, 1, lib.FM_DYNAMIC, None, self.q, self.sx)
        if ev is not None:
            ev[0][0].record(stream)
        lib.w8a8_gemm(self.q, self.sx, self.wq, self.sw, self.Y)
        if ev is not None:
            ev[0][1].record(stream)

    def step(self, ev=None):
        self._run(self.x0, ev)

    def output(self):
        return self.Y

    def public_output(self):
        return None

    def e2e_setup(self):
        torch = self.torch
        self.xh = torch.from_numpy(self.x_host).pin_memory()
        self.oh = torch.empty((self.M, self.N), dtype=torch.float32).pin_memory()
        self.xd = torch.empty_like(self.x0)
        self.h2d_bytes = self.x_host.nbytes
        self.d2h_bytes = self.M * self.N * 4

    def e2e_step(self):
        self.xd.copy_(self.xh, non_blocking=True)
        self._run(self.xd)
        self.oh.copy_(self.Y, non_blocking=True)

    def e2e_matches(self, ref) -> bool:
        return True

    def roofline(self, dom_ms, peaks):
        ops = 2.0 * self.M * self.N * self.K
        achieved = ops / (dom_ms / 1e3) / 1e12
        bf16 = (peaks or {}).get("bf16_tflops", 1590.0)
        peak = bf16 * NOMINAL_INT8_OVER_BF16
        return {"bound": "tensor", "kernel": "fm_w8a8_gemm (k_gemm_i8_persist, tcgen05 kind::i8)",
                "achieved": achieved, "peak": peak, "unit": "TOPS (int8)",
                "frac": achieved / peak, "traffic": None,
                "peak_basis": "measured bf16 burst (bf16_tflops) x nominal int8/bf16 ratio 2",
                "algorithmic": f"2 M N K = {ops:.4g} int8 ops per launch"}


class LqStackWorkload(StackWorkload):
    """The FastMamba-LQ variant of a prefill workload: the same calibrated
    layers, W8A8 linears and scales, the conv, scan and gate in fp32.  The
    timed step calls the stage entry points in the order fm_lq_mixer_prefill
    composes them (checked bit for bit against it), events around each
    layer's scan."""

    launches_per_layer = 6  # FWHT+quant, in_proj, conv, scan (+ gate), norm+FWHT+quant, out_proj

    def __init__(self, args, torch, lib, dev, rank):
        super().__init__(args, torch, lib, dev, rank)
        d, M = self.shape, self.B * self.T
        e = lambda *sh: torch.empty(sh, dtype=torch.float32, device=dev)
        self.lbuf = dict(Y=e(M, d.n_in), xo=e(M, d.conv_ch), g=e(M, d.d_inner))
        self.ws = self.layers[0].lq_workspace(self.B, self.T)
        self.ssd = False
        self.sws = None
        _, extra = _gemm_workspace(torch, lib, d, M, dev)
        self.launches = (self.launches_per_layer + extra) * self.n_layers

    def step(self, ev=None):
        lib, d, B, T, b, lb = self.lib, self.shape, self.B, self.T, self.buf, self.lbuf
        di, cc = d.d_inner, d.conv_ch
        stream = self.torch.cuda.current_stream(self.dev)
        src = self.x0
        for i, Ly in enumerate(self.layers):
            lib.hadamard_quant(src, d.d_model, Ly.prenorm_w, 1, self.mode, Ly.static_amax,
                               b["q_in"], b["sx_in"])
            lib.w8a8_gemm(b["q_in"], b["sx_in"], Ly.w_in_q, Ly.w_in_s, lb["Y"], ws=self.gws)
            lib.lq_conv1d(lb["Y"][:, di:di + cc], B, T, d, Ly.conv_w, Ly.conv_b, None, lb["xo"])
            if ev is not None:
                ev[i][0].record(stream)
            lib.lq_scan(lb["xo"], lb["Y"][:, di + cc:], lb["Y"][:, :di], B, T, d, Ly.dt_bias,
                        Ly.a_log, Ly.D, None, lb["g"])
            if ev is not None:
                ev[i][1].record(stream)
            lib.hadamard_quant(lb["g"], di, Ly.norm_w, 1, self.mode, Ly.static_amax[1:],
                               b["q_out"], b["sx_out"])
            lib.w8a8_gemm(b["q_out"], b["sx_out"], Ly.w_out_q, Ly.w_out_s, self.r,
                          residual=src if self.stack_mode else None, ws=self.gws)
            src = self.r

    def _public(self, x, out):
        if self.stack_mode:
            if out is not x:
                out.copy_(x)
            for Ly in self.layers:
                Ly.lq_prefill(out, residual=True, out=out, ws=self.ws)
            return out
        return self.layers[0].lq_prefill(x, out=out, ws=self.ws)

    def public_output(self):
        return self._public(self.x0, self.torch.empty_like(self.x0))

    def e2e_step(self):
        self.xd.copy_(self.xh, non_blocking=True)
        self._public(self.xd, self.od)
        self.oh.copy_(self.od, non_blocking=True)

    def roofline(self, dom_ms, peaks):
        d = self.shape
        cells = self.B * d.nheads * d.headdim * d.d_state * self.T
        achieved = cells * LQ_FLOPS_PER_CELL / (dom_ms / 1e3) / 1e12
        mhz = (peaks or {}).get("sm_max_mhz", 1965.0)
        peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
        return {"bound": "alu", "kernel": "fm_lq_scan (k_lq_scan)", "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s (fp32)", "frac": achieved / peak, "traffic": None,
                "peak_basis": f"derived: 148 SMs x 128 fp32 FMA lanes x 2 flops x {mhz:.0f} MHz",
                "algorithmic": f"{LQ_FLOPS_PER_CELL} fp32 flops per state-cell update x {cells} "
                               "updates per launch"}


def make_workload(args, torch, lib, dev, rank):
    if args.workload == "gemm2p7b_inproj":
        return GemmWorkload(args, torch, lib, dev, rank)
    if args.workload == "decode2p7b_64l_b64":
        return DecodeWorkload(args, torch, lib, dev, rank)
    if getattr(args, "lq", False):
        return LqStackWorkload(args, torch, lib, dev, rank)
    return StackWorkload(args, torch, lib, dev, rank)


# ---------------------------------------------------------------- the GPU arm
def max_over_ranks(torch, dist, world, value, dev) -> float:
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measure(args, wl, torch, dist, lib, dev, world, flush) -> dict:
    """W untimed warm-up steps, then K timed steps bracketed by a barrier and
    synchronize on both sides (CUDA events on the launching stream, L2
    flushed before each), then K end-to-end steps through the public API with
    host copies.  Times are the max over ranks."""
    stream = torch.cuda.current_stream(dev)
    # a stack prefill pipelined by fm_stack_prefill: its kernels overlap on the
    # library's streams, so the dominant kernel is timed on the stage-by-stage
    # layer loop in a region of its own after the headline's
    pipelined = getattr(wl, "chunks", 1) > 1
    # the timed step (and the stage-by-stage one) must equal the public
    # per-layer entry points bit for bit
    ref = wl.public_output()
    for staged in ((False, True) if pipelined else (False,)):
        wl.step(staged=True) if staged else wl.step()
        torch.cuda.synchronize()
        lib.sync_status()
        if ref is not None and not torch.equal(ref, wl.output()):
            raise SystemExit("bench: the " + ("stage-by-stage" if staged else "timed") +
                             " step differs from the public entry points")
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()

    # events record timestamps even inside a captured graph (external records)
    E = lambda: torch.cuda.Event(enable_timing=True, external=not args.eager)

    def region(staged):
        """K steps, each: L2 flush, the step, its events (and with dev_ev the
        dominant kernel's, per layer).  Unless --eager, captured as one CUDA
        graph and replayed once untimed, which must give exactly what the
        same K steps give launched one by one."""
        ev = [(E(), E()) for _ in range(args.steps)]
        dev_ev = [[(E(), E()) for _ in range(wl.n_layers)] for _ in range(args.steps)]
        one = (lambda k: wl.step(dev_ev[k], staged=True)) if staged else \
              (lambda k: wl.step(None if pipelined else dev_ev[k]))
        tag = "bench_roofline_step" if staged else "bench_step"

        def timed_steps():
            for k in range(args.steps):
                flush.zero_()
                torch.cuda.nvtx.range_push(tag)
                ev[k][0].record()
                one(k)
                ev[k][1].record()
                torch.cuda.nvtx.range_pop()

        graph = None
        if not args.eager:
            restore = getattr(wl, "restore", None)
            if restore:
                restore()
            for _ in range(args.steps):
                wl.step(staged=True) if staged else wl.step()
            torch.cuda.synchronize()
            want = wl.output().clone()
            if restore:
                restore()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="relaxed"):
                timed_steps()
            graph.replay()
            torch.cuda.synchronize()
            lib.sync_status()
            if not torch.equal(want, wl.output()):
                raise SystemExit("bench: the captured graph differs from the same steps "
                                 "launched eagerly")
        return ev, dev_ev, graph, timed_steps

    def run(graph, timed_steps):
        if graph is not None:
            torch.cuda.nvtx.range_push("bench_graph")
            graph.replay()
            torch.cuda.nvtx.range_pop()
        else:
            timed_steps()

    ev, dev_ev, graph, timed_steps = region(False)
    clocks = ClockSampler(dev.index or 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    run(graph, timed_steps)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    lib.sync_status()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(torch, dist, world, sum(step_ms), dev)
    value = world * wl.tokens * args.steps / (total_ms / 1000.0)
    base_ms = step_ms
    if pipelined:
        del graph
        rev, dev_ev, graph, timed_steps = region(True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        run(graph, timed_steps)
        torch.cuda.synchronize()
        lib.sync_status()
        base_ms = [a.elapsed_time(b) for a, b in rev]
    dom_ms = [a.elapsed_time(b) for row in dev_ev for a, b in row]
    roofline = wl.roofline(statistics.mean(dom_ms), measured_peaks())
    roofline["avg_launch_us"] = 1000.0 * statistics.mean(dom_ms)
    roofline["share_of_step"] = sum(dom_ms) / sum(base_ms)
    if pipelined:
        roofline["measured_on"] = (
            "the stage-by-stage layer loop (one stream, the same kernels and sizes as "
            "fm_mixer_prefill), timed in its own region after the headline's: inside the "
            "pipelined step the scans overlap other kernels")
        roofline["staged_ms_per_step"] = statistics.mean(base_ms)
    roofline["traffic"] = dram_traffic(roofline["kernel"], args)

    # end to end through the public API: pinned host input -> device, the
    # computation, device -> pinned host output, every step
    wl.e2e_setup()
    for _ in range(2):
        wl.e2e_step()
    torch.cuda.synchronize()
    e2e_ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        wl.e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    lib.sync_status()
    if ref is not None and not wl.e2e_matches(ref):
        raise SystemExit("bench: end-to-end output differs from the device-resident step")
    e2e_total = max_over_ranks(torch, dist, world, sum(e2e_ms), dev)
    e2e_value = world * wl.tokens * args.steps / (e2e_total / 1000.0)
    del graph
    return {"value": value, "ms_per_step": total_ms / args.steps, "roofline": roofline,
            "clocks": clk, "launch": ("eager" if args.eager else "one CUDA graph of the K steps") +
            (", programmatic dependent launch" if getattr(args, "pdl", "on") == "on" else ""),
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": wl.h2d_bytes,
                    "d2h_bytes_per_step": wl.d2h_bytes},
            "gpu_launches": wl.launches * args.steps}


def apply_modes(args, lib):
    """Process-wide library settings of one run (scan tile, scan mode, state spec)."""
    if args.scan_tile:
        lib.set_scan_tile(*[int(v) for v in args.scan_tile.split(",")])
    lib.set_scan_mode(args.scan_mode)
    lib.set_state_spec(*[int(v) for v in args.state_spec.split(",")])
    lib.set_gemm_tile(args.gemm_tile)
    lib.set_pdl(getattr(args, "pdl", "on") == "on")
    lib.set_gemm_cluster(getattr(args, "gemm_cluster", "off") == "on")
    lib.set_lq_scan_cpw(getattr(args, "lq_cpw", 0))
    lib.set_xbc_exponents(args.xbc_exponents)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import datetime

    import torch
    import torch.distributed as dist

    from quantized_state_space_mamba2_b200 import build, lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    lib.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    apply_modes(args, lib)
    wl = make_workload(args, torch, lib, dev, rank)
    head = measure(args, wl, torch, dist, lib, dev, world, flush)
    del wl
    subs = {}
    for m in sub_modes(args):
        va = variant_args(args, m)
        apply_modes(va, lib)
        torch.cuda.empty_cache()
        w2 = make_workload(va, torch, lib, dev, rank)
        r = measure(va, w2, torch, dist, lib, dev, world, flush)
        del w2
        r["config"] = {k: v for k, v in config_block(va).items()
                       if config_block(args).get(k) != v}
        subs[m] = r
    apply_modes(args, lib)

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(args)
        line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "int8 x int8 -> int32 GEMM + int32 fixed point"
                         if not args.lq else "int8 x int8 -> int32 GEMM + fp32 conv/scan/gate",
                "data": "synthetic (seeded outlier-injected N(0,1), random-init weights)",
                "config": config_block(args), "roofline": head["roofline"],
                "cpu_baseline": cpu, "clocks": head["clocks"], "e2e": head["e2e"],
                "gpu_launches": head["gpu_launches"]}
        line["config"]["launch"] = head.pop("launch")
        for r in subs.values():
            r.pop("launch", None)
        if subs:
            line["modes"] = subs
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
