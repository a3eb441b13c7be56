"""Host-side logic of bench.py: argument defaults, the clock-sample parser,
the per-workload token counts, the oracle sample's scaling, and the
max-over-ranks step time across two gloo ranks on CPU."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_defaults_are_the_headline_workload():
    a = bench.parse([])
    assert a.workload == "stack130m_24l_b1_t2048" and a.gpus == 1 and a.warmup >= 3
    assert bench.workload_tokens(a) == 2048
    c = bench.config_block(a)
    assert c["layers"] == 24 and c["batch"] == 1 and c["seq_len"] == 2048


@pytest.mark.parametrize("w,tokens", [("mixer130m_b1_t256", 256), ("stack2p7b_64l_b2_t4096", 8192),
                                      ("decode2p7b_64l_b64", 64)])
def test_workload_tokens(w, tokens):
    assert bench.workload_tokens(bench.parse(["--workload", w])) == tokens


def test_gemm_sweep_sizes():
    for m in (2048, 8192, 32768):
        a = bench.parse(["--workload", "gemm2p7b_inproj", "--gemm-m", str(m)])
        c = bench.config_block(a)
        assert bench.workload_tokens(a) == m and (c["M"], c["N"], c["K"]) == (m, 10576, 2560)
    with pytest.raises(SystemExit):
        bench.parse(["--workload", "gemm2p7b_inproj", "--gemm-m", "100"])


def test_clock_parser():
    text = ("1965, 1965, 700.1, Not Active, Not Active, Not Active, Not Active\n"
            "1950, 1965, 900.0, Not Active, Not Active, Not Active, Active\n"
            "1800, 1965, 990.0, Not Active, Not Active, Not Active, Active\n"
            "garbage line\n")
    c = bench.parse_clock_samples(text)
    assert c["sm_mhz"] == 1950 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"]
    assert bench.parse_clock_samples("")["sm_mhz"] is None


def test_oracle_sample_scaling():
    o = bench.OracleSample.__new__(bench.OracleSample)
    o.tokens, o.layers = 512, 64
    assert o.value(2.0) == pytest.approx(512 / (2.0 * 64))


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        v = bench.max_over_ranks(torch, dist, world, 10.0 + 5.0 * rank, torch.device("cpu"))
        out[rank] = v
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == out[1] == 15.0


def test_reference_arm_line():
    """--impl reference prints one JSON line with the contract's keys."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "mixer130m_b1_t256", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "config", "cpu_baseline", "e2e"):
        assert k in line
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    # what was timed: one sample per host core, and the factor to a full step
    cores = line["cpu_baseline"]["cores"]
    assert cores == bench.host_cores() >= 1
    ex = line["extrapolation"]
    assert ex["factor"] == pytest.approx(256 / (cores * min(256, bench.CPU_ALLCORE_TOKENS)))
    # the reported step time is the timed sample's, consistent with value
    per_core_tokens = min(256, bench.CPU_ALLCORE_TOKENS)
    assert line["value"] == pytest.approx(cores * per_core_tokens / (line["ms_per_step"] / 1e3),
                                          rel=1e-6)


def test_sub_record_modes():
    """The headline runs alone except on the default workload, where the
    static, chunked-scan, 16-bit-state and LQ modes follow as sub-records;
    each sub-record differs from the headline in exactly its mode's settings
    and, where that mode runs the layer loop instead of the pipelined stack
    (the chunked scan, LQ), in the pipeline."""
    a = bench.parse([])
    assert bench.sub_modes(a) == ["static", "ssd", "state16", "candidate", "lq"]
    assert bench.sub_modes(bench.parse(["--modes", "none"])) == []
    assert bench.sub_modes(bench.parse(["--workload", "stack2p7b_64l_b2_t4096"])) == []
    assert bench.sub_modes(bench.parse(["--workload", "stack2p7b_64l_b2_t4096",
                                        "--modes", "ssd"])) == ["ssd"]
    with pytest.raises(SystemExit):
        bench.sub_modes(bench.parse(["--modes", "fast"]))
    base = bench.config_block(a)
    for m, keys in (("static", {"act_quant"}), ("ssd", {"scan_mode", "pipeline"}),
                    ("state16", {"state_spec"}), ("candidate", {"state_spec", "xbc_exponents"}),
                    ("lq", {"variant", "pipeline"})):
        v = bench.variant_args(a, m)
        diff = {k for k, x in bench.config_block(v).items() if base.get(k) != x}
        assert diff == keys, (m, diff)
    assert not a.lq and a.mode == "dynamic"          # the headline's args are untouched


def test_pipeline_defaults():
    """Single-sequence stack prefills with the sequential scan are pipelined in
    4 runs by default; every other workload runs the layer loop, and every
    stack workload class (including those that build themselves without the
    base constructor, like the decode step) reads 1 run by default."""
    for cls in (bench.StackWorkload, bench.DecodeWorkload, bench.LqStackWorkload):
        assert cls.chunks == 1, cls
    assert bench.stack_chunks(bench.parse([])) == 4
    assert bench.stack_chunks(bench.parse(["--chunks", "2"])) == 2
    for argv in (["--workload", "stack2p7b_64l_b2_t4096"], ["--workload", "decode2p7b_64l_b64"],
                 ["--workload", "mixer130m_b1_t256"], ["--scan-mode", "ssd"], ["--lq"],
                 ["--workload", "decode2p7b_64l_b64", "--chunks", "4"]):
        assert bench.stack_chunks(bench.parse(argv)) == 1, argv
    assert bench.stack_runs(2048, 4) == (4, 512)
    assert bench.stack_runs(200, 3) == (3, 96)
    assert bench.stack_runs(40, 64) == (2, 32)
    assert bench.stack_runs(1, 2) == (1, 1)
