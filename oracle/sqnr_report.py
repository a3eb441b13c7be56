"""SQNR of the quantised mixer against the unquantised fp64 Mamba2 mixer, with
and without the Hadamard rotation, in both activation-scale modes, on
outlier-injected inputs (FastMamba, arXiv 2505.18975, pith.science review:
"What carries the argument" -- rotation spreads the outlier channels before
8-bit quantisation; mlsanity page on Mamba-PTQ: Mamba's activations carry
outlier channels).

The GPU library reproduces the oracle bit for bit, so these numbers are also
the GPU path's.  Runs on the CPU in about a quarter of an hour:

    python -m oracle.sqnr_report            # rotation tables
    python -m oracle.sqnr_report --stages   # per-stage attribution only
    python -m oracle.sqnr_report --baselines  # plain W8A8 / SmoothQuant / rotated
    python -m oracle.sqnr_report --state-bits # width of the SSM state word
    python -m oracle.sqnr_report --readings   # conv-output exponents x state width
    python -m oracle.sqnr_report --ssd        # the chunked (tensor-core form) scan mode
    python -m oracle.sqnr_report --2p7b       # one 2.7B-shaped layer (about half an hour)

The attribution (``oracle.stages``) quantises the stages of one layer alone
and cumulatively, in pipeline order; its first row is FastMamba-LQ, the
linears-only variant.
"""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from oracle import baselines as BL  # noqa: E402
from oracle import stages as ST  # noqa: E402
from quantized_state_space_mamba2_b200 import synth as S  # noqa: E402

OUTLIER_SEED = 4242


def layer_case(rotate: int, mode: int, n_outliers: int, scale: float, T: int = 256):
    """One 130M-shaped layer (B=1): calibrated on 16 x min(T, 512) seeded
    sequences, evaluated on a fresh seeded sequence."""
    shape = S.MAMBA2_130M
    P = S.layer_params(shape, 1000)
    xcal = S.calibration_batch(shape.d_model, T, n_outliers, scale, OUTLIER_SEED)
    L = O.prepare_layer(P, shape, rotate=rotate, mode=mode)
    O.calibrate_layer(L, xcal)
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=n_outliers, outlier_scale=scale,
                      outlier_seed=OUTLIER_SEED)
    ref = O.ref_mixer_f64(P, shape, x)
    return O.sqnr_db(ref, O.mixer_prefill(L, x))


def stack_case(rotate: int, mode: int, layers: int = 4, T: int = 256):
    """The first layers of the 130M stack (pre-norm + residual): SQNR of each
    layer's mixer contribution (output - input), the quantised stack against
    the fp64 stack run on the same input."""
    shape = S.MAMBA2_130M
    P = [S.layer_params(shape, 1000 + l) for l in range(layers)]
    c = S.calibration_batch(shape.d_model, T, 8, 50.0, OUTLIER_SEED)
    Ls = []
    for p in P:
        L = O.prepare_layer(p, shape, rotate=rotate, mode=mode, prenorm=True)
        c = O.calibrate_layer(L, c, residual=True)
        Ls.append(L)
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    xq, xr, out = x, x.astype(np.float64), []
    for p, L in zip(P, Ls):
        yq = O.mixer_prefill(L, xq, residual=True)
        yr = O.ref_mixer_f64(p, shape, xr, prenorm=True, residual=True)
        out.append(O.sqnr_db(yr - xr, yq.astype(np.float64) - xq))
        xq, xr = yq, yr
    return out


def stage_rows(mode: int, T: int = 256):
    """SQNR (dB) of one rotated 130M-shaped layer with the named stages
    quantised, calibrated as in ``layer_case`` (8 outlier channels x50)."""
    shape = S.MAMBA2_130M
    P = S.layer_params(shape, 1000)
    L = O.prepare_layer(P, shape, rotate=1, mode=mode)
    O.calibrate_layer(L, S.calibration_batch(shape.d_model, T, 8, 50.0, OUTLIER_SEED))
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    ref = O.ref_mixer_f64(P, shape, x)
    rows = [("linears only (FastMamba-LQ)", ("lin",)),
            ("conv only (PoT codes, PWL SiLU)", ("conv",)),
            ("SoftPlus as Eq. (5), exact arithmetic", ("eq5",)),
            ("dt, dA through the fixed-point 2^v unit", ("pwl",)),
            ("fixed-point scan (with its dt, dA)", ("scan",)),
            ("linears + conv", ("lin", "conv")),
            ("linears + conv + dt, dA", ("lin", "conv", "pwl")),
            ("linears + conv + scan", ("lin", "conv", "scan")),
            ("all stages (the full method)", ST.STAGES)]
    return [(name, O.sqnr_db(ref, ST.staged_mixer(L, P, x, q))) for name, q in rows]


def print_stage_table():
    dyn, sta = stage_rows(O.DYNAMIC), stage_rows(O.STATIC)
    print("| stages quantised (rest exact fp64) | SQNR, dynamic (dB) | SQNR, static (dB) |")
    print("|---|---|---|")
    for (name, a), (_, b) in zip(dyn, sta):
        print(f"| {name} | {a:.2f} | {b:.2f} |")


def baseline_rows(T: int = 256):
    """One 130M-shaped pre-norm layer (stack form, residual), 8 outlier
    channels x50: SQNR of the mixer's contribution with plain W8A8,
    SmoothQuant (alpha 0.5) and the Hadamard rotation, linears only (LQ) and
    the full method, in both activation-scale modes."""
    shape = S.MAMBA2_130M
    P = S.layer_params(shape, 1000)
    xc = S.calibration_batch(shape.d_model, T, 8, 50.0, OUTLIER_SEED)
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    xr = x.astype(np.float64)
    ref = O.ref_mixer_f64(P, shape, x, prenorm=True, residual=True) - xr
    Q = BL.smooth_params(P, shape, xc)
    rows = []
    for name, prm, rot in (("plain W8A8", P, 0), ("SmoothQuant, alpha 0.5", Q, 0),
                           ("Hadamard rotation (the method)", P, 1)):
        vals = []
        for mode in (O.DYNAMIC, O.STATIC):
            L = O.prepare_layer(prm, shape, rotate=rot, mode=mode, prenorm=True)
            O.calibrate_layer(L, xc, residual=True)
            vals.append(O.sqnr_db(ref, ST.lq_mixer(L, prm, x, residual=True) - xr))
            vals.append(O.sqnr_db(ref, O.mixer_prefill(L, x, residual=True) - xr))
        rows.append((name, vals))
    return rows


def print_baseline_table():
    print("| linears | LQ, dynamic (dB) | full, dynamic (dB) | LQ, static (dB) | full, static (dB) |")
    print("|---|---|---|---|---|")
    for name, v in baseline_rows():
        print(f"| {name} | " + " | ".join(f"{a:.2f}" for a in v) + " |")


def state_bits_rows(bits=(31, 24, 20, 16), T_cal: int = 512, T: int = 1024):
    """One rotated 130M-shaped layer calibrated on 16 x 512 tokens and run
    over 1024: SQNR of the whole output and of its last 256 tokens for
    each width of the state word (both activation-scale modes)."""
    shape = S.MAMBA2_130M
    P = S.layer_params(shape, 1000)
    xc = S.calibration_batch(shape.d_model, T_cal, 8, 50.0, OUTLIER_SEED)
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    ref = O.ref_mixer_f64(P, shape, x)
    rows = []
    for b in bits:
        vals = []
        for mode in (O.DYNAMIC, O.STATIC):
            L = O.prepare_layer(P, shape, mode=mode, state_bits=b)
            O.calibrate_layer(L, xc)
            out = O.mixer_prefill(L, x)
            vals += [O.sqnr_db(ref, out), O.sqnr_db(ref[:, -256:], out[:, -256:])]
        rows.append((b, vals))
    return rows


def print_state_bits_table():
    print("| state word | dynamic, all (dB) | dynamic, last 256 (dB) | static, all (dB) | "
          "static, last 256 (dB) |")
    print("|---|---|---|---|---|")
    for b, v in state_bits_rows():
        name = f"{b} bits" + (" (as built)" if b == 31 else "")
        print(f"| {name} | " + " | ".join(f"{a:.2f}" for a in v) + " |")


def readings_rows(T: int = 256):
    """One rotated 130M-shaped layer as in ``layer_case`` (8 outlier channels
    x50): conv-output exponents static per head or per token, with the 31-bit
    and the 16-bit state word."""
    shape = S.MAMBA2_130M
    P = S.layer_params(shape, 1000)
    xc = S.calibration_batch(shape.d_model, T, 8, 50.0, OUTLIER_SEED)
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    ref = O.ref_mixer_f64(P, shape, x)
    rows = []
    for xe, bits, g in (("static", 31, 0), ("token", 31, 0), ("static", 16, 0), ("token", 16, 0),
                        ("static", 16, 7), ("token", 16, 7)):
        vals = []
        for mode in (O.DYNAMIC, O.STATIC):
            L = O.prepare_layer(P, shape, mode=mode, state_bits=bits, xbc_exponents=xe,
                                ub_guard=g)
            O.calibrate_layer(L, xc)
            vals.append(O.sqnr_db(ref, O.mixer_prefill(L, x)))
        rows.append((xe, bits, g, vals))
    return rows


def print_readings_table():
    print("| conv-output exponents | state word | increment rounded | SQNR, dynamic (dB) | "
          "SQNR, static (dB) |")
    print("|---|---|---|---|---|")
    for xe, bits, g, v in readings_rows():
        name = "static per head" if xe == "static" else "per token"
        tag = " (as built)" if (xe, bits, g) == ("static", 31, 0) else ""
        rnd = "u, then u B" if g == 0 else f"after u B ({g} guard bits)"
        print(f"| {name}{tag} | {bits} bits | {rnd} | {v[0]:.2f} | {v[1]:.2f} |")


def ssd_rows(T: int = 256):
    """One rotated 130M-shaped layer as in ``layer_case``: the sequential
    fixed-point scan against the chunked scan mode (bf16 operands, chunks of
    64 and 128 tokens), calibrated the same way."""
    shape = S.MAMBA2_130M
    P = S.layer_params(shape, 1000)
    xc = S.calibration_batch(shape.d_model, T, 8, 50.0, OUTLIER_SEED)
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    ref = O.ref_mixer_f64(P, shape, x)
    rows = {("seq", 0): [], ("ssd", 64): [], ("ssd", 128): []}
    for mode in (O.DYNAMIC, O.STATIC):
        L = O.prepare_layer(P, shape, mode=mode)
        O.calibrate_layer(L, xc)
        for (sm, q), v in rows.items():
            L.scan_mode, L.ssd_chunk = sm, q or 64
            v.append(O.sqnr_db(ref, O.mixer_prefill(L, x)))
    return rows


def print_ssd_table():
    print("| scan | SQNR, dynamic (dB) | SQNR, static (dB) |")
    print("|---|---|---|")
    for (sm, q), v in ssd_rows().items():
        name = "sequential fixed point (as built)" if sm == "seq" else \
            f"chunked, {q}-token chunks, bf16 operands"
        print(f"| {name} | {v[0]:.2f} | {v[1]:.2f} |")


def rows_2p7b(T: int = 256, n_cal: int = 4):
    """One 2.7B-shaped layer (d_model 2560, 80 heads), 8 outlier channels x50,
    dynamic scales, calibrated on n_cal seeded sequences of T tokens (fewer
    than the 16 of the 130M tables: the oracle's 2.7B calibration takes
    minutes per sequence): the method with and without the rotation, and the
    candidate spec (per-token exponents, 16-bit state, guard-bit increment)."""
    shape = S.MAMBA2_2P7B
    P = S.layer_params(shape, 1000)
    xc = S.calibration_batch(shape.d_model, T, 8, 50.0, OUTLIER_SEED, n_seqs=n_cal)
    x = S.activations(1, T, shape.d_model, seed=1, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    ref = O.ref_mixer_f64(P, shape, x)
    rows = []
    for name, kw in (("the method, rotated (as built)", dict(rotate=1)),
                     ("the method, not rotated", dict(rotate=0)),
                     ("rotated, per-token exponents, 16-bit state, guard bits",
                      dict(rotate=1, state_bits=16, xbc_exponents="token", ub_guard=7))):
        L = O.prepare_layer(P, shape, **kw)
        O.calibrate_layer(L, xc)
        rows.append((name, O.sqnr_db(ref, O.mixer_prefill(L, x))))
    return rows


def print_2p7b_table():
    print("| 2.7B-shaped layer, dynamic scales | SQNR (dB) |")
    print("|---|---|")
    for name, v in rows_2p7b():
        print(f"| {name} | {v:.2f} |", flush=True)


def main():
    if "--2p7b" in sys.argv[1:]:
        print_2p7b_table()
        return
    if "--ssd" in sys.argv[1:]:
        print_ssd_table()
        return
    if "--readings" in sys.argv[1:]:
        print_readings_table()
        return
    if "--state-bits" in sys.argv[1:]:
        print_state_bits_table()
        return
    if "--stages" in sys.argv[1:]:
        print_stage_table()
        return
    if "--baselines" in sys.argv[1:]:
        print_baseline_table()
        return
    modes = [("dynamic", O.DYNAMIC), ("static", O.STATIC)]
    print("| input | act. scales | SQNR, rotated (dB) | SQNR, not rotated (dB) |")
    print("|---|---|---|---|")
    for n_out, scale, label in [(8, 50.0, "8 outlier channels x50"), (0, 1.0, "no outliers")]:
        for mname, m in modes:
            r = layer_case(1, m, n_out, scale)
            p = layer_case(0, m, n_out, scale)
            print(f"| {label} | {mname} | {r:.2f} | {p:.2f} |")
    print()
    print("| 130M stack, mixer contribution | act. scales | rotated, layers 1-4 (dB) | not rotated (dB) |")
    print("|---|---|---|---|")
    for mname, m in modes:
        r = stack_case(1, m)
        p = stack_case(0, m)
        print(f"| 8 outlier channels x50 | {mname} | {' / '.join(f'{v:.1f}' for v in r)} | "
              f"{' / '.join(f'{v:.1f}' for v in p)} |")
    print()
    print_stage_table()
    print()
    print_baseline_table()
    print()
    print_state_bits_table()
    print()
    print_readings_table()
    print()
    print_ssd_table()


if __name__ == "__main__":
    main()
