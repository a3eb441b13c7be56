"""SQNR of the quantised mixer against the unquantised fp64 Mamba2 mixer, with
and without the Hadamard rotation, in both activation-scale modes, on
outlier-injected inputs (FastMamba, arXiv 2505.18975, pith.science review:
"What carries the argument" -- rotation spreads the outlier channels before
8-bit quantisation; mlsanity page on Mamba-PTQ: Mamba's activations carry
outlier channels).

The GPU library reproduces the oracle bit for bit, so these numbers are also
the GPU path's.  Runs on the CPU in about a quarter of an hour:

    python -m oracle.sqnr_report
"""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
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


def main():
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


if __name__ == "__main__":
    main()
