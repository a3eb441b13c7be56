"""The comparison arms of the rotated linears (``oracle.baselines``):
SmoothQuant's smoothing is an exact re-parametrisation of the unquantised
mixer; at alpha = 0.5 it balances each channel's activation and weight
maxima; at alpha = 1 it flattens every activation channel to max 1 -- both
closed forms of its definition; and on outlier inputs the linears rank as
the pages report (rotated > SmoothQuant > plain W8A8).  CPU only."""
import numpy as np
import pytest

from quantized_state_space_mamba2_b200 import synth as S

SMALL = S.MixerShape(d_model=256, d_inner=512, headdim=64, d_state=128)
OUT_SEED = 99


@pytest.fixture(scope="module")
def BL(oracle):
    from oracle import baselines
    return baselines


@pytest.fixture(scope="module")
def setup(oracle):
    P = S.layer_params(SMALL, 3)
    xc = S.calibration_batch(256, 48, 4, 50.0, outlier_seed=OUT_SEED, n_seqs=3)
    x = S.activations(1, 64, 256, seed=5, n_outliers=4, outlier_scale=50.0,
                      outlier_seed=OUT_SEED)
    return P, xc, x


def test_smoothing_leaves_the_unquantised_mixer_unchanged(oracle, BL, setup):
    P, xc, x = setup
    Q = BL.smooth_params(P, SMALL, xc)
    assert not np.array_equal(Q["w_in"], P["w_in"])
    a = oracle.ref_mixer_f64(P, SMALL, x, prenorm=True, residual=True)
    b = oracle.ref_mixer_f64(Q, SMALL, x, prenorm=True, residual=True)
    contrib = np.abs(a - x).max()
    assert np.abs(a - b).max() <= 1e-5 * contrib


@pytest.mark.parametrize("alpha", [0.5, 1.0])
def test_smoothing_closed_forms(oracle, BL, setup, alpha):
    """alpha = 0.5: max|X'_j| = max|W'[:, j]| = sqrt(max|X_j| max|W[:, j]|);
    alpha = 1: max|X'_j| = 1.  Measured on the smoothed model's own
    activations over the calibration set."""
    P, xc, _ = setup
    Q = BL.smooth_params(P, SMALL, xc, alpha=alpha)
    a0 = BL.activation_absmax(P, SMALL, xc)
    a1 = BL.activation_absmax(Q, SMALL, xc)
    for k, w in ((0, "w_in"), (1, "w_out")):
        wmax0 = np.abs(P[w].astype(np.float64)).max(axis=0)
        wmax1 = np.abs(Q[w].astype(np.float64)).max(axis=0)
        if alpha == 0.5:
            np.testing.assert_allclose(a1[k], wmax1, rtol=2e-6)
            np.testing.assert_allclose(a1[k], np.sqrt(a0[k] * wmax0), rtol=2e-6)
        else:
            np.testing.assert_allclose(a1[k], 1.0, rtol=2e-6)


def test_smoothing_factor_edge_cases(BL):
    W = np.array([[0.0, 2.0, 0.5], [0.0, -4.0, 0.25]])
    s = BL.smoothing_factors([3.0, 0.0, 4.0], W, alpha=0.5)
    assert s[0] == 1.0 and s[1] == 1.0              # a zero weight column / activation
    assert s[2] == pytest.approx(np.sqrt(4.0) / np.sqrt(0.5))


def test_linears_rank_as_the_pages_report(oracle, BL, setup):
    """Linears-only (LQ) SQNR of the mixer's contribution on outlier inputs,
    dynamic scales: Hadamard rotation > SmoothQuant > plain W8A8."""
    from oracle import stages as ST
    P, xc, x = setup
    ref = oracle.ref_mixer_f64(P, SMALL, x, prenorm=True, residual=True) - x
    Q = BL.smooth_params(P, SMALL, xc)
    out = {}
    for name, prm, rot in (("plain", P, 0), ("smooth", Q, 0), ("rotated", P, 1)):
        L = oracle.prepare_layer(prm, SMALL, rotate=rot, prenorm=True)
        oracle.calibrate_layer(L, xc, residual=True)
        out[name] = oracle.sqnr_db(ref, ST.lq_mixer(L, prm, x, residual=True) - x)
    assert out["rotated"] > out["smooth"] + 1.0, out
    assert out["smooth"] > out["plain"] + 3.0, out
