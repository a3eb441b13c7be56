"""The stage-by-stage mixer (``oracle.stages``) used for the error
attribution and the FastMamba-LQ variant: its two ends are pinned to the
quantised pipeline (every stage quantised, bit for bit) and to the fp64
reference (no stage quantised); its boundary quantiser agrees with the
oracle's own in_proj epilogue; each stage on its own changes the output by
a bounded amount; the LQ variant is closer to fp64 than the full method,
as the pages' accuracy table has it.  CPU only."""
import numpy as np
import pytest

from quantized_state_space_mamba2_b200 import synth as S

SMALL = S.MixerShape(d_model=256, d_inner=512, headdim=64, d_state=128)
OUT_SEED = 99


@pytest.fixture(scope="module")
def ST(oracle):
    from oracle import stages
    return stages


@pytest.fixture(scope="module")
def layers(oracle):
    """Calibrated small layers: (rotate, mode, prenorm) -> (params, layer)."""
    out = {}
    for rot, mode, pre in ((1, oracle.DYNAMIC, False), (1, oracle.STATIC, True),
                           (0, oracle.DYNAMIC, True)):
        P = S.layer_params(SMALL, 3)
        xc = S.calibration_batch(256, 48, 4, 50.0, outlier_seed=OUT_SEED, n_seqs=2)
        L = oracle.prepare_layer(P, SMALL, rotate=rot, mode=mode, prenorm=pre)
        oracle.calibrate_layer(L, xc, residual=pre)
        out[(rot, mode, pre)] = (P, L)
    return out


def _x(B=1, T=40, seed=5):
    return S.activations(B, T, 256, seed=seed, n_outliers=4, outlier_scale=50.0,
                         outlier_seed=OUT_SEED)


def test_every_stage_quantised_is_the_quantised_pipeline(oracle, ST, layers):
    x = _x(2, 33)
    for (rot, mode, pre), (P, L) in layers.items():
        got = ST.staged_mixer(L, P, x, ST.STAGES, residual=pre)
        ref = oracle.mixer_prefill(L, x, residual=pre)
        assert np.array_equal(got, ref.astype(np.float64)), (rot, mode, pre)


def test_no_stage_quantised_is_the_fp64_reference(oracle, ST, layers):
    x = _x(2, 33)
    for (rot, mode, pre), (P, L) in layers.items():
        got = ST.staged_mixer(L, P, x, (), residual=pre)
        ref = oracle.ref_mixer_f64(P, SMALL, x, prenorm=pre, residual=pre)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), (rot, mode, pre)


def test_boundary_quantiser_matches_the_in_proj_epilogue(oracle, ST, layers):
    """Quantising the dequantised in_proj output at e_u (the staged mixer's
    boundary rule) gives the epilogue's own int8 codes: 2^-e scaling is
    exact in fp32 and fp64 alike."""
    P, L = layers[(1, oracle.DYNAMIC, False)]
    s = SMALL
    x = _x(1, 40).reshape(40, 256)
    q, sx = oracle.hadamard_quant(x, None, L.rotate, L.mode, L.amax_in)
    acc = oracle.gemm_i8(q, L.wq_in)
    _, xbc, _ = oracle.in_proj_epilogue(acc, sx, L.sw_in, s.d_inner, s.conv_ch, s.nheads, L.e_u)
    Y = oracle.dequant(acc, sx, L.sw_in)[:, s.d_inner:s.d_inner + s.conv_ch]
    assert np.array_equal(ST._codes(Y, L.e_u, 8).astype(np.int8), xbc)


def test_each_stage_alone_changes_the_output_by_a_bounded_amount(oracle, ST, layers):
    P, L = layers[(1, oracle.DYNAMIC, False)]
    x = _x()
    ref = oracle.ref_mixer_f64(P, SMALL, x)
    for q in (("lin",), ("conv",), ("pwl",), ("scan",), ("eq5",)):
        got = ST.staged_mixer(L, P, x, q)
        assert not np.array_equal(got, ref), q
        assert oracle.sqnr_db(ref, got) > 15.0, q


def test_stage_implications(oracle, ST, layers):
    P, L = layers[(1, oracle.DYNAMIC, False)]
    x = _x(1, 20)
    assert np.array_equal(ST.staged_mixer(L, P, x, ("scan",)),
                          ST.staged_mixer(L, P, x, ("scan", "pwl")))
    # the fixed-point dt / dA overrides the exact Eq. (5) form
    assert np.array_equal(ST.staged_mixer(L, P, x, ("pwl",)),
                          ST.staged_mixer(L, P, x, ("pwl", "eq5")))
    with pytest.raises(ValueError):
        ST.staged_mixer(L, P, x, ("gate",))
    with pytest.raises(ValueError):
        ST.staged_mixer(L, P, x, ("nope",))


def test_lq_variant_is_closer_to_fp64_than_the_full_method(oracle, ST, layers):
    """FastMamba-LQ (linears only) keeps more accuracy than the fully
    quantised mixer: by several dB with the rotation (the method), by less
    without it, where the unrotated linears dominate the error.  Stacked
    layers compare the mixer's contribution (output - input)."""
    x = _x(1, 64, seed=8)
    for (rot, mode, pre), (P, L) in layers.items():
        base = x.astype(np.float64) if pre else 0.0
        ref = oracle.ref_mixer_f64(P, SMALL, x, prenorm=pre, residual=pre) - base
        lq = ST.lq_mixer(L, P, x, residual=pre)
        assert np.array_equal(lq, ST.staged_mixer(L, P, x, ("lin",), residual=pre))
        s_lq = oracle.sqnr_db(ref, lq - base)
        s_full = oracle.sqnr_db(ref, oracle.mixer_prefill(L, x, residual=pre) - base)
        assert s_lq > s_full + (3.0 if rot else 0.5), (rot, mode, pre)
