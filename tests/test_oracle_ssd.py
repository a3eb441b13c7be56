"""The chunked (state-space-dual) scan mode (``oracle.ssd``): with exact
operands it is the recurrence h_t = 2^(w_t) h_{t-1} + dt_t x_t B_t^T,
y_t = C_t h_t on the codes -- pinned to an fp64 recurrence for one chunk and
for many (a wrong decay index or a dropped inter-chunk term moves the result
far beyond fp32 rounding); bf16 operands stay inside the bf16 error budget;
its bf16 rounding matches torch's; the state hands over to and from the
sequential scan's int32 word; a layer run in this mode is as close to fp64
as the sequential method.  CPU only."""
import numpy as np
import pytest

from quantized_state_space_mamba2_b200 import synth as S

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def SSD(oracle):
    from oracle import ssd
    return ssd


def _inputs(Bsz=1, T=40, nh=2, hd=8, ds=16, seed=120):
    cc = nh * hd + 2 * ds
    xbc = S.uniform_ints((Bsz, T, cc), -127, 127, seed=seed, dtype=np.int8)
    dt_raw = S.normal((Bsz, T, nh), 1.0, seed=seed + 1)
    dt_bias = np.array([-1.0, 0.5], np.float32)[:nh]
    A_q = np.array([3000, 9000], np.int32)[:nh]
    return xbc, dt_raw, dt_bias, A_q


def _f64_recurrence(SSD, xbc, dt_raw, dt_bias, A_q, hd, ds, h0=None):
    """y (code units, no skip term) and the final state by the plain recurrence
    in fp64 with decay 2^(w_t / 2^16) and dt_q / 2^16."""
    Bsz, T, cc = xbc.shape
    nh = len(A_q)
    di = nh * hd
    dtq, w = SSD.decay_exponents(xbc, dt_raw, dt_bias, A_q, hd, ds)
    X = xbc[..., :di].reshape(Bsz, T, nh, hd).astype(np.float64)
    Bm = xbc[..., di:di + ds].astype(np.float64)
    Cm = xbc[..., di + ds:].astype(np.float64)
    h = np.zeros((Bsz, nh, hd, ds)) if h0 is None else h0.copy()
    y = np.empty((Bsz, T, nh, hd))
    for t in range(T):
        dA = np.exp2(w[:, t] / 65536.0)
        h = dA[:, :, None, None] * h + (dtq[:, t, :, None] / 65536.0 * X[:, t])[..., None] \
            * Bm[:, t, None, None, :]
        y[:, t] = np.einsum("bhpn,bn->bhp", h, Cm[:, t])
    return y.reshape(Bsz, T, di), h


def _args(nh):
    z = np.zeros(nh, np.int32)
    # e_x = e_B = e_C = 0, e_y = 0, e_D = 0 with D_q = 0: y codes = rint(SSM part)
    return dict(D_q=z, e_x=z, e_B=0, e_C=0, e_h=z, e_y=z, e_D=z)


@pytest.mark.parametrize("Q", [64, 8, 5])
def test_exact_operands_equal_the_recurrence(oracle, SSD, Q):
    """One chunk (Q = 64 > T) and many chunks (Q = 8, 5 with a ragged last
    chunk): the fp32 SSM part equals the fp64 recurrence to fp32 rounding."""
    xbc, dt_raw, dt_bias, A_q = _inputs()
    hd, ds = 8, 16
    _, yf = SSD.ssd_scan(xbc, dt_raw, dt_bias, A_q, hd=hd, ds=ds, Q=Q, operand="fp32",
                         want_f32=True, **_args(2))
    ref, _ = _f64_recurrence(SSD, xbc, dt_raw, dt_bias, A_q, hd, ds)
    scale = np.abs(ref).max()
    assert np.abs(yf - ref).max() <= 2e-6 * scale
    assert scale > 1e4


def test_bf16_operands_within_budget(oracle, SSD):
    """bf16 rounding of M, U, the decayed C and the carried state: each
    rounded operand is off by at most 2^-9 of itself, so the output error
    stays below 3 * 2^-9 of the sum of |terms| (a product of two rounded
    operands is off by at most 2 * 2^-9 + 2^-18; the state adds its own)."""
    xbc, dt_raw, dt_bias, A_q = _inputs(T=48)
    hd, ds = 8, 16
    _, yb = SSD.ssd_scan(xbc, dt_raw, dt_bias, A_q, hd=hd, ds=ds, Q=16, operand="bf16",
                         want_f32=True, **_args(2))
    _, ye = SSD.ssd_scan(xbc, dt_raw, dt_bias, A_q, hd=hd, ds=ds, Q=16, operand="fp32",
                         want_f32=True, **_args(2))
    # sum of |terms|: the recurrence run on |x|, |B|, |C|
    absx = np.abs(xbc.astype(np.int16)).astype(np.int8)
    mag, _ = _f64_recurrence(SSD, absx, dt_raw, dt_bias, A_q, hd, ds)
    err = np.abs(yb.astype(np.float64) - ye)
    assert (err <= 3 * 2.0 ** -9 * mag + 1e-3).all()
    assert err.max() > 0                                    # the rounding is really applied


def test_bf16_rounding_matches_torch(SSD):
    v = (S.normal(4096, 1.0, seed=130) * np.exp2(S.uniform_ints(4096, -20, 20, seed=131))
         ).astype(np.float32)
    v[:4] = [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0]   # ties
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    assert np.array_equal(SSD.bf16(v), ref)


def test_state_hands_over_to_the_sequential_scan(oracle, SSD):
    """Chunked prefill of T1 tokens, then the rest: with exact operands the
    state leaving the first call (int32 at e_h) carries the recurrence on,
    within the state word's rounding; and the chunked state agrees with the
    sequential scan's state."""
    hd, ds, nh = 8, 16, 2
    xbc, dt_raw, dt_bias, A_q = _inputs(T=40)
    a = _args(nh)
    a["e_h"] = np.full(nh, -8, np.int32)                    # state LSB 2^-8 code units
    st = np.zeros((1, nh, hd, ds), np.int32)
    SSD.ssd_scan(xbc[:, :23].copy(), dt_raw[:, :23].copy(), dt_bias, A_q, hd=hd, ds=ds, Q=8,
                 state=st, operand="fp32", **a)
    _, h_ref = _f64_recurrence(SSD, xbc[:, :23], dt_raw[:, :23], dt_bias, A_q, hd, ds)
    assert np.abs(st * 2.0 ** -8 - h_ref).max() <= 2.0 ** -9 + 1e-6 * np.abs(h_ref).max()
    _, yf = SSD.ssd_scan(xbc[:, 23:].copy(), dt_raw[:, 23:].copy(), dt_bias, A_q, hd=hd, ds=ds,
                         Q=8, state=st, operand="fp32", want_f32=True, **a)
    ref, _ = _f64_recurrence(SSD, xbc, dt_raw, dt_bias, A_q, hd, ds)
    # the handed-over state is off by <= 2^-9 per cell: |C| sum * 2^-9 on y
    tol = 128 * ds * 2.0 ** -9 + 2e-6 * np.abs(ref).max()
    assert np.abs(yf - ref[:, 23:]).max() <= tol


def test_ssd_layer_is_as_close_to_fp64_as_the_method(oracle, SSD):
    """A small layer calibrated as the method, run with the chunked bf16
    scan: its SQNR against the fp64 mixer is within 0.5 dB of the
    sequential method's (the scan mode's own error is far below the
    method's)."""
    shape = S.MixerShape(d_model=256, d_inner=512, headdim=64, d_state=128)
    P = S.layer_params(shape, 3)
    xc = S.calibration_batch(256, 64, 4, 50.0, outlier_seed=99, n_seqs=2)
    L = oracle.prepare_layer(P, shape)
    oracle.calibrate_layer(L, xc)
    x = S.activations(1, 96, 256, seed=5, n_outliers=4, outlier_scale=50.0, outlier_seed=99)
    ref = oracle.ref_mixer_f64(P, shape, x)
    seq = oracle.sqnr_db(ref, oracle.mixer_prefill(L, x))
    L.scan_mode = "ssd"
    ssd = oracle.sqnr_db(ref, oracle.mixer_prefill(L, x))
    assert ssd > seq - 0.5, (ssd, seq)
