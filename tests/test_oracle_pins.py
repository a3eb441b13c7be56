"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a library routine (scipy's Sylvester
Hadamard matrix, numpy integer matmul / convolution, numpy exp2 / exp,
torch's depthwise conv1d), a closed form, an exact identity of the
mathematics, or brute force -- chosen so that a dropped term, a wrong sign
or index, or a transposed operand fails one of them.  No GPU is needed.
"""
import numpy as np
import pytest
import scipy.linalg

from quantized_state_space_mamba2_b200 import synth as S

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def hadamard_bd(K):
    """Block-diagonal Sylvester Hadamard (block 256) / 16 from scipy."""
    H = scipy.linalg.hadamard(256).astype(np.float64) / 16.0
    return scipy.linalg.block_diag(*([H] * (K // 256)))


# ------------------------------------------------------------------ Hadamard

def test_fwht_equals_scipy_sylvester(oracle):
    eye = np.eye(256)
    H = oracle.fwht256(eye)               # row i = e_i H
    assert np.array_equal(H, scipy.linalg.hadamard(256) / 16.0)
    H32 = oracle.fwht256(eye.astype(np.float32))
    assert np.array_equal(H32.astype(np.float64), scipy.linalg.hadamard(256) / 16.0)


def test_hadamard_orthonormal_exact(oracle):
    H = oracle.fwht256(np.eye(256))
    assert np.array_equal(H @ H.T, np.eye(256))      # entries +-1/16: exact in fp64
    assert set(np.unique(H)) == {-1 / 16, 1 / 16}


def test_fwht_dense_multiply_and_involution(oracle):
    x = S.uniform_ints((5, 768), -1000, 1000, seed=3).astype(np.float32)
    a = oracle.fwht256(x)
    assert np.array_equal(a.astype(np.float64), x.astype(np.float64) @ hadamard_bd(768))
    assert np.array_equal(oracle.fwht256(a), x)       # H H = I, exact for small integers


def test_rotation_preserves_linear_layer(oracle):
    # (XH)(H^T W^T) = X W^T in fp64 to 1e-10 (rotation of both operands)
    X = S.normal((16, 768), 1.0, seed=4).astype(np.float64)
    W = S.normal((40, 768), 0.02, seed=5).astype(np.float64)
    Y = oracle.fwht256(X) @ oracle.fwht256(W).T
    ref = X @ W.T
    assert np.max(np.abs(Y - ref)) <= 1e-10 * np.max(np.abs(ref))


# ------------------------------------------------------------------ quantisation

def test_dynamic_act_quant_closed_form(oracle):
    x = S.activations(1, 32, 768, seed=6, n_outliers=8, outlier_scale=50.0)[0]
    q, sx, am = oracle.hadamard_quant(x, want_amax=True)
    a = x.astype(np.float64) @ hadamard_bd(768)
    assert np.allclose(am, np.abs(a).max(1), rtol=1e-6)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    assert np.all(np.abs(q).max(1) == 127)                     # the max element maps to 127
    err = np.abs(q * sx[:, None].astype(np.float64) - a)
    assert np.all(err <= sx[:, None] * (0.5 + 1e-4))           # |dequant - a| <= s/2
    q0, s0 = oracle.hadamard_quant(np.zeros((2, 256), np.float32))
    assert not q0.any() and not s0.any()


def test_static_act_quant_clips(oracle):
    x = S.normal((8, 512), 1.0, seed=7)
    a = x.astype(np.float64) @ hadamard_bd(512)
    amax = float(np.quantile(np.abs(a), 0.5))
    q, sx = oracle.hadamard_quant(x, mode=oracle.STATIC, static_amax=amax)
    assert np.allclose(sx, amax / 127.0, rtol=1e-7)
    inside = np.abs(a) <= amax
    assert np.all(np.abs(q[inside] * np.float64(sx[0]) - a[inside]) <= sx[0] * (0.5 + 1e-4))
    assert np.all(np.abs(q[~inside]) == 127) and np.all(np.sign(q[~inside]) == np.sign(a[~inside]))


def test_prenorm_rotation_quant(oracle):
    x = S.activations(1, 16, 768, seed=8, n_outliers=8, outlier_scale=50.0)[0]
    w = 1.0 + S.normal(768, 0.1, seed=9)
    q, sx = oracle.hadamard_quant(x, prenorm_w=w)
    xd = x.astype(np.float64)
    u = xd / np.sqrt((xd * xd).mean(1, keepdims=True) + 1e-5) * w
    a = u @ hadamard_bd(768)
    err = np.abs(q * sx[:, None].astype(np.float64) - a)
    assert np.all(err <= sx[:, None] * (0.5 + 1e-3))


def test_prepare_linear_per_channel(oracle):
    W = S.normal((64, 512), 0.02, seed=10)
    wq, sw = oracle.prepare_linear(W)
    Wr = W.astype(np.float64) @ hadamard_bd(512)
    assert np.allclose(sw, np.abs(Wr).max(1) / 127.0, rtol=1e-7)
    assert np.all(np.abs(wq).max(1) == 127)
    assert np.all(np.abs(wq * sw[:, None].astype(np.float64) - Wr) <= sw[:, None] * (0.5 + 1e-6))
    wq0, sw0 = oracle.prepare_linear(W, rotate=0)
    assert np.all(np.abs(wq0 * sw0[:, None].astype(np.float64) - W) <= sw0[:, None] * 0.5001)


def test_gemm_matches_numpy_and_layer_output(oracle):
    A = S.uniform_ints((33, 512), -127, 127, seed=11, dtype=np.int8)
    W = S.uniform_ints((47, 512), -127, 127, seed=12, dtype=np.int8)
    acc = oracle.gemm_i8(A, W)
    assert np.array_equal(acc, A.astype(np.int64) @ W.astype(np.int64).T)
    # W8A8 layer output approximates the fp64 product of the unrotated operands
    X = S.normal((16, 768), 1.0, seed=13)
    Wf = S.normal((96, 768), 0.02, seed=14)
    q, sx = oracle.hadamard_quant(X)
    wq, sw = oracle.prepare_linear(Wf)
    Y = oracle.dequant(oracle.gemm_i8(q, wq), sx, sw)
    ref = X.astype(np.float64) @ Wf.astype(np.float64).T
    assert np.sqrt(((Y - ref) ** 2).mean()) < 0.02 * np.sqrt((ref ** 2).mean())
    Yr = oracle.dequant(oracle.gemm_i8(q, wq), sx, sw, residual=np.ones_like(Y))
    assert np.array_equal(Yr, np.float32(1.0) + Y)


def test_in_proj_split_order(oracle):
    di, cc, nh = 64, 96, 3
    acc = S.uniform_ints((5, di + cc + nh), -5000, 5000, seed=15)
    sx = np.full(5, 0.01, np.float32)
    sw = np.full(di + cc + nh, 0.5, np.float32)
    e_u = np.full(cc, -3, np.int32)
    z, xbc, dt = oracle.in_proj_epilogue(acc, sx, sw, di, cc, nh, e_u)
    Y = oracle.dequant(acc, sx, sw)
    assert np.array_equal(z, Y[:, :di]) and np.array_equal(dt, Y[:, di + cc:])
    ref = np.clip(np.rint(Y[:, di:di + cc].astype(np.float64) * 8.0), -127, 127)
    assert np.array_equal(xbc, ref)


# ------------------------------------------------------------------ nonlinear unit

def _chord_rel_bound():
    """Max relative error of 8-chord interpolation of 2^f on [0,1) (fine grid, fp64)."""
    f = np.linspace(0.0, 0.125, 200001)
    chord = 1.0 + (2.0 ** 0.125 - 1.0) * f / 0.125
    return float(np.max(chord / 2.0 ** f - 1.0))


def test_pow2_pwl_exact_points_and_bound(oracle):
    k = np.arange(0, 17)
    assert np.array_equal(oracle.eval_array("pow2", -k * 65536), 65536 >> k)   # 2^-k exact
    seg = np.arange(0, 8)
    pts = oracle.eval_array("pow2", -65536 + seg * 8192)                       # f = i/8
    assert np.all(np.abs(pts - 65536.0 * 2.0 ** (-1 + seg / 8)) <= 0.5)
    w = np.arange(-16 * 65536, 1)
    got = oracle.eval_array("pow2", w).astype(np.float64)
    exact = 65536.0 * np.exp2(w / 65536.0)
    bound = _chord_rel_bound()
    assert 9.3e-4 < bound < 9.5e-4
    assert np.all(np.abs(got - exact) <= bound * exact + 1.0)
    assert np.all(np.diff(got) >= 0)                                           # monotone
    assert oracle.eval_array("pow2", np.array([-18 * 65536]))[0] == 0


def test_exp_pwl_bound(oracle):
    x = np.arange(-12 * 65536, 1, 7)
    got = oracle.eval_array("exp", x).astype(np.float64)
    exact = 65536.0 * np.exp(x / 65536.0)
    rel = _chord_rel_bound() + 1.2e-4 * (np.abs(x) / 65536.0 + 1.0)
    assert np.all(np.abs(got - exact) <= rel * exact + 1.5)


def test_softplus_symmetry_and_eq5_error(oracle):
    v = np.arange(1, 8 * 65536, 13)
    pos = oracle.eval_array("softplus", v)
    neg = oracle.eval_array("softplus", -v)
    assert np.array_equal(pos - v, neg)                  # SoftPlus(x) = x + SoftPlus(-x)
    assert oracle.eval_array("softplus", np.array([0]))[0] == 65536
    # Eq. (5) error on x <= 0: 0 <= e^x - ln(1+e^x) <= e^(2x)/2, plus the PWL error
    x = -v / 65536.0
    exact_sp = np.log1p(np.exp(x))
    got = neg / 65536.0
    tol = np.exp(2 * x) / 2 + (_chord_rel_bound() + 1.2e-4 * (np.abs(x) + 1)) * np.exp(x) + 2 / 65536
    assert np.all(np.abs(got - exact_sp) <= tol)


def test_silu_pwl(oracle):
    x = np.arange(-10 * 65536, 10 * 65536, 11)
    got = oracle.eval_array("silu", x).astype(np.float64) / 65536.0
    xf = x / 65536.0
    exact = xf / (1 + np.exp(-xf))
    assert oracle.eval_array("silu", np.array([0]))[0] == 0
    # sigma = 1/(1+E) or E/(1+E) moves by at most dE (|d sigma/dE| <= 1) plus one
    # truncation LSB; dE <= PWL relative error * E + 1 LSB; the product rounds once.
    rel = _chord_rel_bound() + 1.2e-4 * (np.abs(xf) + 1.0)
    d_sigma = rel * np.exp(-np.abs(xf)) + 2.0 / 65536
    assert np.all(np.abs(got - exact) <= np.abs(xf) * d_sigma + 1.0 / 65536)
    # silu(x) - silu(-x) = x: the two truncated sigmas sum to 1 within one LSB
    # (|x| LSB after the product), plus the two final roundings
    a = oracle.eval_array("silu", x) - oracle.eval_array("silu", -x)
    assert np.all(np.abs(a - x) <= np.abs(xf) + 1.0)


def test_to_q16(oracle):
    f = np.array([0.0, 1.0, -1.5, 2.0 ** -17, 3 * 2.0 ** -17, 1e9, -1e9, np.nan], np.float32)
    got = oracle.eval_array("to_q16", f)
    assert list(got) == [0, 65536, -98304, 0, 2, 2 ** 31 - 1, -(2 ** 31 - 1), 0]


def test_rshr_definition(oracle):
    a = np.arange(-40, 41)
    got = oracle.eval_array("rshr", a, shift=3)
    assert np.array_equal(got, np.floor((a + 4) / 8).astype(np.int64))
    assert np.array_equal(oracle.eval_array("rshr", a, shift=-2), a * 4)


@pytest.mark.parametrize("amax,Q", [(1.0, 127.0), (127.0, 127.0), (128.0, 127.0), (3e-7, 2.0 ** 29),
                                    (2.0 ** 40, 2.0 ** 29), (0.75, 32767.0)])
def test_pot_exponent(oracle, amax, Q):
    e = oracle.pot_exponent(amax, Q)
    assert amax <= Q * 2.0 ** e and amax > Q * 2.0 ** (e - 1)


# ------------------------------------------------------------------ conv

def test_conv_matches_library_convolution(oracle):
    import torch
    Bsz, T, cc = 2, 37, 48
    u = S.uniform_ints((Bsz, T, cc), -127, 127, seed=20, dtype=np.int8)
    w = S.normal((cc, 4), 0.2, seed=21)
    b = S.normal(cc, 0.5, seed=22)
    e_u = S.uniform_ints(cc, -6, -2, seed=23)
    wq, bq, e_w = oracle.prepare_conv(w, b, e_u)
    e_o = np.full(cc, -4, np.int32)
    state = S.uniform_ints((Bsz, 3, cc), -127, 127, seed=24, dtype=np.int8)
    st = state.copy()
    out, am = oracle.conv1d_pot(u, wq, bq, e_u, e_w, e_o, conv_state=st, want_amax=True)
    # integer accumulation via torch depthwise conv1d (cross-correlation) over [state | u]
    full = np.concatenate([state, u], axis=1).astype(np.float64)
    acc = torch.nn.functional.conv1d(torch.tensor(full).permute(0, 2, 1),
                                     torch.tensor(wq.astype(np.float64))[:, None, :],
                                     groups=cc).permute(0, 2, 1).numpy() + bq
    real = acc * np.exp2(e_w + e_u)
    ref = real / (1 + np.exp(-real))                     # SiLU of the real-valued accumulation
    got = out * 2.0 ** -4
    assert np.all(np.abs(got - np.clip(ref, -127 / 16, 127 / 16)) <= 2.0 ** -5 + 2e-3 * np.abs(ref) + 1e-3)
    assert np.array_equal(st, u[:, -3:])                 # new state = last three inputs
    assert np.all(am > 0)
    # the Q.16 SiLU values before requantisation (per-token exponent reading):
    # the SiLU of the real-valued accumulation within the PWL SiLU's bound
    _, s16 = oracle.conv1d_pot(u, wq, bq, e_u, e_w, e_o, conv_state=state.copy(), want_s16=True)
    sv = s16 / 65536.0
    rel = _chord_rel_bound() + 1.2e-4 * (np.abs(real) + 1.0)
    bound = np.abs(real) * (rel * np.exp(-np.abs(real)) + 2.0 / 65536) + 2.0 / 65536
    assert np.all(np.abs(sv - ref) <= bound)
    assert np.abs(ref).max() > 4.0                       # spans the nonlinear range


def test_conv_state_chunking_bit_exact(oracle):
    Bsz, T, cc = 1, 20, 32
    u = S.uniform_ints((Bsz, T, cc), -127, 127, seed=25, dtype=np.int8)
    wq, bq, e_w = oracle.prepare_conv(S.normal((cc, 4), 0.2, seed=26), np.zeros(cc, np.float32),
                                      np.full(cc, -3, np.int32))
    args = (wq, bq, np.full(cc, -3, np.int32), e_w, np.full(cc, -5, np.int32))
    full = oracle.conv1d_pot(u, *args)
    for split in (1, 2, 3, 7):
        st = np.zeros((Bsz, 3, cc), np.int8)
        a = oracle.conv1d_pot(u[:, :split].copy(), *args, conv_state=st)
        b = oracle.conv1d_pot(u[:, split:].copy(), *args, conv_state=st)
        assert np.array_equal(np.concatenate([a, b], 1), full)


# ------------------------------------------------------------------ scan

def _scan_inputs(Bsz=1, T=24, nh=2, hd=8, ds=16, seed=30):
    cc = nh * hd + 2 * ds
    xbc = S.uniform_ints((Bsz, T, cc), -127, 127, seed=seed, dtype=np.int8)
    dt_raw = S.normal((Bsz, T, nh), 1.5, seed=seed + 1)
    dt_bias = np.full(nh, -3.0, np.float32)
    A_q, D_q, e_D = oracle_prepare_ssm(nh, seed + 2)
    e_x = np.full(nh, -5, np.int32)
    return xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x


def oracle_prepare_ssm(nh, seed):
    import oracle as O
    a_log = np.log(S.normal(nh, 0.0, seed) + np.linspace(1.0, 16.0, nh)).astype(np.float32)
    return O.prepare_ssm(a_log, np.ones(nh, np.float32))


def test_ssm_prepare(oracle):
    A_q, D_q, e_D = oracle.prepare_ssm(np.log(np.array([1.0, 2.0, 16.0], np.float32)),
                                       np.array([1.0, 0.5, -3.0], np.float32))
    assert list(A_q) == [round(a / np.log(2) * 4096) for a in (1.0, 2.0, 16.0)]
    assert list(D_q * 2.0 ** e_D) == [1.0, 0.5, -3.0]


def test_scan_zero_dt_keeps_state(oracle):
    xbc, _, dt_bias, A_q, D_q, e_D, e_x = _scan_inputs()
    dt_raw = np.full((1, 24, 2), -1e4, np.float32)       # softplus ~ e^-1e4 -> dt = 0, dA = 1
    st0 = S.uniform_ints((1, 2, 8, 16), -10 ** 6, 10 ** 6, seed=40)
    st = st0.copy()
    _, dtq, dA = oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, -5, -5,
                                     np.full(2, -15, np.int32), np.full(2, -10, np.int32), e_D,
                                     8, 16, state=st, want_dt=True)
    assert not dtq.any() and np.all(dA == 65536)
    assert np.array_equal(st, st0)


def test_scan_one_hot_B_isolates_column(oracle):
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x = _scan_inputs()
    nh, hd, ds = 2, 8, 16
    xbc[..., nh * hd:nh * hd + ds] = 0
    xbc[..., nh * hd + 5] = 100                          # B = 100 e_5
    st = np.zeros((1, nh, hd, ds), np.int32)
    oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, -5, -5, np.full(nh, -14, np.int32),
                        np.full(nh, -10, np.int32), e_D, hd, ds, state=st)
    assert np.any(st[..., 5] != 0)
    assert not np.delete(st, 5, axis=-1).any()


def test_scan_against_double_recurrence(oracle):
    """Fixed-point state vs the naive fp64 recurrence on the same (dequantised)
    inputs, within the rounding budget: each step adds at most 1/2 LSB from the
    decay and |B|/2 LSB from the dt*x factor."""
    Bsz, T, nh, hd, ds = 1, 48, 2, 8, 16
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x = _scan_inputs(Bsz, T, nh, hd, ds, seed=50)
    e_B = e_C = -5
    e_h = np.full(nh, -20, np.int32)
    e_y = np.full(nh, -6, np.int32)
    st = np.zeros((Bsz, nh, hd, ds), np.int32)
    y, dtq, dA = oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D,
                                     hd, ds, state=st, want_dt=True)
    x = xbc[..., :nh * hd].reshape(Bsz, T, nh, hd) * 2.0 ** -5
    Bm = xbc[..., nh * hd:nh * hd + ds] * 2.0 ** e_B
    Cm = xbc[..., nh * hd + ds:] * 2.0 ** e_C
    dtr = dtq / 65536.0
    h = np.zeros((Bsz, nh, hd, ds))
    for t in range(T):
        h = (dA[:, t] / 65536.0)[:, :, None, None] * h + (dtr[:, t, :, None] * x[:, t])[..., None] \
            * Bm[:, t, None, None, :]
    lsb = 2.0 ** e_h[0]
    budget = T * (0.5 + 0.5 * 127 + 1) * lsb
    assert np.max(np.abs(st * lsb - h)) <= budget
    assert np.max(np.abs(h)) > 100 * budget                # the check is not vacuous


def test_scan_chunking_bit_exact(oracle):
    Bsz, T, nh, hd, ds = 2, 30, 2, 8, 16
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x = _scan_inputs(Bsz, T, nh, hd, ds, seed=60)
    args = (dt_bias, A_q, D_q, e_x, -5, -5, np.full(nh, -13, np.int32), np.full(nh, -6, np.int32),
            e_D, hd, ds)
    st_full = np.zeros((Bsz, nh, hd, ds), np.int32)
    y_full = oracle.ssm_scan_pot(xbc, dt_raw, *args, state=st_full)
    st = np.zeros_like(st_full)
    ya = oracle.ssm_scan_pot(xbc[:, :11].copy(), dt_raw[:, :11].copy(), *args, state=st)
    yb = oracle.ssm_scan_pot(xbc[:, 11:].copy(), dt_raw[:, 11:].copy(), *args, state=st)
    assert np.array_equal(np.concatenate([ya, yb], 1), y_full)
    assert np.array_equal(st, st_full)


# ------------------------------------------------------------------ fp64 reference

def test_reference_scan_matches_dual_quadratic_form(oracle):
    """Structured state-space duality (the paper's reference [2]): y_t = sum_{s<=t}
    (C_t . B_s) exp(sum_{r=s+1..t} dt_r A) dt_s x_s + D x_t."""
    rng = np.random.default_rng(0)
    Bsz, T, nh, hd, ds = 1, 12, 2, 3, 4
    xs = rng.standard_normal((Bsz, T, nh, hd))
    Bm = rng.standard_normal((Bsz, T, ds))
    Cm = rng.standard_normal((Bsz, T, ds))
    dt = rng.uniform(0.01, 0.5, (Bsz, T, nh))
    A = -rng.uniform(1, 4, nh)
    D = rng.standard_normal(nh)
    y, _ = oracle.ref_scan_f64(xs, Bm, Cm, dt, A, D)
    for h in range(nh):
        cum = np.cumsum(dt[0, :, h] * A[h])
        L = np.tril(np.exp(cum[:, None] - cum[None, :]))
        G = (Cm[0] @ Bm[0].T) * L * dt[0, None, :, h]
        ref = G @ xs[0, :, h, :] + D[h] * xs[0, :, h, :]
        assert np.allclose(y[0, :, h, :], ref, rtol=1e-12, atol=1e-12)


def test_reference_conv_matches_torch(oracle):
    import torch
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 9, 5))
    w = rng.standard_normal((5, 4))
    b = rng.standard_normal(5)
    got = oracle.ref_conv_f64(x, w, b)
    ref = torch.nn.functional.conv1d(torch.tensor(x).permute(0, 2, 1), torch.tensor(w)[:, None],
                                     torch.tensor(b), padding=3, groups=5)[..., :9]
    assert np.allclose(got, ref.permute(0, 2, 1).numpy(), rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------ whole layer

SMALL = S.MixerShape(d_model=256, d_inner=512, headdim=64, d_state=128)


@pytest.fixture(scope="module")
def small_layers(oracle):
    P = S.layer_params(SMALL, 3)
    xc = S.calibration_batch(256, 64, 4, 50.0, outlier_seed=99, n_seqs=2)
    out = {}
    for rot in (1, 0):
        L = oracle.prepare_layer(P, SMALL, rotate=rot)
        oracle.calibrate_layer(L, xc)
        out[rot] = L
    return P, out


def test_layer_sqnr_and_rotation(oracle, small_layers):
    P, Ls = small_layers
    x = S.activations(1, 64, 256, seed=5, n_outliers=4, outlier_scale=50.0, outlier_seed=99)
    ref = oracle.ref_mixer_f64(P, SMALL, x)
    s_rot = oracle.sqnr_db(ref, oracle.mixer_prefill(Ls[1], x))
    s_plain = oracle.sqnr_db(ref, oracle.mixer_prefill(Ls[0], x))
    # measured 20.6 dB rotated, 18.6 dB not: the floor sits 1.6 dB below
    assert s_rot > 19.0
    assert s_rot > s_plain


def test_layer_chunked_and_decode_bit_exact(oracle, small_layers):
    _, Ls = small_layers
    L = Ls[1]
    s = SMALL
    x = S.activations(2, 10, 256, seed=6, n_outliers=4, outlier_scale=50.0, outlier_seed=99)
    cs = np.zeros((2, 3, s.conv_ch), np.int8)
    ss = np.zeros((2, s.nheads, s.headdim, s.d_state), np.int32)
    full = oracle.mixer_prefill(L, x, conv_state=cs, ssm_state=ss)
    cs2, ss2 = np.zeros_like(cs), np.zeros_like(ss)
    parts = [oracle.mixer_prefill(L, x[:, :4].copy(), conv_state=cs2, ssm_state=ss2)]
    for t in range(4, 10):                              # decode steps: one token each
        parts.append(oracle.mixer_prefill(L, x[:, t:t + 1].copy(), conv_state=cs2, ssm_state=ss2))
    assert np.array_equal(np.concatenate(parts, 1), full)
    assert np.array_equal(cs2, cs) and np.array_equal(ss2, ss)


def test_calibrated_exponents_fit_their_codes(oracle):
    """Each calibrated power-of-two exponent is the smallest e with
    amax <= Q 2^e, so on the calibration set itself the largest code of every
    group lands in [64, 127]: conv input codes per channel, conv output codes
    per head (x) and for B and C; in static mode the largest in_proj input
    code is 127 and the static scale is the calibration set's amax."""
    s = SMALL
    P = S.layer_params(s, 4)
    xc = S.calibration_batch(256, 64, 4, 50.0, outlier_seed=99, n_seqs=2)
    L = oracle.prepare_layer(P, s, rotate=1, mode=oracle.STATIC)
    oracle.calibrate_layer(L, xc)
    tr = {}
    oracle.mixer_prefill(L, xc, trace=tr)
    u = np.abs(tr["xbc"].reshape(-1, s.conv_ch).astype(np.int32)).max(0)
    assert u.min() >= 64 and u.max() <= 127
    co = np.abs(tr["conv_out"].reshape(-1, s.conv_ch).astype(np.int32))
    per_head = co[:, :s.d_inner].reshape(-1, s.nheads, s.headdim).max(axis=(0, 2))
    assert per_head.min() >= 64 and per_head.max() <= 127
    for part in (co[:, s.d_inner:s.d_inner + s.d_state], co[:, s.d_inner + s.d_state:]):
        assert 64 <= part.max() <= 127
    assert np.abs(tr["q_in"].astype(np.int32)).max() == 127
    assert np.abs(tr["q_out"].astype(np.int32)).max() == 127


def test_scan_state_amax_no_decay_closed_form(oracle):
    """The calibration statistic of the state (64-bit state at the finest
    exponent, u = rshr(dt_q x, 1), no clamp) against a closed form: with A = 0
    the decay is exactly 2^0 (65536 in Q.16), so the state is the running sum
    of u_t B_t[n]; with B one-hot (code 1 at one n) and positive x codes it
    grows monotonically, and its maximum over the head is
    max_p sum_t rshr(dt_q[t] x[t, p], 1), dt_q taken from the scan's own
    dt output."""
    nh, hd, ds, T = 2, 64, 128, 24
    di = nh * hd
    xbc = np.zeros((1, T, di + 2 * ds), np.int8)
    xbc[0, :, :di] = S.uniform_ints((T, di), 1, 127, seed=31, dtype=np.int8)
    xbc[0, :, di + 5] = 1                                    # B = e_5
    xbc[0, :, di + ds:] = S.uniform_ints((T, ds), -127, 127, seed=32, dtype=np.int8)  # C
    dt_raw = S.normal((1, T, nh), 1.0, seed=33)
    dt_bias = np.array([0.5, -1.0], np.float32)
    A_q = np.zeros(nh, np.int32)
    am = oracle.scan_state_amax(xbc, dt_raw, dt_bias, A_q, hd, ds)
    z = np.zeros(nh, np.int32)
    _, dtq, dA = oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, z + 16384, z - 4, -4, -4, z - 12,
                                     z - 12, z - 14, hd, ds, want_dt=True)
    assert (dA == 65536).all()
    x = xbc[0, :, :di].astype(np.int64).reshape(T, nh, hd)
    u = (dtq[0].astype(np.int64)[:, :, None] * x + 1) >> 1   # rshr(., 1) = floor((v + 1) / 2)
    expect = u.sum(axis=0).max(axis=1)
    assert np.array_equal(am, expect)
    assert (expect > 0).all()


def test_output_statistic_skip_term_closed_form(oracle):
    """The calibration statistic of the scan output (max |y| at the finer of
    the two term exponents) against a closed form: with B = 0 the state stays
    0, so only the skip term D x remains; with e_D + e_x the finer exponent it
    enters unshifted and the statistic is max_{t,p} |D_q x[t, p]| per head."""
    nh, hd, ds, T = 2, 64, 128, 12
    di = nh * hd
    xbc = np.zeros((1, T, di + 2 * ds), np.int8)
    xbc[0, :, :di] = S.uniform_ints((T, di), -127, 127, seed=41, dtype=np.int8)
    xbc[0, :, di + ds:] = S.uniform_ints((T, ds), -127, 127, seed=42, dtype=np.int8)  # C, B = 0
    dt_raw = S.normal((1, T, nh), 1.0, seed=43)
    dt_bias = np.zeros(nh, np.float32)
    A_q = np.array([4000, 9000], np.int32)
    D_q = np.array([16384, -9000], np.int32)
    e_x, e_D = np.array([-4, -5], np.int32), np.array([-14, -13], np.int32)
    e_B, e_C = -4, -3
    e_h = np.array([-2, -3], np.int32)            # e_C + e_h = -5 / -6 > e_D + e_x = -18
    e_y = np.array([-10, -10], np.int32)
    _, ys = oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D,
                                hd, ds, want_ystat=True)
    x = xbc[0, :, :di].astype(np.int64).reshape(T, nh, hd)
    expect = np.abs(D_q.astype(np.int64)[None, :, None] * x).max(axis=(0, 2))
    assert np.array_equal(ys, expect)


def test_gate_statistic_closed_form(oracle):
    """The calibration statistic of the gate (max |g| per head, g = y
    SiLU(z) in Q.16) against a closed form: for z >= 40, e^-z is below the
    2^v unit's smallest step, sigma is exactly 1 (2^16 in Q.16) and the PWL
    SiLU returns its input, so g = y rint(z 2^16)."""
    M, nh, hd = 5, 3, 64
    di = nh * hd
    y = S.uniform_ints((M, di), -2 ** 20, 2 ** 20, seed=51)
    z = (40.0 + 3.0 * np.abs(S.normal((M, di), 1.0, seed=52))).astype(np.float32)
    e_y = np.array([-20, -21, -19], np.int32)
    *_, gs = oracle.gate_norm_quant(y, z, hd, e_y, -20, np.ones(di, np.float32), want_gstat=True)
    z16 = np.rint(z.astype(np.float64) * 65536.0).astype(np.int64)
    g = np.abs(y.astype(np.int64) * z16).reshape(M, nh, hd)
    assert np.array_equal(gs, g.max(axis=(0, 2)))


def _gated_norm_case(M=6, nh=3, hd=64, seed=53):
    """Inputs on which the gate and the int16 gated code are exact: z = 64
    exactly, so z16 = 2^22, e^-z is below the 2^v unit's smallest step and
    the PWL SiLU returns z16 unchanged; with e_g = e_y + 6 the gated code is
    rshr(y 2^22, 22) = y.  The gated value is then y 2^e_y times z, exactly.
    Rows 0-2 are large (the norm is a plain RMS); rows 3-5 are scaled so that
    mean(g^2) is near or below eps = 1e-5 (eps then sets the scale)."""
    di = nh * hd
    y = S.uniform_ints((M, di), -30000, 30000, seed=seed)
    y[3:5] //= 256                                 # mean(g^2) near eps in rows 3, 4
    y[5] //= 2048                                  # and well below it in row 5
    z = np.full((M, di), 64.0, np.float32)
    e_y = np.full(nh, -20, np.int32)
    e_g = -14
    w = (0.5 + 1.5 * S.uniform_ints(di, 0, 1000, seed=seed + 1) / 1000.0).astype(np.float32)
    g = y.astype(np.float64) * 2.0 ** -20 * 64.0   # the gated value, exact
    return y, z, hd, e_y, e_g, w, g


def _gated_norm_f64(g, w, eps=1e-5):
    """Mamba2's gated RMSNorm (gate first, then normalise over all of d_inner
    with one group), the paper's reference [10] (RMSNorm) and its Figure 2
    block flow, in fp64."""
    return g / np.sqrt((g * g).mean(axis=1, keepdims=True) + eps) * w.astype(np.float64)


def test_gated_rmsnorm_closed_form(oracle):
    """The gate + gated RMSNorm against its fp64 definition, on inputs where
    the gate is exact (_gated_norm_case): the norm uses eps = 1e-5, the
    per-channel weight, and the mean over d_inner.  Without rotation the
    dequantised output is within half a quantisation step of the fp64 value
    (plus fp32 rounding); the rows where eps dominates pin eps itself."""
    y, z, hd, e_y, e_g, w, g = _gated_norm_case()
    o = _gated_norm_f64(g, w)
    ms = (g * g).mean(axis=1)
    assert ms[0] > 1e3 * 1e-5 and ms[5] < 1e-5 < 1e3 * ms[5]
    for mode, amax in ((oracle.DYNAMIC, 0.0), (oracle.STATIC, 1.25 * np.abs(o).max())):
        q, sx = oracle.gate_norm_quant(y, z, hd, e_y, e_g, w, rotate=0, mode=mode,
                                       static_amax=amax)
        deq = q.astype(np.float64) * sx.astype(np.float64)[:, None] if mode == oracle.DYNAMIC \
            else q.astype(np.float64) * float(sx[0])
        step = sx.astype(np.float64)[:, None] if mode == oracle.DYNAMIC else float(sx[0])
        err = np.abs(deq - o)
        assert (err <= 0.5 * step + 1e-6 * np.abs(o) + 1e-30).all()
        if mode == oracle.DYNAMIC:              # the row maximum maps to 127
            assert (np.abs(q).max(axis=1) == 127).all()
    # other eps, dropped weights, a mean over a part of d_inner: each is off
    q, sx = oracle.gate_norm_quant(y, z, hd, e_y, e_g, w, rotate=0)
    deq = q.astype(np.float64) * sx.astype(np.float64)[:, None]
    for wrong in (_gated_norm_f64(g, w, eps=1e-3), _gated_norm_f64(g, np.ones_like(w)),
                  g / np.sqrt((g[:, :hd] ** 2).mean(axis=1, keepdims=True) + 1e-5) * w):
        assert not (np.abs(deq - wrong) <= 0.5 * sx[:, None] + 1e-6 * np.abs(wrong)).all()


def test_gated_rmsnorm_rotated_closed_form(oracle):
    """With the rotation on, the codes dequantise to the rotated fp64 output
    o H (block 256) within half a step, so inverting the (orthonormal)
    rotation gives o back within the step's L2 bound."""
    y, z, hd, e_y, e_g, w, g = _gated_norm_case(nh=4)
    o = _gated_norm_f64(g, w)
    di = o.shape[1]
    H = hadamard_bd(di)
    q, sx = oracle.gate_norm_quant(y, z, hd, e_y, e_g, w, rotate=1)
    deq = q.astype(np.float64) * sx.astype(np.float64)[:, None]
    assert (np.abs(deq - o @ H) <= 0.5 * sx[:, None] + 1e-6 * np.abs(o @ H).max()).all()
    back = deq @ H.T
    assert (np.linalg.norm(back - o, axis=1) <= 0.5 * sx * np.sqrt(di) * (1 + 1e-6)).all()


# ------------------------------------------------------------------ state word width

def test_narrow_state_clamps_at_its_width(oracle):
    """A 16-bit state word: with no decay (A = 0, dA exactly 1) and a one-hot
    B the state is the running sum of u * B clamped at 2^15 - 1, closed form
    min(sum_t u_t * 127, 32767) in the hot column and 0 elsewhere; the 31-bit
    word does not clamp on the same input."""
    nh, hd, ds, T = 1, 8, 16, 40
    di = nh * hd
    xbc = np.zeros((1, T, di + 2 * ds), np.int8)
    xbc[0, :, :di] = S.uniform_ints((T, di), 20, 127, seed=71, dtype=np.int8)
    xbc[0, :, di + 3] = 127                                  # B = 127 e_3
    dt_raw = S.normal((1, T, nh), 1.0, seed=72)
    z = np.zeros(nh, np.int32)
    args = (np.array([0.5], np.float32), z, z + 16384, z - 4, -4, -4, z - 9, z - 12, z - 14, hd,
            ds)
    sums = {}
    for bits in (16, 31):
        st = np.zeros((1, nh, hd, ds), np.int32)
        _, dtq, dA = oracle.ssm_scan_pot(xbc, dt_raw, *args, state=st, want_dt=True,
                                         state_bits=bits)
        assert (dA == 65536).all()
        s_h = -9 - (-4) - (-4) + 16                          # e_h - e_B - e_x + 16
        x = xbc[0, :, :di].astype(np.int64)
        u = (dtq[0].astype(np.int64) * x + (1 << (s_h - 1))) >> s_h     # rshr(dt_q x, s_h)
        total = (u * 127).sum(axis=0)
        lim = (1 << (bits - 1)) - 1
        assert np.array_equal(st[0, 0, :, 3], np.minimum(total, lim))
        assert not np.delete(st, 3, axis=-1).any()
        sums[bits] = total
    assert (sums[16] > 32767).all()                          # the narrow word really clamps


def test_narrow_state_against_double_recurrence(oracle):
    """A 16-bit state at a coarser exponent stays within the same per-step
    rounding budget of the naive fp64 recurrence, when the exponent leaves
    room for the running maximum plus the budget (so nothing clamps)."""
    Bsz, T, nh, hd, ds = 1, 48, 2, 8, 16
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x = _scan_inputs(Bsz, T, nh, hd, ds, seed=50)
    e_B = e_C = -5
    e_h = np.full(nh, -10, np.int32)
    st = np.zeros((Bsz, nh, hd, ds), np.int32)
    _, dtq, dA = oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h,
                                     np.full(nh, -6, np.int32), e_D, hd, ds, state=st,
                                     want_dt=True, state_bits=16)
    x = xbc[..., :nh * hd].reshape(Bsz, T, nh, hd) * 2.0 ** -5
    Bm = xbc[..., nh * hd:nh * hd + ds] * 2.0 ** e_B
    h = np.zeros((Bsz, nh, hd, ds))
    peak = 0.0
    for t in range(T):
        h = (dA[:, t] / 65536.0)[:, :, None, None] * h + \
            (dtq[:, t, :, None] / 65536.0 * x[:, t])[..., None] * Bm[:, t, None, None, :]
        peak = max(peak, float(np.abs(h).max()))
    lsb = 2.0 ** e_h[0]
    budget = T * (0.5 + 0.5 * 127 + 1) * lsb
    assert (peak + budget) / lsb < 2 ** 15 - 1               # the word never clamps
    assert np.max(np.abs(st * lsb - h)) <= budget
    assert peak > 5 * budget                                 # the check is not vacuous


# ------------------------------------------------------------------ per-token conv-output exponents

def _token_case(oracle, seed=81, Bsz=2, T=30, nh=2, hd=8, ds=16):
    """Random Q.16 SiLU values with per-token magnitudes spread over 2^10."""
    cc = nh * hd + 2 * ds
    mag = np.exp2(S.uniform_ints((Bsz, T, 1), 0, 10, seed=seed)).astype(np.int64)
    s16 = (S.uniform_ints((Bsz, T, cc), -2 ** 14, 2 ** 14, seed=seed + 1).astype(np.int64)
           * mag // 4).astype(np.int32)
    e_o = np.concatenate([np.repeat(np.array([-2, -3], np.int32), hd),
                          np.full(ds, -1, np.int32), np.full(ds, -2, np.int32)])
    return s16, e_o


def test_per_token_exponents_fit_their_codes(oracle):
    """E(amax, 127) is the smallest exponent that holds the token's group
    maximum: the largest code of each (token, group) is in [64, 127] unless
    the floor (16 below the static exponent) applies; zero groups give 0."""
    nh, hd, ds = 2, 8, 16
    s16, e_o = _token_case(oracle)
    s16[0, 3, :hd] = 0                                       # an all-zero head group
    codes, e_tok = oracle.requant_per_token(s16, nh, hd, ds, e_o)
    groups = [slice(h * hd, (h + 1) * hd) for h in range(nh)] + \
        [slice(nh * hd, nh * hd + ds), slice(nh * hd + ds, nh * hd + 2 * ds)]
    floors = [e_o[g.start] - 16 for g in groups]
    for b in range(s16.shape[0]):
        for t in range(s16.shape[1]):
            for g, (sl, fl) in enumerate(zip(groups, floors)):
                top = np.abs(codes[b, t, sl].astype(np.int64)).max()
                e = e_tok[b, t, g]
                assert e >= fl
                if np.abs(s16[b, t, sl]).max() == 0:
                    assert top == 0
                elif e > fl:
                    assert 64 <= top <= 127, (b, t, g, top)
                # dequantised codes within half a step of the value
                err = np.abs(codes[b, t, sl] * 2.0 ** e - s16[b, t, sl] / 65536.0)
                assert err.max() <= 2.0 ** e / 2 + 1e-12


def test_scan_with_static_exponents_per_token_is_the_static_scan(oracle):
    Bsz, T, nh, hd, ds = 2, 20, 2, 8, 16
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x = _scan_inputs(Bsz, T, nh, hd, ds, seed=90)
    e_h, e_y = np.full(nh, -13, np.int32), np.full(nh, -6, np.int32)
    e_tok = np.empty((Bsz, T, nh + 2), np.int32)
    e_tok[..., :nh], e_tok[..., nh], e_tok[..., nh + 1] = e_x, -5, -4
    args = (dt_bias, A_q, D_q, e_x, -5, -4, e_h, e_y, e_D, hd, ds)
    s1, s2 = (np.zeros((Bsz, nh, hd, ds), np.int32) for _ in range(2))
    y1, ys1 = oracle.ssm_scan_pot(xbc, dt_raw, *args, state=s1, want_ystat=True)
    y2, ys2 = oracle.ssm_scan_pot(xbc, dt_raw, *args, state=s2, want_ystat=True, e_tok=e_tok)
    assert np.array_equal(y1, y2) and np.array_equal(s1, s2) and np.array_equal(ys1, ys2)
    a1 = oracle.scan_state_amax(xbc, dt_raw, dt_bias, A_q, hd, ds)
    a2 = oracle.scan_state_amax(xbc, dt_raw, dt_bias, A_q, hd, ds, e_tok, e_x, -5)
    assert np.array_equal(a1, a2)


def test_per_token_scan_against_double_recurrence(oracle):
    """Per-token exponents for x, B, C: the fixed-point state and output
    against the naive fp64 recurrence on the values the codes stand for,
    within the per-step rounding budget (a sign or offset slip in any
    per-token shift moves the result by powers of two)."""
    Bsz, T, nh, hd, ds = 1, 40, 2, 8, 16
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, _ = _scan_inputs(Bsz, T, nh, hd, ds, seed=95)
    e_tok = S.uniform_ints((Bsz, T, nh + 2), -9, -5, seed=96)
    e_x, e_B, e_C = np.full(nh, -5, np.int32), -5, -5        # the static references
    e_h, e_y = np.full(nh, -22, np.int32), np.full(nh, -14, np.int32)
    st = np.zeros((Bsz, nh, hd, ds), np.int32)
    y, dtq, dA = oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y,
                                     e_D, hd, ds, state=st, want_dt=True, e_tok=e_tok)
    x = xbc[..., :nh * hd].reshape(Bsz, T, nh, hd) * np.exp2(e_tok[..., :nh, None])
    Bm = xbc[..., nh * hd:nh * hd + ds] * np.exp2(e_tok[..., nh, None])
    Cm = xbc[..., nh * hd + ds:] * np.exp2(e_tok[..., nh + 1, None])
    D = D_q * 2.0 ** e_D
    h = np.zeros((Bsz, nh, hd, ds))
    yr = np.empty((Bsz, T, nh, hd))
    for t in range(T):
        h = (dA[:, t] / 65536.0)[:, :, None, None] * h + \
            (dtq[:, t, :, None] / 65536.0 * x[:, t])[..., None] * Bm[:, t, None, None, :]
        yr[:, t] = np.einsum("bhpn,bn->bhp", h, Cm[:, t]) + D[None, :, None] * x[:, t]
    lsb = 2.0 ** -22
    budget = T * (0.5 + 0.5 * 127 + 1) * lsb
    assert np.max(np.abs(st * lsb - h)) <= budget
    assert np.max(np.abs(h)) > 100 * budget
    # output: the state error times sum |C|, plus the two output roundings
    ybud = budget * np.abs(Cm).sum(-1).max() + 2 ** -14
    assert np.max(np.abs(y.reshape(Bsz, T, nh, hd) * 2.0 ** -14 - yr)) <= ybud
    assert np.max(np.abs(yr)) > 50 * ybud


def test_per_token_layer_chunking_and_gain(oracle):
    """A layer with per-token conv-output exponents: chunked prefill plus
    decode steps equal one prefill bit for bit (the exponents depend on the
    token alone), and on outlier inputs it is closer to fp64 than the
    static-exponent layer."""
    P = S.layer_params(SMALL, 3)
    xc = S.calibration_batch(256, 64, 4, 50.0, outlier_seed=99, n_seqs=2)
    Ls = {}
    for xe in ("static", "token"):
        Ls[xe] = oracle.prepare_layer(P, SMALL, xbc_exponents=xe)
        oracle.calibrate_layer(Ls[xe], xc)
    L, s = Ls["token"], SMALL
    x = S.activations(2, 10, 256, seed=6, n_outliers=4, outlier_scale=50.0, outlier_seed=99)
    cs0, ss0 = np.zeros((2, 3, s.conv_ch), np.int8), np.zeros((2, s.nheads, s.headdim, s.d_state),
                                                              np.int32)
    full = oracle.mixer_prefill(L, x, conv_state=cs0, ssm_state=ss0)
    cs, ss = np.zeros_like(cs0), np.zeros_like(ss0)
    parts = [oracle.mixer_prefill(L, x[:, :7].copy(), conv_state=cs, ssm_state=ss)]
    for t in range(7, 10):
        parts.append(oracle.mixer_prefill(L, x[:, t:t + 1].copy(), conv_state=cs, ssm_state=ss))
    assert np.array_equal(np.concatenate(parts, 1), full)
    assert np.array_equal(cs, cs0) and np.array_equal(ss, ss0)
    xt = S.activations(1, 64, 256, seed=5, n_outliers=4, outlier_scale=50.0, outlier_seed=99)
    ref = oracle.ref_mixer_f64(P, SMALL, xt)
    gain = oracle.sqnr_db(ref, oracle.mixer_prefill(Ls["token"], xt)) - \
        oracle.sqnr_db(ref, oracle.mixer_prefill(Ls["static"], xt))
    assert gain > 0.5, gain


def test_guard_bit_rounding_tightens_the_narrow_state_budget(oracle):
    """Rounding the state increment after the u B product (7 guard bits on u)
    bounds each step's rounding by about one state LSB (decay 1/2, u 2^-8 per
    unit of |B| <= 127, product 1/2), against |B|/2 LSBs when u is rounded
    first: a 16-bit state then tracks the fp64 recurrence within 1.6 LSB per
    step, which the as-built rounding exceeds on the same input."""
    Bsz, T, nh, hd, ds = 1, 48, 2, 8, 16
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x = _scan_inputs(Bsz, T, nh, hd, ds, seed=50)
    e_B = e_C = -5
    e_h = np.full(nh, -10, np.int32)
    X = xbc[..., :nh * hd].reshape(Bsz, T, nh, hd) * 2.0 ** -5
    Bm = xbc[..., nh * hd:nh * hd + ds] * 2.0 ** e_B
    lsb = 2.0 ** e_h[0]
    err = {}
    for g in (0, 7):
        st = np.zeros((Bsz, nh, hd, ds), np.int32)
        _, dtq, dA = oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h,
                                         np.full(nh, -6, np.int32), e_D, hd, ds, state=st,
                                         want_dt=True, state_bits=16, ub_guard=g)
        h = np.zeros((Bsz, nh, hd, ds))
        for t in range(T):
            h = (dA[:, t] / 65536.0)[:, :, None, None] * h + \
                (dtq[:, t, :, None] / 65536.0 * X[:, t])[..., None] * Bm[:, t, None, None, :]
        err[g] = np.max(np.abs(st * lsb - h)) / lsb
    assert err[7] <= T * 1.6
    assert err[0] > T * 1.6                      # the pin tells the two roundings apart
    with pytest.raises(ValueError):
        oracle.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h,
                            np.full(nh, -6, np.int32), e_D, hd, ds, state_bits=31, ub_guard=7)


def test_candidate_spec_layer_chunking_and_gain(oracle):
    """Per-token conv-output exponents, a 16-bit state and the guard-bit
    increment together: chunked prefill plus decode steps equal one prefill
    bit for bit, the carried state stays inside 16 bits, and on outlier
    inputs the layer is closer to fp64 than the method as built."""
    P = S.layer_params(SMALL, 3)
    xc = S.calibration_batch(256, 64, 4, 50.0, outlier_seed=99, n_seqs=2)
    built = oracle.prepare_layer(P, SMALL)
    oracle.calibrate_layer(built, xc)
    L = oracle.prepare_layer(P, SMALL, state_bits=16, xbc_exponents="token", ub_guard=7)
    oracle.calibrate_layer(L, xc)
    s = SMALL
    x = S.activations(2, 12, 256, seed=16, n_outliers=4, outlier_scale=50.0, outlier_seed=99)
    cs0 = np.zeros((2, 3, s.conv_ch), np.int8)
    ss0 = np.zeros((2, s.nheads, s.headdim, s.d_state), np.int32)
    full = oracle.mixer_prefill(L, x, conv_state=cs0, ssm_state=ss0)
    cs, ss = np.zeros_like(cs0), np.zeros_like(ss0)
    parts = [oracle.mixer_prefill(L, x[:, :9].copy(), conv_state=cs, ssm_state=ss)]
    for t in range(9, 12):
        parts.append(oracle.mixer_prefill(L, x[:, t:t + 1].copy(), conv_state=cs, ssm_state=ss))
    assert np.array_equal(np.concatenate(parts, 1), full)
    assert np.array_equal(ss, ss0) and np.abs(ss0).max() <= 2 ** 15 - 1
    xt = S.activations(1, 64, 256, seed=5, n_outliers=4, outlier_scale=50.0, outlier_seed=99)
    ref = oracle.ref_mixer_f64(P, SMALL, xt)
    gain = oracle.sqnr_db(ref, oracle.mixer_prefill(L, xt)) - \
        oracle.sqnr_db(ref, oracle.mixer_prefill(built, xt))
    assert gain > 0.5, gain
