"""GPU parity of every kernel against the CPU oracle, through the C ABI.

Integer codes, int32 accumulators and all fixed-point stages must be
bit-exact; fp32 outputs computed from identical codes by the same IEEE
operations in the same order must be bit-exact too.  Sizes span several
tiles with ragged tails.
"""
import numpy as np
import pytest

import oracle as O
from quantized_state_space_mamba2_b200 import synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MAMBA130 = S.MAMBA2_130M


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_state_space_mamba2_b200 import build, lib
    build.build()
    lib.load()
    return lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


# ------------------------------------------------------------------ nonlinear unit

@pytest.mark.parametrize("kind,name,lo,hi", [(0, "pow2", -20 * 65536, 0), (1, "exp", -20 * 65536, 0),
                                             (2, "softplus", -12 * 65536, 12 * 65536),
                                             (3, "silu", -40 * 65536, 40 * 65536)])
def test_pwl_exhaustive(L, kind, name, lo, hi):
    x = np.arange(lo, hi + 1, dtype=np.int64)
    out = torch.empty(x.size, dtype=torch.int64, device="cuda")
    L.eval_pwl(kind, dev(x), out)
    assert np.array_equal(host(out), O.eval_array(name, x))
    L.sync_status()


def test_pwl_extremes_and_to_q16(L):
    x = np.array([-(2 ** 31) + 1, -(2 ** 31) + 1000, -1, 0, 1, 2 ** 31 - 1, 123456789, -98765432],
                 np.int64)
    out = torch.empty(x.size, dtype=torch.int64, device="cuda")
    for kind, name in ((2, "softplus"), (3, "silu")):
        L.eval_pwl(kind, dev(x), out)
        assert np.array_equal(host(out), O.eval_array(name, x))
    f = np.concatenate([S.normal(4096, 3.0, seed=1), S.normal(64, 1e5, seed=2),
                        np.array([0.0, -0.0, 1e30, -1e30, np.inf, -np.inf, np.nan, 2.0 ** -20,
                                  32767.99], np.float32)]).astype(np.float32)
    bits = f.view(np.uint32).astype(np.int64)
    out = torch.empty(bits.size, dtype=torch.int64, device="cuda")
    L.eval_pwl(4, dev(bits), out)
    assert np.array_equal(host(out), O.eval_array("to_q16", f))


# ------------------------------------------------------------------ rotation + quantisation

@pytest.mark.parametrize("M,K", [(1, 256), (7, 768), (300, 768), (33, 2560), (5, 5120)])
@pytest.mark.parametrize("rotate", [1, 0])
def test_hadamard_quant_dynamic(L, M, K, rotate):
    x = S.activations(1, M, K, seed=M + K, n_outliers=8, outlier_scale=50.0)[0]
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    am = torch.empty(M, dtype=torch.float32, device="cuda")
    L.hadamard_quant(dev(x), K, None, rotate, 0, None, q, sx, am)
    qr, sr, ar = O.hadamard_quant(x, None, rotate, O.DYNAMIC, want_amax=True)
    assert np.array_equal(host(q), qr)
    assert np.array_equal(host(sx), sr)
    assert np.array_equal(host(am), ar)


@pytest.mark.parametrize("K", [768, 2560])
def test_hadamard_quant_prenorm_static(L, K):
    M = 130
    x = S.activations(1, M, K, seed=9, n_outliers=8, outlier_scale=50.0)[0]
    w = (1.0 + S.normal(K, 0.1, seed=10)).astype(np.float32)
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    L.hadamard_quant(dev(x), K, dev(w), 1, 0, None, q, sx)
    qr, sr = O.hadamard_quant(x, w, 1, O.DYNAMIC)
    assert np.array_equal(host(q), qr) and np.array_equal(host(sx), sr)
    amax = np.float32(3.5)
    L.hadamard_quant(dev(x), K, dev(w), 1, 1, dev(np.array([amax, 0, 0, 0], np.float32)), q, sx)
    qr, sr = O.hadamard_quant(x, w, 1, O.STATIC, float(amax))
    assert np.array_equal(host(q), qr) and np.array_equal(host(sx), sr)


@pytest.mark.parametrize("N,K", [(3352, 768), (768, 1536), (40, 5120)])
def test_prepare_linear(L, N, K):
    W = S.normal((N, K), 0.02, seed=N)
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, dtype=torch.float32, device="cuda")
    for rot in (1, 0):
        L.prepare_linear(dev(W), rot, wq, sw)
        wr, sr = O.prepare_linear(W, rot)
        assert np.array_equal(host(wq), wr) and np.array_equal(host(sw), sr)


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("M,N,K", [(1, 24, 128), (100, 136, 256), (256, 3352, 768),
                                   (300, 768, 1536), (129, 257, 640), (2048, 768, 1536)])
def test_w8a8_gemm(L, M, N, K):
    A = S.uniform_ints((M, K), -127, 127, seed=M * 3 + K, dtype=np.int8)
    W = S.uniform_ints((N, K), -127, 127, seed=N * 5 + K, dtype=np.int8)
    sx = np.abs(S.normal(M, 0.01, seed=1)) + 1e-3
    sw = np.abs(S.normal(N, 0.001, seed=2)) + 1e-4
    res = S.normal((M, N), 1.0, seed=3)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Y, None, acc)
    ref = A.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(host(acc), ref)
    assert np.array_equal(host(Y), O.dequant(ref.astype(np.int32), sx, sw))
    Yr = dev(res)
    L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Yr, Yr, None)    # residual aliasing Y
    assert np.array_equal(host(Yr), O.dequant(ref.astype(np.int32), sx, sw, residual=res))
    L.sync_status()


@pytest.mark.parametrize("M,N,K", [(64, 2560, 5120), (1, 768, 1536), (37, 100, 1152),
                                   (16, 1000, 256)])
def test_w8a8_gemm_cluster_split(L, M, N, K):
    """Decode-size GEMMs with fewer 32-wide tiles than SMs, K split over a
    thread-block cluster (2..8 ranks, the last rank's slice ragged where K
    does not divide): the int32 accumulator, the dequantised output and the
    residual form are bit-identical to one CTA per tile and to the exact
    product."""
    A = S.uniform_ints((M, K), -127, 127, seed=M * 3 + K + 1, dtype=np.int8)
    W = S.uniform_ints((N, K), -127, 127, seed=N * 5 + K + 1, dtype=np.int8)
    sx = np.abs(S.normal(M, 0.01, seed=11)) + 1e-3
    sw = np.abs(S.normal(N, 0.001, seed=12)) + 1e-4
    res = S.normal((M, N), 1.0, seed=13)
    ref = A.astype(np.int64) @ W.astype(np.int64).T
    outs = []
    for on in (True, False):
        L.set_gemm_cluster(on)
        try:
            Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
            acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
            L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Y, None, acc)
            Yr = dev(res)
            L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Yr, Yr, None)
            L.sync_status()
            outs.append((host(acc), host(Y), host(Yr)))
        finally:
            L.set_gemm_cluster(L.GEMM_CLUSTER_DEFAULT)
    (a1, y1, r1), (a0, y0, r0) = outs
    assert np.array_equal(a1, ref) and np.array_equal(a0, ref)
    assert np.array_equal(y1, y0) and np.array_equal(r1, r0)
    assert np.array_equal(y1, O.dequant(ref.astype(np.int32), sx, sw))
    assert np.array_equal(r1, O.dequant(ref.astype(np.int32), sx, sw, residual=res))


def _sample_rows(M, step=7, tail=130):
    return np.unique(np.concatenate([np.arange(0, M, step), np.arange(max(0, M - tail), M)]))


@pytest.mark.parametrize("M,N,K", [(2093, 3352, 768), (4173, 10576, 2560), (8192, 2560, 5120)])
def test_w8a8_gemm_persistent(L, M, N, K):
    """Grids with at least one 128-wide tile per SM run the persistent kernel
    (128 x 128 tiles; 128 x 256 from two tiles per SM on; accumulators
    double-buffered in TMEM, ring and tiles carried across the CTA's tiles).
    Ragged M and N; every 7th row and the last 130 rows (the partial tile)
    compared bit for bit."""
    A = S.uniform_ints((M, K), -127, 127, seed=M + K, dtype=np.int8)
    W = S.uniform_ints((N, K), -127, 127, seed=N + K, dtype=np.int8)
    sx = np.abs(S.normal(M, 0.01, seed=7)) + 1e-3
    sw = np.abs(S.normal(N, 0.001, seed=8)) + 1e-4
    res = S.normal((M, N), 1.0, seed=9)
    rows = _sample_rows(M)
    ref = (A[rows].astype(np.float64) @ W.astype(np.float64).T).astype(np.int64)  # exact: |acc| < 2^53
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Y, None, acc)
    assert np.array_equal(host(acc)[rows], ref)
    assert np.array_equal(host(Y)[rows], O.dequant(ref.astype(np.int32), sx[rows], sw))
    Yr = dev(res)
    L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Yr, Yr, None)
    assert np.array_equal(host(Yr)[rows],
                          O.dequant(ref.astype(np.int32), sx[rows], sw, residual=res[rows]))
    L.sync_status()


def test_in_proj_split_2p7b_full_size(L):
    """The in_proj split epilogue at the 2.7B shapes and 8192 tokens (the
    persistent 128 x 256 kernel), sampled rows bit for bit."""
    s, M = S.MAMBA2_2P7B, 8192
    A = S.uniform_ints((M, s.d_model), -127, 127, seed=21, dtype=np.int8)
    W = S.uniform_ints((s.n_in, s.d_model), -127, 127, seed=22, dtype=np.int8)
    sx = np.abs(S.normal(M, 0.01, seed=23)) + 1e-3
    sw = np.abs(S.normal(s.n_in, 3e-3, seed=24)) + 1e-4
    e_u = S.uniform_ints(s.conv_ch, -6, -2, seed=25)
    exps = np.zeros(L.exp_table_layout(s).size, np.int32)
    exps[:s.conv_ch] = e_u
    z = torch.empty((M, s.d_inner), dtype=torch.float32, device="cuda")
    xbc = torch.empty((M, s.conv_ch), dtype=torch.int8, device="cuda")
    dt = torch.empty((M, s.nheads), dtype=torch.float32, device="cuda")
    L.in_proj(dev(A), dev(sx), dev(W), dev(sw), s, dev(exps), z, xbc, dt)
    rows = _sample_rows(M, step=13)
    acc = (A[rows].astype(np.float64) @ W.astype(np.float64).T).astype(np.int32)
    zr, xr, dr = O.in_proj_epilogue(acc, sx[rows], sw, s.d_inner, s.conv_ch, s.nheads, e_u)
    assert np.array_equal(host(z)[rows], zr)
    assert np.array_equal(host(xbc)[rows], xr)
    assert np.array_equal(host(dt)[rows], dr)


@pytest.mark.parametrize("M", [5, 256, 1000])
def test_in_proj_split(L, M):
    s = MAMBA130
    A = S.uniform_ints((M, s.d_model), -127, 127, seed=M, dtype=np.int8)
    W = S.uniform_ints((s.n_in, s.d_model), -127, 127, seed=M + 1, dtype=np.int8)
    sx = np.abs(S.normal(M, 0.01, seed=4)) + 1e-3
    sw = np.abs(S.normal(s.n_in, 5e-3, seed=5)) + 1e-4
    e_u = S.uniform_ints(s.conv_ch, -6, -2, seed=6)
    exps = np.zeros(L.exp_table_layout(s).size, np.int32)
    exps[:s.conv_ch] = e_u
    z = torch.empty((M, s.d_inner), dtype=torch.float32, device="cuda")
    xbc = torch.empty((M, s.conv_ch), dtype=torch.int8, device="cuda")
    dt = torch.empty((M, s.nheads), dtype=torch.float32, device="cuda")
    L.in_proj(dev(A), dev(sx), dev(W), dev(sw), s, dev(exps), z, xbc, dt)
    acc = (A.astype(np.int64) @ W.astype(np.int64).T).astype(np.int32)
    zr, xr, dr = O.in_proj_epilogue(acc, sx, sw, s.d_inner, s.conv_ch, s.nheads, e_u)
    assert np.array_equal(host(z), zr)
    assert np.array_equal(host(xbc), xr)
    assert np.array_equal(host(dt), dr)
    assert np.abs(xr).max() == 127 and (xr == 0).mean() < 0.5   # codes exercise the range


# ------------------------------------------------------------------ conv

def _conv_case(s, seed):
    cc = s.conv_ch
    w = S.normal((cc, 4), 0.2, seed=seed)
    b = S.normal(cc, 0.3, seed=seed + 1)
    e_u = S.uniform_ints(cc, -5, -1, seed=seed + 2)
    wq, bq, e_w = O.prepare_conv(w, b, e_u)
    e_x = S.uniform_ints(s.nheads, -5, -3, seed=seed + 3)
    e_B, e_C = -4, -3
    e_o = np.concatenate([np.repeat(e_x, s.headdim), np.full(s.d_state, e_B),
                          np.full(s.d_state, e_C)]).astype(np.int32)
    return w, wq, bq, e_u, e_w, e_o


@pytest.mark.parametrize("B,T", [(1, 1), (2, 5), (1, 37), (2, 300), (1, 2048)])
@pytest.mark.parametrize("with_state", [False, True])
def test_conv1d_pot(L, B, T, with_state):
    s = MAMBA130
    cc = s.conv_ch
    _, wq, bq, e_u, e_w, e_o = _conv_case(s, 40)
    exps = np.zeros(L.exp_table_layout(s).size, np.int32)
    exps[:cc], exps[cc:2 * cc], exps[2 * cc:3 * cc] = e_u, e_w, e_o
    u = S.uniform_ints((B, T, cc), -127, 127, seed=B * 1000 + T, dtype=np.int8)
    st = S.uniform_ints((B, 3, cc), -127, 127, seed=7, dtype=np.int8) if with_state else None
    out = torch.empty((B, T, cc), dtype=torch.int8, device="cuda")
    st_d = dev(st) if with_state else None
    L.conv1d_pot(dev(u), B, T, s, dev(wq), dev(bq), dev(exps), st_d, out)
    st_r = st.copy() if with_state else None
    ref = O.conv1d_pot(u, wq, bq, e_u, e_w, e_o, conv_state=st_r)
    assert np.array_equal(host(out), ref)
    if with_state:
        assert np.array_equal(host(st_d), st_r)


@pytest.mark.parametrize("B,T", [(1, 1), (2, 37)])
def test_conv1d_pot_extreme_exponents(L, B, T):
    """Per-channel exponents and biases far from a calibrated layer's: large
    left shifts that saturate the Q.16 input, right shifts past 29, biases
    beyond 2^29, output shifts from -5 to 40.  Threads whose four channels
    all stay clear of saturation and overflow take the kernel's short path,
    the others its general 64-bit form; both must equal the oracle."""
    s = MAMBA130
    cc = s.conv_ch
    wq = S.uniform_ints((cc, 4), -127, 127, seed=301, dtype=np.int8)
    bq = S.uniform_ints(cc, -2 ** 12, 2 ** 12, seed=302)
    big = S.uniform_ints(cc, 0, 29, seed=303) == 0           # ~3 % of channels
    bq = np.where(big, S.uniform_ints(cc, -2 ** 30, 2 ** 30, seed=304), bq).astype(np.int32)
    wild = S.uniform_ints(cc, 0, 19, seed=309) < 3          # ~15 % of channels
    s_in = np.where(wild, S.uniform_ints(cc, -30, 35, seed=305),
                    S.uniform_ints(cc, -10, 10, seed=310))
    s_out = np.where(wild, S.uniform_ints(cc, -5, 40, seed=306),
                     S.uniform_ints(cc, 10, 24, seed=311))
    e_u = S.uniform_ints(cc, -8, 2, seed=307).astype(np.int32)
    e_w = (-(s_in + 16) - e_u).astype(np.int32)
    e_o = (s_out - 16).astype(np.int32)
    exps = np.zeros(L.exp_table_layout(s).size, np.int32)
    exps[:cc], exps[cc:2 * cc], exps[2 * cc:3 * cc] = e_u, e_w, e_o
    u = S.uniform_ints((B, T, cc), -127, 127, seed=308 + T, dtype=np.int8)
    out = torch.empty((B, T, cc), dtype=torch.int8, device="cuda")
    L.conv1d_pot(dev(u), B, T, s, dev(wq), dev(bq), dev(exps), None, out)
    ref = O.conv1d_pot(u, wq, bq, e_u, e_w, e_o)
    assert np.array_equal(host(out), ref)
    # both regimes occur: saturated Q.16 inputs and channels on the short path
    assert (np.abs(ref) == 127).mean() > 0.02 and (np.abs(ref) < 127).mean() > 0.5


def test_prepare_mixer_params(L):
    s = MAMBA130
    P = S.layer_params(s, 11, conv_bias_std=0.1)
    conv_wq = torch.empty((s.conv_ch, 4), dtype=torch.int8, device="cuda")
    A_q = torch.empty(s.nheads, dtype=torch.int32, device="cuda")
    D_q = torch.empty(s.nheads, dtype=torch.int32, device="cuda")
    exps = torch.zeros(L.exp_table_layout(s).size, dtype=torch.int32, device="cuda")
    D = (S.normal(s.nheads, 1.0, seed=12)).astype(np.float32)
    L.prepare_mixer_params(s, dev(P["conv_w"]), dev(P["a_log"]), dev(D), conv_wq, A_q, D_q, exps)
    wq, _, e_w = O.prepare_conv(P["conv_w"], P["conv_b"])
    Aq, Dq, eD = O.prepare_ssm(P["a_log"], D)
    X = L.exp_table_layout(s)
    e = host(exps)
    assert np.array_equal(host(conv_wq), wq)
    assert np.array_equal(e[X.e_w:X.e_w + s.conv_ch], e_w)
    assert np.array_equal(host(A_q), Aq) and np.array_equal(host(D_q), Dq)
    assert np.array_equal(e[X.e_D:X.e_D + s.nheads], eD)


# ------------------------------------------------------------------ scan

def _scan_case(s, B, T, seed):
    cc, nh = s.conv_ch, s.nheads
    xbc = S.uniform_ints((B, T, cc), -127, 127, seed=seed, dtype=np.int8)
    dt_raw = S.normal((B, T, nh), 2.0, seed=seed + 1)
    P = S.layer_params(s, seed)
    A_q, D_q, e_D = O.prepare_ssm(P["a_log"], P["D"])
    e_x = S.uniform_ints(nh, -5, -3, seed=seed + 2)
    e_B, e_C = -4, -3
    e_h = (e_x + e_B - 15 + S.uniform_ints(nh, 2, 8, seed=seed + 3)).astype(np.int32)
    e_y = (np.maximum(e_C + e_h, e_D + e_x) - S.uniform_ints(nh, 0, 6, seed=seed + 4)).astype(np.int32)
    return xbc, dt_raw, P["dt_bias"], A_q, D_q, e_D, e_x, e_B, e_C, e_h, e_y


def _exps_for_scan(L, s, e_x, e_B, e_C, e_h, e_y, e_D):
    X = L.exp_table_layout(s)
    nh = s.nheads
    e = np.zeros(X.size, np.int32)
    e[X.e_x:X.e_x + nh], e[X.e_B], e[X.e_C] = e_x, e_B, e_C
    e[X.e_h:X.e_h + nh], e[X.e_y:X.e_y + nh], e[X.e_D:X.e_D + nh] = e_h, e_y, e_D
    return e


def _run_scan(L, s, B, T, with_state, seed):
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x, e_B, e_C, e_h, e_y = _scan_case(s, B, T, seed)
    exps = _exps_for_scan(L, s, e_x, e_B, e_C, e_h, e_y, e_D)
    st = S.uniform_ints((B, s.nheads, s.headdim, s.d_state), -2 ** 26, 2 ** 26,
                        seed=5) if with_state else None
    y = torch.empty((B, T, s.d_inner), dtype=torch.int32, device="cuda")
    st_d = dev(st) if with_state else None
    ws = torch.empty(L.scan_workspace_bytes(s, B, T), dtype=torch.uint8, device="cuda")
    L.ssm_scan_pot(dev(xbc), dev(dt_raw), B, T, s, dev(dt_bias), dev(A_q), dev(D_q), dev(exps),
                   st_d, y, ws)
    st_r = st.copy() if with_state else None
    yr = O.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D,
                        s.headdim, s.d_state, state=st_r)
    assert np.array_equal(host(y), yr)
    if with_state:
        assert np.array_equal(host(st_d), st_r)


@pytest.mark.parametrize("B,T", [(1, 1), (2, 33), (1, 100), (1, 513)])
@pytest.mark.parametrize("with_state", [False, True])
def test_ssm_scan_pot(L, B, T, with_state):
    _run_scan(L, MAMBA130, B, T, with_state, 60 + T)


@pytest.mark.parametrize("tile", [(4, 4, 16), (4, 2, 16), (4, 8, 16), (8, 4, 16), (8, 2, 16),
                                  (8, 8, 16), (4, 8, 32)])
def test_ssm_scan_tiles(L, tile):
    """Every compiled tile of the sequential kernel computes the same bits
    (ragged chunk tail, carried state, two heads' worth of CTAs per SM)."""
    L.set_scan_tile(*tile)
    try:
        _run_scan(L, MAMBA130, 2, 45, True, 70)
    finally:
        L.set_scan_tile(*L.SCAN_TILE_DEFAULT)


def test_ssm_scan_2p7b_shape(L):
    _run_scan(L, S.MAMBA2_2P7B, 1, 37, True, 80)


@pytest.mark.parametrize("shape,B", [("130m", 3), ("2p7b", 64)])
def test_ssm_scan_decode_step(L, shape, B):
    """T = 1 runs the single-step decode kernel (no staging): same bits as
    the oracle's one recurrence step, state updated in place."""
    s = MAMBA130 if shape == "130m" else S.MAMBA2_2P7B
    _run_scan(L, s, B, 1, True, 85)


def test_ssm_scan_decode_step_clamped(L):
    """One decode step from a state at the clamp with saturated inputs: the
    single-step kernel clamps exactly like the oracle."""
    s = MAMBA130
    B, T = 2, 1
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x, e_B, e_C, e_h, e_y = _scan_case(s, B, T, 95)
    e_h = (e_x + e_B - 16 - 4).astype(np.int32)
    dt_raw = np.zeros_like(dt_raw)
    xbc[..., :s.d_inner] = 127
    xbc[..., s.d_inner:s.d_inner + s.d_state] = np.where(
        S.uniform_ints((B, T, s.d_state), 0, 1, seed=96) > 0, 127, -127).astype(np.int8)
    e_y = (np.maximum(e_C + e_h, e_D + e_x) - 2).astype(np.int32)
    exps = _exps_for_scan(L, s, e_x, e_B, e_C, e_h, e_y, e_D)
    lim = 2 ** 30 - 1
    st = np.where(S.uniform_ints((B, s.nheads, s.headdim, s.d_state), 0, 1, seed=97) > 0,
                  lim, -lim).astype(np.int32)
    y = torch.empty((B, T, s.d_inner), dtype=torch.int32, device="cuda")
    st_d = dev(st)
    ws = torch.empty(L.scan_workspace_bytes(s, B, T), dtype=torch.uint8, device="cuda")
    L.ssm_scan_pot(dev(xbc), dev(dt_raw), B, T, s, dev(dt_bias), dev(A_q), dev(D_q), dev(exps),
                   st_d, y, ws)
    yr = O.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D,
                        s.headdim, s.d_state, state=st)
    assert np.array_equal(host(y), yr)
    assert np.array_equal(host(st_d), st)
    assert (np.abs(st) == lim).mean() > 0.2


@pytest.mark.parametrize("T", [1, 40])
def test_ssm_scan_skip_term_beyond_int32(L, T):
    """Exponents where both output terms exceed int32 before they are added
    (s_D = -12, s_y = s_D - 15): the skip term rshr(D_q x, s_D) is formed in
    64 bits and the sum saturates once, as the oracle does -- outputs whose two
    terms cancel back into range must match exactly (sequential and
    single-step kernels)."""
    s = MAMBA130
    B = 2
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x, e_B, e_C, e_h, e_y = _scan_case(s, B, T, 111)
    e_h = (e_D + e_x - e_C - 15).astype(np.int32)
    e_y = (e_D + e_x - 12).astype(np.int32)
    exps = _exps_for_scan(L, s, e_x, e_B, e_C, e_h, e_y, e_D)
    st = S.uniform_ints((B, s.nheads, s.headdim, s.d_state), -2 ** 26, 2 ** 26, seed=112)
    y = torch.empty((B, T, s.d_inner), dtype=torch.int32, device="cuda")
    st_d = dev(st)
    ws = torch.empty(L.scan_workspace_bytes(s, B, T), dtype=torch.uint8, device="cuda")
    L.ssm_scan_pot(dev(xbc), dev(dt_raw), B, T, s, dev(dt_bias), dev(A_q), dev(D_q), dev(exps),
                   st_d, y, ws)
    yr = O.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D,
                        s.headdim, s.d_state, state=st)
    assert np.array_equal(host(y), yr)
    assert np.array_equal(host(st_d), st)
    # the case is exercised: skip terms beyond int32 with an unsaturated output
    x = xbc[..., :s.d_inner].astype(np.int64).reshape(B, T, s.nheads, s.headdim)
    skip = (D_q.astype(np.int64)[None, None, :, None] * x) << 12
    big = np.abs(skip.reshape(B, T, s.d_inner)) > 2 ** 31 - 1
    assert (big & (np.abs(yr.astype(np.int64)) < 2 ** 31 - 1)).sum() > 0


@pytest.mark.parametrize("tile", [(4, 4, 16), (4, 4, 32)])
@pytest.mark.parametrize("regime", ["saturating", "small"])
def test_ssm_scan_clamp_regimes(L, regime, tile):
    """The sequential kernel skips the clamp for a chunk only when
    max|h| + sum |u| max|B| stays below it; both regimes must match the oracle:
    a state driven into the +-(2^30 - 1) clamp, and one that never nears it
    (16- and 32-step chunks: the latter add two 16-step bounds)."""
    L.set_scan_tile(*tile)
    try:
        _clamp_regime(L, regime)
    finally:
        L.set_scan_tile(*L.SCAN_TILE_DEFAULT)


def _clamp_regime(L, regime):
    s = MAMBA130
    B, T = 1, 160
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x, e_B, e_C, e_h, e_y = _scan_case(s, B, T, 90)
    if regime == "saturating":
        e_h = (e_x + e_B - 16 - 4).astype(np.int32)          # s_h = -4: u saturates at 2^23
        dt_raw = np.zeros_like(dt_raw)                        # dt = softplus(bias), small
        xbc[..., :s.d_inner] = 127
        xbc[..., s.d_inner:s.d_inner + s.d_state] = 127       # B = 127 everywhere
    else:
        e_h = (e_x + e_B - 15 + 12).astype(np.int32)          # s_h = 13: small u
    e_y = (np.maximum(e_C + e_h, e_D + e_x) - 2).astype(np.int32)
    exps = _exps_for_scan(L, s, e_x, e_B, e_C, e_h, e_y, e_D)
    st = np.zeros((B, s.nheads, s.headdim, s.d_state), np.int32)
    y = torch.empty((B, T, s.d_inner), dtype=torch.int32, device="cuda")
    st_d = dev(st)
    ws = torch.empty(L.scan_workspace_bytes(s, B, T), dtype=torch.uint8, device="cuda")
    L.ssm_scan_pot(dev(xbc), dev(dt_raw), B, T, s, dev(dt_bias), dev(A_q), dev(D_q), dev(exps),
                   st_d, y, ws)
    yr = O.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D,
                        s.headdim, s.d_state, state=st)
    assert np.array_equal(host(y), yr)
    assert np.array_equal(host(st_d), st)
    lim = 2 ** 30 - 1
    if regime == "saturating":
        assert (np.abs(st) == lim).mean() > 0.5
    else:
        assert np.abs(st).max() < lim // 4 and np.abs(st).max() > 1000


# ------------------------------------------------------------------ gate + norm

@pytest.mark.parametrize("M", [1, 77, 512])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("di", [1536, 768, 5120])
@pytest.mark.parametrize("shift", ["small", "large"])
def test_gate_norm_quant(L, M, mode, di, shift):
    """d_inner with an even number of 256-blocks (two per warp) and an odd one
    (one per warp).  The gate shift e_g - e_y + 16 per head: 14..18 ("small",
    the 64-bit form) or 32..36 ("large": heads at 33 and above take the
    high-word form, the head at 32 the 64-bit one, and the largest products
    saturate the int16 gated code)."""
    s = S.MixerShape(d_model=768, d_inner=di, headdim=64, d_state=128)
    y = S.uniform_ints((M, s.d_inner), -2 ** 29, 2 ** 29, seed=M, dtype=np.int32)
    z = S.normal((M, s.d_inner), 3.0, seed=M + 1)
    e_y = S.uniform_ints(s.nheads, -22, -18, seed=M + 2)
    e_g = int(e_y.max()) - 16 + (14 if shift == "small" else 32)
    w = (1.0 + S.normal(s.d_inner, 0.2, seed=9)).astype(np.float32)
    X = L.exp_table_layout(s)
    exps = np.zeros(X.size, np.int32)
    exps[X.e_y:X.e_y + s.nheads] = e_y
    exps[X.e_g] = e_g
    amax = np.array([0.0, 2.5, 0, 0], np.float32)
    q = torch.empty((M, s.d_inner), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    am = torch.empty(M, dtype=torch.float32, device="cuda")
    L.gate_norm_quant(dev(y), dev(z), s, dev(exps), dev(w), 1, mode, dev(amax)[1:], q, sx, am)
    qr, sr, ar = O.gate_norm_quant(y, z, s.headdim, e_y, e_g, w, 1, mode, 2.5, want_amax=True)
    assert np.array_equal(host(q), qr)
    assert np.array_equal(host(sx), sr)
    assert np.array_equal(host(am), ar)
