"""Per-token conv-output exponents on the GPU (fm_set_xbc_exponents(1)): the
conv requantises each token's groups (a head's x channels, B, C) at their own
power-of-two exponent, and every scan kernel (sequential prefill, decode
step, calibration statistics) shifts by the token's exponents.  A calibrated
layer's tables, prefill output, decode steps and carried states equal the
oracle's layer with xbc_exponents="token" bit for bit, with the int32 state
as built and with the candidate spec of the 16-bit state and the guard-bit
increment.  The granularity and the state spec are process-wide, so each
test restores the defaults."""
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


@pytest.mark.parametrize("bits,guard", [(31, 0), (16, 7)])
@pytest.mark.parametrize("mode", [O.DYNAMIC, O.STATIC])
def test_layer_per_token_exponents_match_oracle(L, bits, guard, mode):
    """Calibration, a 130M prefill of 2 x 70 tokens (a ragged last 32-token
    staging tile), two decode steps and the carried states."""
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    s = MAMBA130
    L.set_xbc_exponents("token")
    L.set_state_spec(bits, guard)
    try:
        P = S.layer_params(s, 1000, conv_bias_std=0.05)
        xcal = S.calibration_batch(s.d_model, 64, 8, 50.0, 4242, n_seqs=2)
        ol = O.prepare_layer(P, s, mode=mode, state_bits=bits, xbc_exponents="token",
                             ub_guard=guard)
        O.calibrate_layer(ol, xcal)
        dl = DeviceLayer(P, s, mode=mode)
        dl.calibrate(dev(xcal))
        g = dl.exponents()
        for k in ("e_u", "e_x", "e_h", "e_y"):
            assert np.array_equal(g[k], getattr(ol, k)), k
        assert (g["e_B"], g["e_C"], g["e_g"]) == (ol.e_B, ol.e_C, ol.e_g)
        assert (g["amax_in"], g["amax_out"]) == (np.float32(ol.amax_in), np.float32(ol.amax_out))
        x = S.activations(2, 72, s.d_model, seed=3, n_outliers=8, outlier_scale=50.0,
                          outlier_seed=4242)
        cs, ss = dl.new_states(2)
        out = dl.prefill(dev(x[:, :70]), conv_state=cs, ssm_state=ss)
        outs = [host(out)]
        for t in (70, 71):
            outs.append(host(dl.decode(dev(x[:, t]), cs, ss))[:, None])
        L.sync_status()
        cs_r = np.zeros((2, 3, s.conv_ch), np.int8)
        ss_r = np.zeros((2, s.nheads, s.headdim, s.d_state), np.int32)
        ref = O.mixer_prefill(ol, x, conv_state=cs_r, ssm_state=ss_r)
        assert np.array_equal(np.concatenate(outs, 1), ref)
        assert np.array_equal(host(cs), cs_r)
        assert np.array_equal(host(ss).astype(np.int32), ss_r)
    finally:
        L.set_xbc_exponents("static")
        L.set_state_spec(31, 0)


def test_per_token_refused_by_the_chunked_scan(L):
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    s = MAMBA130
    L.set_xbc_exponents("token")
    L.set_scan_mode("ssd")
    try:
        dl = DeviceLayer(S.layer_params(s, 7), s)
        with pytest.raises(L.FmError) as e:
            dl.prefill(torch.zeros((1, 40, s.d_model), device="cuda"))
        assert e.value.status == 8
    finally:
        L.set_scan_mode("seq")
        L.set_xbc_exponents("static")


@pytest.mark.parametrize("B,T", [(1, 1), (2, 37), (1, 300)])
def test_standalone_per_token_conv_and_scan(L, B, T):
    """fm_conv1d_pot_tok and fm_ssm_scan_pot_tok (independent of the
    process-wide setting) against the oracle's per-token requantisation and
    scan, on a calibrated layer's tables and random in_proj codes."""
    s = MAMBA130
    P = S.layer_params(s, 1002, conv_bias_std=0.05)
    xcal = S.calibration_batch(s.d_model, 64, 8, 50.0, 4242, n_seqs=1)
    ol = O.prepare_layer(P, s, xbc_exponents="token")
    O.calibrate_layer(ol, xcal)
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    L.set_xbc_exponents("token")
    try:
        dl = DeviceLayer(P, s)
        dl.calibrate(dev(xcal))
    finally:
        L.set_xbc_exponents("static")
    u = S.uniform_ints((B, T, s.conv_ch), -127, 127, seed=61 + T, dtype=np.int8)
    dt_raw = S.normal((B, T, s.nheads), 1.0, seed=62 + T)
    st = S.uniform_ints((B, s.nheads, s.headdim, s.d_state), -2 ** 20, 2 ** 20, seed=63)
    xo = torch.empty((B, T, s.conv_ch), dtype=torch.int8, device="cuda")
    e_tok = torch.empty((B * T, s.nheads + 2), dtype=torch.int32, device="cuda")
    L.conv1d_pot_tok(dev(u), B, T, s, dl.conv_wq, dl.conv_bq, dl.exps, None, xo, e_tok)
    xo_r, et_r = O.conv_out(ol, u)
    assert np.array_equal(host(xo), xo_r)
    assert np.array_equal(host(e_tok).reshape(et_r.shape), et_r)
    y = torch.empty((B, T, s.d_inner), dtype=torch.int32, device="cuda")
    std = dev(st)
    ws = torch.empty(L.scan_workspace_bytes_tok(s, B, T), dtype=torch.uint8, device="cuda")
    L.ssm_scan_pot_tok(xo, dev(dt_raw), B, T, s, dl.dt_bias, dl.A_q, dl.D_q, dl.exps, e_tok, std,
                       y, ws)
    L.sync_status()
    st_r = st.copy()
    y_r = O.ssm_scan_pot(xo_r, dt_raw, ol.dt_bias, ol.A_q, ol.D_q, ol.e_x, ol.e_B, ol.e_C, ol.e_h,
                         ol.e_y, ol.e_D, s.headdim, s.d_state, state=st_r, e_tok=et_r)
    assert np.array_equal(host(y), y_r)
    assert np.array_equal(host(std), st_r)
