"""The narrow state spec on the GPU (fm_set_state_spec(16, 7)): every scan
kernel (sequential prefill, decode step, calibration statistics) against the
oracle's 16-bit state with the guard-bit increment, bit for bit, the state
stored as int16; a calibrated layer's tables, prefill output, decode steps
and carried states likewise.
The spec is process-wide, so each test restores the default."""
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


@pytest.fixture
def spec16(L):
    L.set_state_spec(16, 7)
    yield
    L.set_state_spec(31, 0)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def _case(s, B, T, seed):
    cc, nh = s.conv_ch, s.nheads
    xbc = S.uniform_ints((B, T, cc), -127, 127, seed=seed, dtype=np.int8)
    dt_raw = S.normal((B, T, nh), 2.0, seed=seed + 1)
    P = S.layer_params(s, seed)
    A_q, D_q, e_D = O.prepare_ssm(P["a_log"], P["D"])
    e_x = S.uniform_ints(nh, -5, -3, seed=seed + 2)
    e_B, e_C = -4, -3
    # a 16-bit state: 2^14 headroom instead of 2^29
    e_h = (e_x + e_B - 15 + 15 + S.uniform_ints(nh, 2, 6, seed=seed + 3)).astype(np.int32)
    e_y = (np.maximum(e_C + e_h, e_D + e_x) - S.uniform_ints(nh, 0, 6, seed=seed + 4)).astype(np.int32)
    return xbc, dt_raw, P["dt_bias"], A_q, D_q, e_D, e_x, e_B, e_C, e_h, e_y


def _exps(L, s, e_x, e_B, e_C, e_h, e_y, e_D):
    X = L.exp_table_layout(s)
    nh = s.nheads
    e = np.zeros(X.size, np.int32)
    e[X.e_x:X.e_x + nh], e[X.e_B], e[X.e_C] = e_x, e_B, e_C
    e[X.e_h:X.e_h + nh], e[X.e_y:X.e_y + nh], e[X.e_D:X.e_D + nh] = e_h, e_y, e_D
    return e


@pytest.mark.parametrize("B,T", [(1, 1), (3, 1), (64, 1), (2, 33), (1, 513)])
def test_scan_state16_matches_oracle(L, spec16, B, T):
    s = MAMBA130
    xbc, dt_raw, dt_bias, A_q, D_q, e_D, e_x, e_B, e_C, e_h, e_y = _case(s, B, T, 300 + T)
    exps = _exps(L, s, e_x, e_B, e_C, e_h, e_y, e_D)
    st = S.uniform_ints((B, s.nheads, s.headdim, s.d_state), -20000, 20000, seed=9)
    y = torch.empty((B, T, s.d_inner), dtype=torch.int32, device="cuda")
    st_d = dev(st.astype(np.int16))                          # the narrow spec's storage
    ws = torch.empty(L.scan_workspace_bytes(s, B, T), dtype=torch.uint8, device="cuda")
    L.ssm_scan_pot(dev(xbc), dev(dt_raw), B, T, s, dev(dt_bias), dev(A_q), dev(D_q), dev(exps),
                   st_d, y, ws)
    L.sync_status()
    st_r = st.copy()
    yr = O.ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D, s.headdim,
                        s.d_state, state=st_r, state_bits=16, ub_guard=7)
    assert np.abs(st_r).max() <= 32767
    assert np.array_equal(host(y), yr)
    assert np.array_equal(host(st_d).astype(np.int32), st_r)


def test_layer_state16_matches_oracle(L, spec16):
    """Calibration (2^14 state headroom), a 130M prefill, two decode steps
    and the carried states, bit for bit against the oracle's layer with the
    same spec."""
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    s = MAMBA130
    P = S.layer_params(s, 1000)
    xcal = S.calibration_batch(s.d_model, 64, 8, 50.0, 4242, n_seqs=2)
    ol = O.prepare_layer(P, s, state_bits=16, ub_guard=7)
    O.calibrate_layer(ol, xcal)
    dl = DeviceLayer(P, s)
    dl.calibrate(dev(xcal))
    g = dl.exponents()
    for k in ("e_u", "e_x", "e_h", "e_y"):
        assert np.array_equal(g[k], getattr(ol, k)), k
    x = S.activations(2, 42, s.d_model, seed=3, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=4242)
    cs, ss = dl.new_states(2)
    out = dl.prefill(dev(x[:, :40]), conv_state=cs, ssm_state=ss)
    outs = [host(out)]
    for t in (40, 41):
        outs.append(host(dl.decode(dev(x[:, t]), cs, ss))[:, None])
    L.sync_status()
    cs_r = np.zeros((2, 3, s.conv_ch), np.int8)
    ss_r = np.zeros((2, s.nheads, s.headdim, s.d_state), np.int32)
    ref = O.mixer_prefill(ol, x, conv_state=cs_r, ssm_state=ss_r)
    assert np.array_equal(np.concatenate(outs, 1), ref)
    assert ss.dtype == torch.int16
    assert np.array_equal(host(cs), cs_r) and np.array_equal(host(ss).astype(np.int32), ss_r)
