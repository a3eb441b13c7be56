"""GPU parity of whole layers against the CPU oracle, through the C ABI:
calibration (exponent tables and static scales), one-layer prefill in both
activation modes with and without rotation, chunked prefill with carried
state, decode steps, and a stack of layers."""
import numpy as np
import pytest

import oracle as O
from quantized_state_space_mamba2_b200 import synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPE = S.MAMBA2_130M
CFG0 = S.WORKLOADS["mixer130m_b1_t256"]
OUTLIER_SEED = 101


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_state_space_mamba2_b200 import build, lib
    build.build()
    lib.load()
    return lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def compare_exponents(gpu: dict, ol) -> None:
    for k in ("e_u", "e_x", "e_h", "e_y"):
        assert np.array_equal(gpu[k], getattr(ol, k)), k
    assert gpu["e_B"] == ol.e_B and gpu["e_C"] == ol.e_C and gpu["e_g"] == ol.e_g
    assert np.array_equal(gpu["e_w"], ol.conv_e_w) and np.array_equal(gpu["e_D"], ol.e_D)
    assert np.array_equal(gpu["conv_bq"], ol.conv_bq)
    assert np.float32(gpu["amax_in"]) == np.float32(ol.amax_in)
    assert np.float32(gpu["amax_out"]) == np.float32(ol.amax_out)


@pytest.fixture(scope="module", params=[(1, 0), (1, 1), (0, 0)], ids=["rot-dyn", "rot-static", "plain-dyn"])
def calibrated(request, env):
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    rotate, mode = request.param
    P = S.layer_params(SHAPE, 0, conv_bias_std=0.05)
    xcal = S.calibration_batch(SHAPE.d_model, 64, CFG0["n_outliers"], CFG0["outlier_scale"],
                               OUTLIER_SEED, n_seqs=3)
    ol = O.prepare_layer(P, SHAPE, rotate=rotate, mode=mode)
    out_o = O.calibrate_layer(ol, xcal)
    dl = DeviceLayer(P, SHAPE, rotate=rotate, mode=mode)
    out_g = dl.calibrate(dev(xcal))
    env.sync_status()
    return P, ol, dl, out_o, out_g.cpu().numpy()


def test_calibration_matches_oracle(calibrated):
    _, ol, dl, out_o, out_g = calibrated
    compare_exponents(dl.exponents(), ol)
    assert np.array_equal(out_g, out_o)


def test_prefill_config0_bit_exact(calibrated, env):
    _, ol, dl, _, _ = calibrated
    x = S.activations(1, CFG0["seqlen"], SHAPE.d_model, seed=1, n_outliers=CFG0["n_outliers"],
                      outlier_scale=CFG0["outlier_scale"], outlier_seed=OUTLIER_SEED)
    tr = {}
    ref = O.mixer_prefill(ol, x, trace=tr)
    got = dl.prefill(dev(x)).cpu().numpy()
    env.sync_status()
    assert np.array_equal(got, ref)


def test_chunked_prefill_and_decode(calibrated, env):
    _, ol, dl, _, _ = calibrated
    B, T = 2, 40
    x = S.activations(B, T, SHAPE.d_model, seed=2, n_outliers=CFG0["n_outliers"],
                      outlier_scale=CFG0["outlier_scale"], outlier_seed=OUTLIER_SEED)
    cs = np.zeros((B, 3, SHAPE.conv_ch), np.int8)
    ss = np.zeros((B, SHAPE.nheads, SHAPE.headdim, SHAPE.d_state), np.int32)
    ref = O.mixer_prefill(ol, x, conv_state=cs, ssm_state=ss)
    csd, ssd = dl.new_states(B)
    xd = dev(x)
    parts = [dl.prefill(xd[:, :17].contiguous(), conv_state=csd, ssm_state=ssd),
             dl.prefill(xd[:, 17:35].contiguous(), conv_state=csd, ssm_state=ssd)]
    for t in range(35, T):
        parts.append(dl.decode(xd[:, t].contiguous(), csd, ssd)[:, None])
    got = torch.cat(parts, 1).cpu().numpy()
    env.sync_status()
    assert np.array_equal(got, ref)
    assert np.array_equal(csd.cpu().numpy(), cs) and np.array_equal(ssd.cpu().numpy(), ss)


def test_stack_layers_match_oracle_stack(env):
    """Three 130M stack layers (pre-norm + residual), B=1, T=512, each side
    calibrated and run on its own: the oracle stack's exponent tables and
    every layer's output equal the GPU stack's."""
    from quantized_state_space_mamba2_b200.model import DeviceStack
    P = [S.layer_params(SHAPE, 100 + l) for l in range(3)]
    xcal = S.calibration_batch(SHAPE.d_model, 32, 8, 50.0, OUTLIER_SEED, n_seqs=2)
    x = S.activations(1, 512, SHAPE.d_model, seed=3, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=OUTLIER_SEED)
    ols, c = [], xcal
    for l in range(3):
        ol = O.prepare_layer(P[l], SHAPE, prenorm=True)
        c = O.calibrate_layer(ol, c, residual=True)
        ols.append(ol)
    st = DeviceStack(P, SHAPE)
    st.calibrate(dev(xcal))
    r, ref = dev(x), x
    for l, (dl, ol) in enumerate(zip(st.layers, ols)):
        compare_exponents(dl.exponents(), ol)
        ref = O.mixer_prefill(ol, ref, residual=True)
        dl.prefill(r, residual=True, out=r)
        env.sync_status()
        assert np.array_equal(r.cpu().numpy(), ref), f"layer {l}"
