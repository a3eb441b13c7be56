"""The comparison arms of the rotated linears on the GPU: plain W8A8 and
SmoothQuant (the paper's reference [7]) run through the library's unchanged
kernels, against the oracle bit for bit.

The pages rank the Hadamard-rotated linears above plain W8A8 and above
SmoothQuant (pith.science review of FastMamba, "If this is right" and the
forward implications).  SmoothQuant divides each input channel of a linear
by s_j and multiplies the weight's column j by s_j; in a Mamba2 block both
linears follow an RMSNorm with a per-channel weight, so 1/s folds into that
weight (oracle.baselines.smooth_params) and the GPU runs the rotate = 0 path
on the folded weights.  Each arm's GPU calibration and prefill must equal the
oracle's exactly; the arms must then rank as the pages report against the
unquantised fp64 mixer."""
import numpy as np
import pytest

import oracle as O
from oracle import baselines
from quantized_state_space_mamba2_b200 import synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("mode", [O.DYNAMIC, O.STATIC])
def test_smoothquant_and_plain_arms_bit_exact_and_ranked(L, mode):
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    s = S.MAMBA2_130M
    P = S.layer_params(s, 1300)
    xcal = S.calibration_batch(s.d_model, 64, 8, 50.0, 4242, n_seqs=3)
    x = S.activations(1, 192, s.d_model, seed=31, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=4242)
    Q = baselines.smooth_params(P, s, xcal, alpha=0.5)
    f64 = O.ref_mixer_f64(P, s, x, prenorm=True, residual=True) - x
    sq = {}
    for arm, params, rot in (("plain", P, 0), ("smooth", Q, 0), ("rotated", P, 1)):
        ol = O.prepare_layer(params, s, rotate=rot, mode=mode, prenorm=True)
        O.calibrate_layer(ol, xcal, residual=True)
        dl = DeviceLayer(params, s, rotate=rot, mode=mode, prenorm=True)
        dl.calibrate(dev(xcal), residual=True)
        got = dl.prefill(dev(x), residual=True)
        torch.cuda.synchronize()
        L.sync_status()
        got = got.cpu().numpy()
        ref = O.mixer_prefill(ol, x, residual=True)
        ex = dl.exponents()
        assert np.array_equal(ex["e_h"], ol.e_h) and np.array_equal(ex["e_y"], ol.e_y), arm
        assert np.array_equal(got, ref), arm
        sq[arm] = O.sqnr_db(f64, got - x)
    assert sq["rotated"] > sq["smooth"] > sq["plain"], sq
