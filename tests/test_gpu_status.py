"""The device error word.  A NaN or an Inf reaching an int8 activation
quantiser is reported by fm_sync_status as FM_ERR_NONFINITE; a bounded
pipeline wait that gives up is reported as FM_ERR_TIMEOUT.  The word is
cleared by that read, and the next call on clean data is exact again.  No
GPU fault is involved: a NaN in an input tensor is ordinary data, and the
timeouts come from producers that issue nothing (fm_set_fault_injection), so
the waits run out on a barrier nothing completes."""
import numpy as np
import pytest

import oracle as O
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


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
def test_nonfinite_input_is_reported_then_cleared(L, bad):
    M, K = 6, 768
    x = S.normal((M, K), 1.0, seed=91)
    xb = x.copy()
    xb[2, 300] = bad
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    L.sync_status()                                   # start from a clear word
    L.hadamard_quant(torch.from_numpy(xb).cuda(), K, None, 1, L.FM_DYNAMIC, None, q, sx)
    with pytest.raises(L.FmError) as e:
        L.sync_status()
    assert e.value.status == 5                        # FM_ERR_NONFINITE
    L.sync_status()                                   # the read cleared it
    # clean data afterwards: exact against the oracle, no error
    L.hadamard_quant(torch.from_numpy(x).cuda(), K, None, 1, L.FM_DYNAMIC, None, q, sx)
    L.sync_status()
    qr, sr = O.hadamard_quant(x)
    assert np.array_equal(q.cpu().numpy(), qr) and np.array_equal(sx.cpu().numpy(), sr)


def _layer_pair(seed=1400):
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    s = S.MAMBA2_130M
    P = S.layer_params(s, seed)
    xcal = S.calibration_batch(s.d_model, 64, 8, 50.0, 4242, n_seqs=2)
    ol = O.prepare_layer(P, s)
    O.calibrate_layer(ol, xcal)
    dl = DeviceLayer(P, s)
    dl.calibrate(torch.from_numpy(xcal).cuda())
    return s, ol, dl


@pytest.mark.parametrize("stall", ["gemm", "scan"])
def test_wait_timeout_is_reported_and_the_next_call_is_exact(L, stall):
    """A producer that issues nothing (the GEMMs' loads, or the scan's chunk
    copies) leaves its consumers waiting on a barrier nothing completes: with
    a 20 ms limit they give up, the call ends (every kernel frees its TMEM and
    has nothing in flight), and fm_sync_status reports FM_ERR_TIMEOUT.  The
    next call, at the normal limit, equals the oracle bit for bit.  800
    tokens put the in_proj on the persistent GEMM and out_proj on the
    small-grid one."""
    s, ol, dl = _layer_pair()
    x = S.activations(1, 800, s.d_model, seed=92, n_outliers=8, outlier_scale=50.0,
                      outlier_seed=4242)
    xd = torch.from_numpy(x).cuda()
    L.sync_status()
    mask = L.STALL_GEMM if stall == "gemm" else L.STALL_SCAN
    L.set_fault_injection(mask, 20_000_000)
    try:
        dl.prefill(xd)
        torch.cuda.synchronize()
    finally:
        L.set_fault_injection(0, 0)
    with pytest.raises(L.FmError) as e:
        L.sync_status()
    assert e.value.status == 6                        # FM_ERR_TIMEOUT
    out = dl.prefill(xd)
    L.sync_status()
    assert np.array_equal(out.cpu().numpy(), O.mixer_prefill(ol, x))


def test_fault_injection_arguments(L):
    with pytest.raises(L.FmError) as e:
        L.set_fault_injection(4, 0)
    assert e.value.status == 1
    with pytest.raises(L.FmError):
        L.set_fault_injection(0, 10_000_000_000)      # above the 4 s default
    L.set_fault_injection(0, 0)
