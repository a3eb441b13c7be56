"""The allocation-free decode step (fm_decode_step_noalloc) against fm_decode_step.

fm_decode_step_noalloc serves callers that cannot allocate device memory
(a plugin inside a host framework that owns all device memory, a serving
loop whose memory budget is fixed at start-up): its scratch is a fixed
device array inside the library instead of a caller workspace.  It must give
exactly what fm_decode_step gives (the tests' bar is bit-exact), on two calls
in a row, since every call reuses the same array.  This file is collected
last so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest

from quantized_state_space_mamba2_b200 import synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_state_space_mamba2_b200 import build, lib
    build.build()
    lib.load()
    return lib


def test_decode_noalloc_matches_decode_step(env):
    lib = env
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    shape = S.MAMBA2_130M
    B = 8
    dl = DeviceLayer(S.layer_params(shape, 5), shape)
    xcal = S.calibration_batch(shape.d_model, 64, 8, 50.0, outlier_seed=55, n_seqs=2)
    dl.calibrate(torch.from_numpy(xcal).cuda())
    # states from a short prefill, then two decode tokens per path
    x = torch.from_numpy(S.activations(B, 20, shape.d_model, seed=9, n_outliers=8,
                                       outlier_scale=50.0, outlier_seed=55)).cuda()
    cs0, ss0 = dl.new_states(B)
    dl.prefill(x[:, :18].contiguous(), conv_state=cs0, ssm_state=ss0)
    cs_ref, ss_ref = cs0.clone(), ss0.clone()
    cs_new, ss_new = cs0.clone(), ss0.clone()
    ws = dl.workspace(B, 1)
    for t in (18, 19):
        xt = x[:, t].contiguous()
        ref = torch.empty_like(xt)
        lib.decode_step(dl.struct, xt, B, 0, cs_ref, ss_ref, ref, ws)
        got = torch.full_like(xt, float("nan"))
        lib.decode_step_noalloc(dl.struct, xt, B, 0, cs_new, ss_new, got)
        torch.cuda.synchronize()
        lib.sync_status()
        assert torch.equal(got, ref), f"token {t}"
        assert torch.equal(cs_new, cs_ref) and torch.equal(ss_new, ss_ref), f"token {t}"
        assert np.isfinite(got.cpu().numpy()).all()


def test_decode_noalloc_rejects_oversized_batch(env):
    lib = env
    from quantized_state_space_mamba2_b200.model import DeviceLayer
    shape = S.MAMBA2_130M
    dl = DeviceLayer(S.layer_params(shape, 6), shape)
    B = lib.NOALLOC_SCRATCH_BYTES // 1000   # far beyond what the fixed array holds
    assert lib.workspace_bytes(shape, B, 1) > lib.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((1, shape.d_model), device="cuda")
    cs, ss = dl.new_states(1)
    with pytest.raises(lib.FmError) as e:
        lib.decode_step_noalloc(dl.struct, x, B, 0, cs, ss, x)
    assert e.value.status == 4 and "FM_NOALLOC_SCRATCH_BYTES" in str(e.value)
