"""Programmatic dependent launch (fm_set_pdl(1)): the hot kernels may be
scheduled while their predecessor drains and wait for it before their first
global access.  The results must be the same bits as plain launches: a
3-layer 130M stack prefill with carried states and decode steps, the chunked
scan mode and the LQ layer, launched directly and inside a captured CUDA
graph.  The setting is process-wide, so the test restores it."""
import numpy as np
import pytest

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


def _run(L, stack, x, T0):
    """Prefill of T0 tokens with states, then decode steps for the rest;
    the chunked-scan prefill and the LQ prefill of the whole input."""
    B, T, _ = x.shape
    states = [Ly.new_states(B) for Ly in stack.layers]
    pre = x[:, :T0].contiguous()
    stack.prefill_(pre, states=states)
    steps = []
    for t in range(T0, T):
        xt = x[:, t].contiguous()
        for (cs, ss), Ly in zip(states, stack.layers):
            Ly.decode(xt, cs, ss, residual=True, out=xt)
        steps.append(xt)
    L.set_scan_mode("ssd")
    try:
        ssd = x.clone()
        stack.prefill_(ssd)
    finally:
        L.set_scan_mode("seq")
    lq = stack.layers[0].lq_prefill(x, residual=True)
    torch.cuda.synchronize()
    L.sync_status()
    return [pre, torch.stack(steps, 1), ssd, lq] + [t for st in states for t in st]


def test_pdl_gives_the_same_bits(L):
    from quantized_state_space_mamba2_b200.model import DeviceStack
    s = S.MAMBA2_130M
    stack = DeviceStack([S.layer_params(s, 1500 + l) for l in range(3)], s)
    xcal = torch.from_numpy(S.calibration_batch(s.d_model, 64, 8, 50.0, 4242, n_seqs=2)).cuda()
    stack.calibrate(xcal)
    x = torch.from_numpy(S.activations(2, 140, s.d_model, seed=8, n_outliers=8,
                                       outlier_scale=50.0, outlier_seed=4242)).cuda()
    ref = _run(L, stack, x, 137)
    L.set_pdl(True)
    try:
        got = _run(L, stack, x, 137)
        # the same launches captured in a CUDA graph and replayed
        out = x.clone()
        ws = stack.layers[0].workspace(2, 140)
        stack.prefill_(out, ws=ws)                      # warm (lazy set-up outside capture)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        out.copy_(x)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            stack.prefill_(out, ws=ws)
        out.copy_(x)
        g.replay()
        torch.cuda.synchronize()
        L.sync_status()
    finally:
        L.set_pdl(False)
    plain = x.clone()
    stack.prefill_(plain, ws=ws)
    torch.cuda.synchronize()
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
    assert torch.equal(out, plain)
