"""GPU: the pipelined stack prefill (fm_stack_prefill) against the CPU oracle's
stack and against the layer loop of fm_mixer_prefill, bit for bit: several
chunk counts, ragged runs, more than one sequence, states in and out, the
chunked scan mode, a CUDA-graph capture of the call, and the host-buffer
variant (fm_stack_prefill_host)."""
import numpy as np
import pytest

import oracle as O
from quantized_state_space_mamba2_b200 import synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPE = S.MAMBA2_130M
OUTLIER_SEED = 101
NL = 3


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


def acts(B, T, seed):
    return S.activations(B, T, SHAPE.d_model, seed=seed, n_outliers=8, outlier_scale=50.0,
                         outlier_seed=OUTLIER_SEED)


@pytest.fixture(scope="module")
def stack3(env):
    """Three 130M stack layers, calibrated on the GPU and, the same way, in the
    oracle (2 seeded sequences of 32 tokens)."""
    from quantized_state_space_mamba2_b200.model import DeviceStack
    P = [S.layer_params(SHAPE, 200 + l) for l in range(NL)]
    xcal = S.calibration_batch(SHAPE.d_model, 32, 8, 50.0, OUTLIER_SEED, n_seqs=2)
    st = DeviceStack(P, SHAPE)
    st.calibrate(dev(xcal))
    ols, c = [], xcal
    for l in range(NL):
        ol = O.prepare_layer(P[l], SHAPE, prenorm=True)
        c = O.calibrate_layer(ol, c, residual=True)
        ols.append(ol)
    return st, ols


def clone_states(states):
    return [(c.clone(), s.clone()) for c, s in states]


def warm_states(st, B, seed):
    """Non-zero conv / SSM states: a 16-token prefill through the layer loop."""
    states = [L.new_states(B) for L in st.layers]
    st.prefill_(dev(acts(B, 16, seed)), states=states)
    return states


def test_pipelined_stack_matches_oracle(env, stack3):
    """B = 2, T = 200 in runs of 96, 96, 8 tokens per sequence, against the
    oracle's three layers applied in turn."""
    st, ols = stack3
    x = acts(2, 200, 7)
    ref = x
    for ol in ols:
        ref = O.mixer_prefill(ol, ref, residual=True)
    r = dev(x)
    st.prefill_pipelined_(r, n_chunks=3)
    env.sync_status()
    assert np.array_equal(r.cpu().numpy(), ref)


@pytest.mark.parametrize("B,T,n", [(1, 512, 2), (1, 300, 3), (2, 256, 4), (3, 97, 2),
                                   (1, 64, 8), (2, 1, 2), (1, 40, 64), (2, 129, 1),
                                   (3, 256, 4)])  # 12 runs share the 8 streams
@pytest.mark.parametrize("with_states", [False, True], ids=["zero", "carried"])
def test_pipelined_stack_equals_layer_loop(env, stack3, B, T, n, with_states):
    """Outputs and (when given) the final conv / SSM states of every layer
    equal those of fm_mixer_prefill applied layer by layer."""
    st, _ = stack3
    x = dev(acts(B, T, 11 + T))
    s0 = warm_states(st, B, 5) if with_states else None
    ref = x.clone()
    s_ref = clone_states(s0) if with_states else None
    st.prefill_(ref, states=s_ref)
    got = x.clone()
    s_got = clone_states(s0) if with_states else None
    st.prefill_pipelined_(got, n_chunks=n, states=s_got)
    env.sync_status()
    assert torch.equal(got, ref)
    if with_states:
        for (c1, h1), (c2, h2) in zip(s_got, s_ref):
            assert torch.equal(c1, c2) and torch.equal(h1, h2)


def test_pipelined_stack_chunked_scan_mode(env, stack3):
    """In the chunked (SSD) scan mode the state crosses each run boundary as
    int32, so the pipelined result is the layer loop applied run after run
    with carried states (T = 384 in runs of 128), bit for bit."""
    st, _ = stack3
    env.set_scan_mode("ssd")
    try:
        x = dev(acts(1, 384, 23))
        ref = x.clone()
        states = [L.new_states(1) for L in st.layers]
        for k in range(3):
            run = ref[:, 128 * k:128 * (k + 1)].contiguous()
            st.prefill_(run, states=states)
            ref[:, 128 * k:128 * (k + 1)] = run
        got = x.clone()
        st.prefill_pipelined_(got, n_chunks=3)
        env.sync_status()
        assert torch.equal(got, ref)
    finally:
        env.set_scan_mode("seq")


def test_pipelined_stack_in_a_cuda_graph(env, stack3):
    """Captured (the first call, outside the capture, creates the streams):
    the replay gives the layer loop's bits."""
    st, _ = stack3
    B, T, n = 1, 256, 2
    x = dev(acts(B, T, 31))
    ref = x.clone()
    st.prefill_(ref)
    buf = x.clone()
    ws = st.stack_workspace(B, T, n)
    st.prefill_pipelined_(buf, n_chunks=n, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            buf.copy_(x)
            st.prefill_pipelined_(buf, n_chunks=n, ws=ws)
    buf.zero_()
    g.replay()
    torch.cuda.synchronize()
    env.sync_status()
    assert torch.equal(buf, ref)
    del g


@pytest.mark.parametrize("B,T,n,pinned,alias", [(1, 512, 4, True, False), (2, 200, 3, True, True),
                                                (1, 300, 1, False, False), (3, 64, 2, False, True)])
def test_stack_prefill_host(env, stack3, B, T, n, pinned, alias):
    """Host input and output through fm_stack_prefill_host (copies per run on
    the runs' streams) equal the device-resident layer loop, states included."""
    st, _ = stack3
    x = acts(B, T, 41 + T)
    ref = dev(x)
    s0 = warm_states(st, B, 9)
    s_ref = clone_states(s0)
    st.prefill_(ref, states=s_ref)
    xh = torch.from_numpy(x.copy())
    if pinned:
        xh = xh.pin_memory()
    oh = xh if alias else (torch.empty_like(xh).pin_memory() if pinned else torch.empty_like(xh))
    xd = torch.empty(ref.shape, dtype=torch.float32, device="cuda")
    s_got = clone_states(s0)
    st.prefill_host(xh, oh, xd, n_chunks=n, states=s_got)
    torch.cuda.synchronize()
    env.sync_status()
    assert torch.equal(oh, ref.cpu())
    for (c1, h1), (c2, h2) in zip(s_got, s_ref):
        assert torch.equal(c1, c2) and torch.equal(h1, h2)
