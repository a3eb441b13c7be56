"""Programmatic dependent launch (fm_set_pdl(1), the default): the hot kernels
may be scheduled while their predecessor drains and wait for it before they
read its outputs.  The results must be the same bits as plain launches: a
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
    L.set_pdl(False)
    try:
        ref = _run(L, stack, x, 137)
    finally:
        L.set_pdl(L.PDL_DEFAULT)
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
        L.set_pdl(L.PDL_DEFAULT)
    L.set_pdl(False)
    try:
        plain = x.clone()
        stack.prefill_(plain, ws=ws)
        torch.cuda.synchronize()
    finally:
        L.set_pdl(L.PDL_DEFAULT)
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
    assert torch.equal(out, plain)


def test_pdl_back_to_back_state_writers(L):
    """Scan calls that hand a state straight to the next one (a prefill scan,
    then two single steps, no other kernel between): under programmatic
    dependent launch the single-step kernel loads its state before its
    dependency wait, which is sound only because the kernels that write a
    state issue no early trigger.  Same bits as plain launches and the oracle."""
    import oracle as O
    s = S.MAMBA2_130M
    B, T = 2, 40
    cc, nh = s.conv_ch, s.nheads
    xbc = S.uniform_ints((B, T + 2, cc), -127, 127, seed=501, dtype=np.int8)
    dt_raw = S.normal((B, T + 2, nh), 2.0, seed=502)
    P = S.layer_params(s, 503)
    A_q, D_q, e_D = O.prepare_ssm(P["a_log"], P["D"])
    e_x = S.uniform_ints(nh, -5, -3, seed=504)
    e_B, e_C = -4, -3
    e_h = (e_x + e_B - 15 + S.uniform_ints(nh, 2, 8, seed=505)).astype(np.int32)
    e_y = (np.maximum(e_C + e_h, e_D + e_x) - 2).astype(np.int32)
    X = L.exp_table_layout(s)
    exps = np.zeros(X.size, np.int32)
    exps[X.e_x:X.e_x + nh], exps[X.e_B], exps[X.e_C] = e_x, e_B, e_C
    exps[X.e_h:X.e_h + nh], exps[X.e_y:X.e_y + nh], exps[X.e_D:X.e_D + nh] = e_h, e_y, e_D
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    args = (dv(P["dt_bias"]), dv(A_q), dv(D_q), dv(exps))

    def run():
        st = torch.zeros((B, nh, s.headdim, s.d_state), dtype=torch.int32, device="cuda")
        ys = []
        for t0, t1 in ((0, T), (T, T + 1), (T + 1, T + 2)):
            n = t1 - t0
            y = torch.empty((B, n, s.d_inner), dtype=torch.int32, device="cuda")
            ws = torch.empty(max(L.scan_workspace_bytes(s, B, n), 16), dtype=torch.uint8,
                             device="cuda")
            L.ssm_scan_pot(dv(xbc[:, t0:t1]), dv(dt_raw[:, t0:t1]), B, n, s, *args, st, y, ws)
            ys.append(y)
        torch.cuda.synchronize()
        L.sync_status()
        return [y.cpu().numpy() for y in ys], st.cpu().numpy()

    L.set_pdl(False)
    try:
        ref_y, ref_st = run()
    finally:
        L.set_pdl(L.PDL_DEFAULT)
    L.set_pdl(True)
    try:
        got_y, got_st = run()
    finally:
        L.set_pdl(L.PDL_DEFAULT)
    for a, b in zip(ref_y, got_y):
        assert np.array_equal(a, b)
    assert np.array_equal(ref_st, got_st)
    st_o = np.zeros((B, nh, s.headdim, s.d_state), np.int32)
    yo = O.ssm_scan_pot(xbc, dt_raw, P["dt_bias"], A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D,
                        s.headdim, s.d_state, state=st_o)
    assert np.array_equal(np.concatenate(got_y, 1), yo)
    assert np.array_equal(got_st, st_o)
