"""Parity at the full workload sizes, in the launch configurations the
benchmark times: the 2.7B-shaped stack prefill over 2 x 4096 tokens and the
2.7B-shaped decode step of 64 sequences.

Against the oracle, on the outputs it computes in seconds:
  * causal prefixes -- a token's output depends on earlier tokens only, so
    the first tokens of the full-size GPU prefill equal the oracle's prefill
    of just those tokens (layers 1 and 2 of the stack);
  * the whole 64-sequence decode batch, after a short prefill.
Against itself, properties that hold at any size: a full-size prefill split
into two prefills, or into a prefill and a decode step, gives the same bits
(outputs and carried states).

Both sides calibrate on the same small seeded set (the benchmark's 16 x 512
calibration would take the oracle minutes per layer)."""
import numpy as np
import pytest

import oracle as O
from quantized_state_space_mamba2_b200 import synth as S

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SHAPE = S.MAMBA2_2P7B
W3 = S.WORKLOADS["stack2p7b_64l_b2_t4096"]
W4 = S.WORKLOADS["decode2p7b_64l_b64"]
OUTLIER_SEED = 4242  # the benchmark's outlier channels


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


def _acts(B, T, seed, w):
    return S.activations(B, T, SHAPE.d_model, seed=seed, n_outliers=w["n_outliers"],
                         outlier_scale=w["outlier_scale"], outlier_seed=OUTLIER_SEED)


def _oracle_stack(P, xcal):
    ols, c = [], xcal
    for p in P:
        ol = O.prepare_layer(p, SHAPE, prenorm=True)
        c = O.calibrate_layer(ol, c, residual=True)
        ols.append(ol)
    return ols


def _check_exponents(dl, ol):
    g = dl.exponents()
    for k in ("e_u", "e_x", "e_h", "e_y"):
        assert np.array_equal(g[k], getattr(ol, k)), k
    assert (g["e_B"], g["e_C"], g["e_g"]) == (ol.e_B, ol.e_C, ol.e_g)
    assert np.array_equal(g["conv_bq"], ol.conv_bq)


@pytest.fixture(scope="module")
def stack2(env):
    """Layers 1 and 2 of the 2.7B stack (the benchmark's weight seeds), both
    sides calibrated on 2 seeded sequences of 48 tokens."""
    from quantized_state_space_mamba2_b200.model import DeviceStack
    P = [S.layer_params(SHAPE, 1000 + l) for l in range(2)]
    xcal = S.calibration_batch(SHAPE.d_model, 48, W3["n_outliers"], W3["outlier_scale"],
                               OUTLIER_SEED, n_seqs=2)
    st = DeviceStack(P, SHAPE)
    st.calibrate(dev(xcal))
    return P, st, _oracle_stack(P, xcal)


def test_stack2p7b_prefix_matches_oracle(env, stack2):
    P, st, ols = stack2
    B, T, Tp = W3["batch"], W3["seqlen"], 40
    x = _acts(B, T, 1, W3)
    r = dev(x)
    ws = st.layers[0].workspace(B, T)
    ref = np.ascontiguousarray(x[:, :Tp])
    for l, (dl, ol) in enumerate(zip(st.layers, ols)):
        _check_exponents(dl, ol)
        dl.prefill(r, residual=True, out=r, ws=ws)
        env.sync_status()
        ref = O.mixer_prefill(ol, ref, residual=True)
        assert np.array_equal(r[:, :Tp].cpu().numpy(), ref), f"layer {l + 1}"


def test_stack2p7b_split_prefill_is_identical(env, stack2):
    """Full size, GPU only: 4096 tokens at once == 2048 + 2047 tokens with
    carried conv / SSM state + one decode step, both layers."""
    _, st, _ = stack2
    B, T = W3["batch"], W3["seqlen"]
    x = dev(_acts(B, T, 1, W3))
    full = x.clone()
    states_full = [L.new_states(B) for L in st.layers]
    st.prefill_(full, states=states_full)
    a = x[:, :2048].contiguous()
    b = x[:, 2048:T - 1].contiguous()
    c = x[:, T - 1].contiguous()
    states = [L.new_states(B) for L in st.layers]
    st.prefill_(a, states=states)
    st.prefill_(b, states=states)
    for (cs, ss), L in zip(states, st.layers):
        L.decode(c, cs, ss, residual=True, out=c)
    env.sync_status()
    got = torch.cat([a, b, c[:, None]], 1)
    assert torch.equal(got, full)
    for (c1, s1), (c2, s2) in zip(states, states_full):
        assert torch.equal(c1, c2) and torch.equal(s1, s2)


def test_decode2p7b_b64_matches_oracle(env, stack2):
    """The decode workload's batch of 64 sequences through layers 1 and 2:
    a 4-token prefill builds the states, then one decode step; outputs and
    both states bit for bit."""
    P, st, ols = stack2
    B, Pn = W4["batch"], 4
    pre, xt = _acts(B, Pn, 77, W4), _acts(B, 1, 5, W4)
    g_states = [L.new_states(B) for L in st.layers]
    r = dev(pre)
    st.prefill_(r, states=g_states)
    xd = dev(xt[:, 0])
    outs = []
    for (cs, ss), L in zip(g_states, st.layers):
        L.decode(xd, cs, ss, residual=True, out=xd)
        outs.append(xd.cpu().numpy())
    env.sync_status()
    ref = xt
    for l, ol in enumerate(ols):
        cs = np.zeros((B, 3, SHAPE.conv_ch), np.int8)
        ss = np.zeros((B, SHAPE.nheads, SHAPE.headdim, SHAPE.d_state), np.int32)
        # the oracle runs the prefill and the step as one sequence per layer;
        # layer l's input is layer l-1's output over all Pn + 1 tokens
        seq = ref if l > 0 else np.concatenate([pre, xt], 1)
        out = O.mixer_prefill(ol, seq, residual=True, conv_state=cs, ssm_state=ss)
        assert np.array_equal(outs[l], out[:, -1]), f"layer {l + 1}"
        assert np.array_equal(g_states[l][0].cpu().numpy(), cs)
        assert np.array_equal(g_states[l][1].cpu().numpy(), ss)
        ref = out


def test_decode2p7b_b64_continues_512_token_prefill(env, stack2):
    """The decode workload's shape, GPU only: 64 sequences prefilled over 512
    tokens then one decode step == a 513-token prefill (last token's output,
    both states), both layers."""
    _, st, _ = stack2
    B, Pn = W4["batch"], W4["prefill_len"]
    x = dev(_acts(B, Pn + 1, 77, W4))
    full = x.clone()
    s_full = [L.new_states(B) for L in st.layers]
    st.prefill_(full, states=s_full)
    a = x[:, :Pn].contiguous()
    c = x[:, Pn].contiguous()
    s = [L.new_states(B) for L in st.layers]
    st.prefill_(a, states=s)
    for (cs, ss), L in zip(s, st.layers):
        L.decode(c, cs, ss, residual=True, out=c)
    env.sync_status()
    assert torch.equal(c, full[:, Pn])
    for (c1, s1), (c2, s2) in zip(s, s_full):
        assert torch.equal(c1, c2) and torch.equal(s1, s2)
