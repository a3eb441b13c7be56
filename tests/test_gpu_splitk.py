"""Split-K of the small-grid GEMM (fm_w8a8_gemm_ws, fm_in_proj_ws and the
layer entry points), switched on for this module (fm_set_gemm_splitk; off by
default): the K slices add exact int32 partial sums, so the results are bit
for bit those of the unsplit kernel and of the oracle, at the decode shapes
(M = 64 at 2.7B) and the 130M out_proj (M = 2048, N = 768).
"""
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
    lib.set_gemm_splitk(True)
    yield lib
    lib.set_gemm_splitk(False)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


@pytest.mark.parametrize("M,N,K", [(64, 10576, 2560), (64, 2560, 5120), (2048, 768, 1536),
                                   (3, 10576, 2560), (130, 768, 1536)])
def test_split_gemm_bit_exact(L, M, N, K):
    nb = L.gemm_workspace_bytes(M, N, K)
    assert nb > 0, "the shape is meant to split"
    A = S.uniform_ints((M, K), -127, 127, seed=M + K, dtype=np.int8)
    W = S.uniform_ints((N, K), -127, 127, seed=N + K, dtype=np.int8)
    sx = np.abs(S.normal(M, 0.01, seed=1)) + 1e-3
    sw = np.abs(S.normal(N, 0.001, seed=2)) + 1e-4
    res = S.normal((M, N), 1.0, seed=3)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    ref = (A.astype(np.float64) @ W.astype(np.float64).T).astype(np.int64)   # exact (< 2^53)
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Y, None, acc, ws=ws)
    assert np.array_equal(host(acc), ref)
    assert np.array_equal(host(Y), O.dequant(ref.astype(np.int32), sx, sw))
    # residual aliasing the output (a stack layer's out_proj)
    Yr = dev(res)
    L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Yr, Yr, None, ws=ws)
    assert np.array_equal(host(Yr), O.dequant(ref.astype(np.int32), sx, sw, residual=res))
    # the unsplit kernel gives the same bits
    Y2 = torch.empty_like(Y)
    L.w8a8_gemm(dev(A), dev(sx), dev(W), dev(sw), Y2)
    assert torch.equal(Y, Y2)
    L.sync_status()


def test_split_in_proj_decode_2p7b(L):
    s, M = S.MAMBA2_2P7B, 64
    nb = L.gemm_workspace_bytes(M, s.n_in, s.d_model)
    assert nb > 0
    A = S.uniform_ints((M, s.d_model), -127, 127, seed=31, dtype=np.int8)
    W = S.uniform_ints((s.n_in, s.d_model), -127, 127, seed=32, dtype=np.int8)
    sx = np.abs(S.normal(M, 0.01, seed=33)) + 1e-3
    sw = np.abs(S.normal(s.n_in, 3e-3, seed=34)) + 1e-4
    e_u = S.uniform_ints(s.conv_ch, -6, -2, seed=35)
    exps = np.zeros(L.exp_table_layout(s).size, np.int32)
    exps[:s.conv_ch] = e_u
    z = torch.empty((M, s.d_inner), dtype=torch.float32, device="cuda")
    xbc = torch.empty((M, s.conv_ch), dtype=torch.int8, device="cuda")
    dt = torch.empty((M, s.nheads), dtype=torch.float32, device="cuda")
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    L.in_proj(dev(A), dev(sx), dev(W), dev(sw), s, dev(exps), z, xbc, dt, ws=ws)
    acc = (A.astype(np.float64) @ W.astype(np.float64).T).astype(np.int32)
    zr, xr, dr = O.in_proj_epilogue(acc, sx, sw, s.d_inner, s.conv_ch, s.nheads, e_u)
    assert np.array_equal(host(z), zr)
    assert np.array_equal(host(xbc), xr)
    assert np.array_equal(host(dt), dr)


def test_split_workspace_validation(L):
    A = torch.zeros((64, 2560), dtype=torch.int8, device="cuda")
    W = torch.zeros((10576, 2560), dtype=torch.int8, device="cuda")
    sx = torch.ones(64, device="cuda")
    sw = torch.ones(10576, device="cuda")
    Y = torch.empty((64, 10576), device="cuda")
    with pytest.raises(RuntimeError):
        L.w8a8_gemm(A, sx, W, sw, Y, ws=torch.empty(16, dtype=torch.uint8, device="cuda"))
    # a problem that would not split needs no workspace
    assert L.gemm_workspace_bytes(8192, 10576, 2560) == 0
