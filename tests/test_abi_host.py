"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/fastmamba.h declares, and rejects bad arguments
before any launch."""
import ctypes as C
import os
import re

import pytest

from quantized_state_space_mamba2_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fastmamba.h")


@pytest.fixture(scope="module")
def so():
    B.build()
    from quantized_state_space_mamba2_b200 import lib
    return lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fm_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(so):
    names = declared_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(so, n), n
    from quantized_state_space_mamba2_b200 import lib
    assert set(names) == set(lib.EXPORTS)


def test_status_strings_and_version(so):
    assert so.fm_status_string(0) == b"FM_OK"
    assert so.fm_status_string(6) == b"FM_ERR_TIMEOUT"
    assert so.fm_version() == 100


def test_exp_layout_and_workspace(so):
    from quantized_state_space_mamba2_b200 import lib, synth as S
    s = S.MAMBA2_130M
    L = lib.exp_table_layout(s)
    cc, nh = s.conv_ch, s.nheads
    assert (L.e_u, L.e_w, L.e_o, L.e_x) == (0, cc, 2 * cc, 3 * cc)
    assert L.e_g == 3 * cc + 4 * nh + 2 and L.size == 3 * cc + 4 * nh + 3
    ws = lib.workspace_bytes(s, 1, 2048)
    # mixer intermediates + the scan's per-token dt/dA, (u, D x) and widened B, C
    # and the per-16-step growth bounds (8 bytes per channel per 16 tokens)
    per_tok = (s.d_model + 9 * s.d_inner + 2 * cc + 4 * nh + 8 + (4 * nh + 8 * s.d_inner + 1024)
               + s.d_inner // 2)
    assert per_tok * 2048 <= ws <= per_tok * 2048 + 256 * 16
    assert lib.calib_workspace_bytes(s, 16, 512) > lib.workspace_bytes(s, 16, 512)
    # a single decode step stages nothing for the scan
    assert lib.scan_workspace_bytes(s, 64, 1) == 256
    bad = S.MixerShape(d_model=300, d_inner=512, headdim=64, d_state=128)
    assert lib.workspace_bytes(bad, 1, 1) == 0


def test_validation_rejects_before_launch(so):
    from quantized_state_space_mamba2_b200 import lib
    from quantized_state_space_mamba2_b200 import synth as S
    sh = lib.shape_struct(S.MAMBA2_130M)
    # null input pointer
    assert so.fm_hadamard_quant(None, 4, 768, None, 1, 0, None, None, None, None, None) == 1
    # K not a multiple of 256
    assert so.fm_hadamard_quant(None, 4, 700, None, 1, 0, None, None, None, None, None) == 2
    # misaligned pointer (never dereferenced)
    assert so.fm_w8a8_gemm(C.c_void_p(0x1001), C.c_void_p(0x2000), 4, C.c_void_p(0x3000),
                           C.c_void_p(0x4000), 8, 128, None, C.c_void_p(0x5000), None, None) == 3
    # K not a multiple of 128
    assert so.fm_w8a8_gemm(None, None, 4, None, None, 8, 100, None, None, None, None) == 2
    # unsupported head size
    bad = lib.fm_shape(768, 1536, 32, 128, 1, 4)
    assert so.fm_conv1d_pot(None, 1, 4, C.byref(bad), None, None, None, None, None, None) == 2
    # empty work is a no-op success
    assert so.fm_conv1d_pot(None, 0, 4, C.byref(sh), None, None, None, None, None, None) == 0
    assert b"shape" in so.fm_last_error() or so.fm_last_error() != b""
    # decode requires both states
    assert so.fm_decode_step(None, None, 1, 0, None, None, None, None, 0, None) == 1
