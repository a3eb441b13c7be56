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
    # mixer intermediates + the scan's per-token dt/dA, u (int32), the x codes
    # (int8) and widened B, C
    # and the per-16-step growth bounds (8 bytes per channel per 16 tokens)
    per_tok = (s.d_model + 9 * s.d_inner + 2 * cc + 4 * nh + 8 + (4 * nh + 5 * s.d_inner + 1024)
               + s.d_inner // 2)
    # split-K is off by default: no partial sums
    assert lib.gemm_workspace_bytes(2048, s.d_model, s.d_inner) == 0
    assert per_tok * 2048 <= ws <= per_tok * 2048 + 256 * 17
    # switched on, the layer holds the partial sums of a GEMM that splits
    # (out_proj at 2048 rows)
    lib.set_gemm_splitk(True)
    try:
        ws = lib.workspace_bytes(s, 1, 2048)
        split = max(lib.gemm_workspace_bytes(2048, s.n_in, s.d_model),
                    lib.gemm_workspace_bytes(2048, s.d_model, s.d_inner))
        assert split == 2048 * s.d_model * 4
        assert per_tok * 2048 + split <= ws <= per_tok * 2048 + split + 256 * 17
    finally:
        lib.set_gemm_splitk(False)
    assert so.fm_set_gemm_splitk(2) == 1
    assert so.fm_set_gemm_cluster(2) == 1 and so.fm_set_gemm_cluster(-1) == 1
    assert so.fm_set_gemm_cluster(0) == 0 and so.fm_set_gemm_cluster(1) == 0
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


def _fake_layer(lib, S, mode=0, static_amax=None):
    """A layer struct whose device pointers are distinct 16-byte-aligned
    addresses that validation never dereferences."""
    p = [C.c_void_p(0x100000 * (i + 1)) for i in range(12)]
    return lib.fm_layer(lib.shape_struct(S.MAMBA2_130M), 1, mode, p[0], p[1], p[2], p[3], None,
                        p[4], p[5], p[6], p[7], p[8], p[9], p[10], static_amax)


def test_layer_validation_before_launch(so):
    from quantized_state_space_mamba2_b200 import lib
    from quantized_state_space_mamba2_b200 import synth as S
    big = 1 << 40
    x, ws = C.c_void_p(0x7000000), C.c_void_p(0x9000000)
    L = _fake_layer(lib, S)
    # out overlapping x partially (a whole-tensor alias is allowed)
    assert so.fm_mixer_prefill(C.byref(L), x, 1, 4, 0, None, None, C.c_void_p(0x7000010), ws, big,
                               None) == 1
    assert b"overlap" in so.fm_last_error()
    # workspace too small
    assert so.fm_mixer_prefill(C.byref(L), x, 1, 4, 0, None, None, x, ws, 16, None) == 4
    # static mode without its scales
    Ls = _fake_layer(lib, S, mode=1)
    assert so.fm_mixer_prefill(C.byref(Ls), x, 1, 4, 0, None, None, x, ws, big, None) == 1
    # bad activation mode
    Lb = _fake_layer(lib, S, mode=7)
    assert so.fm_mixer_prefill(C.byref(Lb), x, 1, 4, 0, None, None, x, ws, big, None) == 1
    # a misaligned required layer pointer
    Lm = _fake_layer(lib, S)
    Lm.w_in_s = C.c_void_p(0x100004)
    assert so.fm_mixer_prefill(C.byref(Lm), x, 1, 4, 0, None, None, x, ws, big, None) == 3
    # misaligned optional state
    assert so.fm_mixer_prefill(C.byref(L), x, 1, 4, 0, C.c_void_p(0x3001), None, x, ws, big,
                               None) == 3
    # negative sizes
    assert so.fm_mixer_prefill(C.byref(L), x, -1, 4, 0, None, None, x, ws, big, None) == 2
    # launch limits, checked before the first kernel: B is a grid dimension
    # (<= 65535), B * T the GEMMs' rows (<= 65535 tiles of 128)
    assert so.fm_mixer_prefill(C.byref(L), x, 70000, 1, 0, None, None, x, ws, big, None) == 2
    assert b"65535" in so.fm_last_error()
    assert so.fm_mixer_prefill(C.byref(L), x, 1, 65535 * 128 + 1, 0, None, None, x, ws, big,
                               None) == 2
    assert so.fm_decode_step_noalloc(C.byref(L), x, 70000, 0, C.c_void_p(0x3000),
                                     C.c_void_p(0x5000), x, None) in (2, 4)


def test_stack_prefill_validation_and_workspace(so):
    from quantized_state_space_mamba2_b200 import lib
    from quantized_state_space_mamba2_b200 import synth as S
    d = S.MAMBA2_130M
    sh = lib.shape_struct(d)
    # one chunk: the layer workspace of the whole batch
    assert lib.stack_workspace_bytes(d, 24, 2, 512, 1) == lib.workspace_bytes(d, 2, 512)
    # pipelined: one run's workspace per internal stream (runs of ceil(T / n)
    # tokens rounded up to 32, at most 8 streams), then zero-started conv and
    # SSM states for every layer and sequence, each piece 256-byte aligned
    al = lambda n: (n + 255) // 256 * 256
    for (nl, B, T, n) in ((24, 1, 2048, 2), (3, 2, 1000, 3), (2, 5, 64, 4)):
        tc = min(T, ((T + n - 1) // n + 31) // 32 * 32)
        runs = (T + tc - 1) // tc
        streams = min(B * runs, 8)
        off = 0
        for _ in range(streams):
            off = al(off) + lib.workspace_bytes(d, 1, tc)
        off = al(off) + nl * B * 3 * d.conv_ch
        off = al(off) + nl * B * d.nheads * d.headdim * d.d_state * 4
        assert lib.stack_workspace_bytes(d, nl, B, T, n) == off + 256, (nl, B, T, n)
    for bad in ((24, 1, 64, 0), (24, 1, 64, 65), (-1, 1, 64, 2), (24, -1, 64, 2)):
        assert lib.stack_workspace_bytes(d, *bad) == 0, bad
    # the entry point rejects before any launch
    big = 1 << 40
    x, ws = C.c_void_p(0x7000000), C.c_void_p(0x9000000)
    L = _fake_layer(lib, S)
    arr = lambda *ls: C.cast((C.POINTER(lib.fm_layer) * len(ls))(*[C.pointer(l) for l in ls]),
                             C.c_void_p)
    two = arr(L, L)
    assert so.fm_stack_prefill(two, 2, x, 1, 64, None, None, 0, ws, big, None) == 1
    assert so.fm_stack_prefill(two, 2, x, 1, 64, None, None, 65, ws, big, None) == 1
    assert so.fm_stack_prefill(two, -1, x, 1, 64, None, None, 2, ws, big, None) == 1
    assert so.fm_stack_prefill(None, 2, x, 1, 64, None, None, 2, ws, big, None) == 1
    assert so.fm_stack_prefill(two, 2, x, -1, 64, None, None, 2, ws, big, None) == 2
    # nothing to do: no layers, or no tokens
    assert so.fm_stack_prefill(None, 0, x, 1, 64, None, None, 2, ws, big, None) == 0
    assert so.fm_stack_prefill(two, 2, x, 0, 64, None, None, 2, ws, big, None) == 0
    # workspace too small or misaligned
    assert so.fm_stack_prefill(two, 2, x, 1, 64, None, None, 2, ws, 16, None) == 4
    assert so.fm_stack_prefill(two, 2, x, 1, 64, None, None, 2, C.c_void_p(0x9000008), big,
                               None) == 3
    # layers of different widths
    L27 = _fake_layer(lib, S)
    L27.shape = lib.shape_struct(S.MAMBA2_2P7B)
    assert so.fm_stack_prefill(arr(L, L27), 2, x, 1, 64, None, None, 2, ws, big, None) == 2
    # a null entry in a state array
    states = (C.c_void_p * 2)(0x3000, None)
    assert so.fm_stack_prefill(two, 2, x, 1, 64, C.cast(states, C.c_void_p), None, 2, ws, big,
                               None) == 1
    assert b"conv_states[1]" in so.fm_last_error()
    # the host-buffer variant: both host buffers are required, the device rows aligned
    h = C.c_void_p(0x5000000)
    assert so.fm_stack_prefill_host(two, 2, None, h, x, 1, 64, None, None, 2, ws, big, None) == 1
    assert so.fm_stack_prefill_host(two, 2, h, None, x, 1, 64, None, None, 2, ws, big, None) == 1
    assert so.fm_stack_prefill_host(two, 2, h, h, C.c_void_p(0x7000004), 1, 64, None, None, 2, ws,
                                    big, None) == 3
    assert so.fm_stack_prefill_host(two, 2, None, None, x, 0, 64, None, None, 2, ws, big,
                                    None) == 0
    assert so.fm_stack_prefill_host(two, 2, h, h, x, 1, 64, None, None, 2, ws, 16, None) == 4


def test_scan_and_tuning_validation(so):
    from quantized_state_space_mamba2_b200 import lib
    from quantized_state_space_mamba2_b200 import synth as S
    sh = lib.shape_struct(S.MAMBA2_130M)
    f = [C.c_void_p(0x200000 * (i + 1)) for i in range(9)]
    # workspace below fm_scan_workspace_bytes
    need = so.fm_scan_workspace_bytes(C.byref(sh), 1, 64)
    assert need > 256
    assert so.fm_ssm_scan_pot(f[0], f[1], 1, 64, C.byref(sh), f[2], f[3], f[4], f[5], None, f[6],
                              f[7], need - 16, None) == 4
    # tile variants: compiled ones accepted, others rejected
    for t in lib.SCAN_TILES:
        assert so.fm_set_scan_tile(*t) == 0
    assert so.fm_set_scan_tile(4, 4, 16) == 0
    assert so.fm_set_scan_tile(4, 3, 16) == 1 and so.fm_set_scan_tile(16, 4, 16) == 1
    # the PWL evaluator: unknown kind, negative count
    assert so.fm_eval_pwl(9, f[0], 4, f[1], None) == 1
    assert so.fm_eval_pwl(0, f[0], -1, f[1], None) == 2
    # gate: bad mode
    assert so.fm_gate_norm_quant(f[0], f[1], 4, C.byref(sh), f[2], f[3], 1, 5, None, f[4], f[5],
                                 None, None) == 1


def test_chunked_scan_validation(so):
    """The chunked scan mode's entry points reject bad arguments before any
    launch; its workspace covers the chunk states (fp32 + bf16) and decays."""
    from quantized_state_space_mamba2_b200 import lib
    from quantized_state_space_mamba2_b200 import synth as S
    sh = lib.shape_struct(S.MAMBA2_130M)
    s = S.MAMBA2_130M
    nch = (300 + 127) // 128
    need = lib.ssd_workspace_bytes(s, 2, 300)
    units = 2 * s.nheads * nch
    assert need >= units * 64 * 128 * (4 + 2) + units * 4
    assert lib.ssd_workspace_bytes(s, 0, 0) <= 1024
    p = C.c_void_p(0x7000000)
    # empty problem: nothing to do
    assert so.fm_ssd_scan(None, None, 0, 7, C.byref(sh), None, None, None, None, None, None, None,
                          0, None) == 0
    # null / misaligned / workspace
    assert so.fm_ssd_scan(None, p, 1, 7, C.byref(sh), p, p, p, p, None, p, p, 1 << 40, None) == 1
    assert so.fm_ssd_scan(p, p, 1, 7, C.byref(sh), p, p, p, p, C.c_void_p(0x3001), p, p, 1 << 40,
                          None) == 3
    assert so.fm_ssd_scan(p, p, 1, 7, C.byref(sh), p, p, p, p, None, p, p, 16, None) == 4
    assert so.fm_ssd_scan(p, p, 70000, 7, C.byref(sh), p, p, p, p, None, p, p, 1 << 40, None) == 2
    # scan mode switch
    assert so.fm_set_scan_mode(2) == 1
    assert so.fm_set_scan_mode(0) == 0
def test_xbc_exponent_setting_validation(so):
    """The conv-output exponent granularity takes 0 (static) or 1 (per token)."""
    assert so.fm_set_xbc_exponents(2) == 1
    assert so.fm_set_xbc_exponents(-1) == 1
    assert so.fm_set_xbc_exponents(1) == 0
    assert so.fm_set_xbc_exponents(0) == 0


def test_state_spec_validation(so):
    """Only the two state specs with kernels behind them are accepted."""
    assert so.fm_set_state_spec(16, 0) == 1
    assert so.fm_set_state_spec(24, 7) == 1
    assert so.fm_set_state_spec(16, 7) == 0
    assert so.fm_set_state_spec(31, 0) == 0


def test_lq_entry_points_validate(so):
    """The FastMamba-LQ entry points reject bad arguments before any launch,
    and the layer workspace covers its fp32 intermediates."""
    from quantized_state_space_mamba2_b200 import lib
    from quantized_state_space_mamba2_b200 import synth as S
    s = S.MAMBA2_130M
    sh = lib.shape_struct(s)
    p = C.c_void_p(0x7000000)
    # empty problems: nothing to do
    assert so.fm_lq_conv1d(None, 0, 0, 5, C.byref(sh), None, None, None, None, None) == 0
    assert so.fm_lq_scan(None, None, 0, None, 0, 3, 0, C.byref(sh), None, None, None, None, None,
                         None) == 0
    # conv: a row stride below conv_ch, a null weight, a misaligned output
    assert so.fm_lq_conv1d(p, s.conv_ch - 1, 1, 5, C.byref(sh), p, p, None, p, None) == 2
    assert so.fm_lq_conv1d(p, s.conv_ch, 1, 5, C.byref(sh), None, p, None, p, None) == 1
    assert so.fm_lq_conv1d(p, s.conv_ch, 1, 5, C.byref(sh), p, p, None, C.c_void_p(0x7000004),
                           None) == 3
    # scan: dt stride below nheads, z stride below d_inner, a null dt_bias
    assert so.fm_lq_scan(p, p, s.nheads - 1, None, 0, 1, 5, C.byref(sh), p, p, p, None, p,
                         None) == 2
    assert so.fm_lq_scan(p, p, s.nheads, p, s.d_inner - 1, 1, 5, C.byref(sh), p, p, p, None, p,
                         None) == 2
    assert so.fm_lq_scan(p, p, s.nheads, None, 0, 1, 5, C.byref(sh), None, p, p, None, p,
                         None) == 1
    # the layer: workspace = int8 input + scale, fp32 in_proj output, conv
    # output, gated value, int8 out_proj input + scale (+ split-K sums)
    M = 300
    need = lib.lq_workspace_bytes(s, 1, M)
    base = M * (s.d_model + 4 + 4 * s.n_in + 4 * s.conv_ch + 4 * s.d_inner + s.d_inner + 4)
    split = max(lib.gemm_workspace_bytes(M, s.n_in, s.d_model),
                lib.gemm_workspace_bytes(M, s.d_model, s.d_inner))
    assert base + split <= need <= base + split + 256 * 10
    L = lib.fm_layer()
    P = lib.fm_lq_params()
    assert so.fm_lq_mixer_prefill(C.byref(L), C.byref(P), p, 1, 5, 0, None, None, p, p, 1 << 30,
                                  None) in (1, 2)


def test_plain_c_consumer(so, tmp_path):
    """The header compiles as C99 (-Wall -Wextra -pedantic -Werror) and a C
    program linked against libfastmamba.so runs its host-only checks."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "quantized_state_space_mamba2_b200")
    exe = str(tmp_path / "abi_consumer")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "abi_consumer.c"), "-L", pkg, "-lfastmamba",
                    f"-Wl,-rpath,{pkg}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "17 checks passed" in r.stdout
