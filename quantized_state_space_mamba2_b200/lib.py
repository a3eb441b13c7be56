"""ctypes binding of libfastmamba.so (include/fastmamba.h), same names.

Argument marshalling only: tensors are torch CUDA tensors (device memory
owned by the caller), streams are torch streams; every computation happens
in the library's kernels.  There is no CPU fallback: if the shared library
is missing or no CUDA device is present the calls raise.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(_HERE, "libfastmamba.so")

FM_DYNAMIC, FM_STATIC = 0, 1
STATUS = {0: "FM_OK", 1: "FM_ERR_INVALID_ARG", 2: "FM_ERR_SHAPE", 3: "FM_ERR_ALIGNMENT",
          4: "FM_ERR_WORKSPACE", 5: "FM_ERR_NONFINITE", 6: "FM_ERR_TIMEOUT", 7: "FM_ERR_CUDA",
          8: "FM_ERR_UNSUPPORTED"}

# every entry point the header declares
EXPORTS = (
    "fm_status_string", "fm_last_error", "fm_sync_status", "fm_version", "fm_exp_table_layout",
    "fm_hadamard_quant", "fm_prepare_linear", "fm_w8a8_gemm", "fm_in_proj", "fm_conv1d_pot",
    "fm_gemm_workspace_bytes", "fm_w8a8_gemm_ws", "fm_in_proj_ws",
    "fm_ssm_scan_pot", "fm_gate_norm_quant", "fm_eval_pwl", "fm_workspace_bytes",
    "fm_mixer_prefill", "fm_decode_step", "fm_prepare_mixer_params", "fm_calib_workspace_bytes",
    "fm_calibrate_layer", "fm_decode_step_noalloc", "fm_scan_workspace_bytes",
    "fm_set_scan_tile", "fm_ssd_workspace_bytes", "fm_ssd_scan", "fm_set_scan_mode",
    "fm_set_state_spec", "fm_lq_conv1d", "fm_lq_scan", "fm_lq_workspace_bytes",
    "fm_lq_mixer_prefill", "fm_set_fault_injection", "fm_set_gemm_splitk",
    "fm_set_gemm_tile", "fm_set_xbc_exponents", "fm_conv1d_pot_tok", "fm_ssm_scan_pot_tok",
    "fm_scan_workspace_bytes_tok", "fm_set_pdl", "fm_set_lq_scan_cpw", "fm_set_gemm_cluster",
    "fm_stack_prefill", "fm_stack_workspace_bytes", "fm_stack_prefill_host",
)
NOALLOC_SCRATCH_BYTES = 16 << 20  # FM_NOALLOC_SCRATCH_BYTES


class FmError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


class fm_shape(C.Structure):
    _fields_ = [("d_model", C.c_int), ("d_inner", C.c_int), ("headdim", C.c_int),
                ("d_state", C.c_int), ("ngroups", C.c_int), ("d_conv", C.c_int)]


class fm_exp_layout(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("e_u", "e_w", "e_o", "e_x", "e_B", "e_C", "e_h", "e_y",
                                       "e_D", "e_g", "size")]


_P = C.c_void_p


class fm_layer(C.Structure):
    _fields_ = [("shape", fm_shape), ("rotate", C.c_int), ("mode", C.c_int),
                ("w_in_q", _P), ("w_in_s", _P), ("w_out_q", _P), ("w_out_s", _P),
                ("prenorm_w", _P), ("conv_wq", _P), ("conv_bq", _P), ("dt_bias", _P),
                ("A_q", _P), ("D_q", _P), ("norm_w", _P), ("exps", _P), ("static_amax", _P)]


class fm_lq_params(C.Structure):
    _fields_ = [("conv_w", _P), ("conv_b", _P), ("a_log", _P), ("D", _P)]


_lib = None


def load():
    """Load the in-tree library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(SO_PATH):
        raise ImportError(f"{SO_PATH} is missing: build it with "
                          "`python -m quantized_state_space_mamba2_b200.build`")
    L = C.CDLL(SO_PATH)
    I, I64, SZ = C.c_int, C.c_int64, C.c_size_t
    sp = C.POINTER(fm_shape)
    lp = C.POINTER(fm_layer)
    sig = {
        "fm_status_string": (C.c_char_p, [I]),
        "fm_last_error": (C.c_char_p, []),
        "fm_sync_status": (I, [_P]),
        "fm_version": (I, []),
        "fm_exp_table_layout": (fm_exp_layout, [sp]),
        "fm_hadamard_quant": (I, [_P, I64, I64, _P, I, I, _P, _P, _P, _P, _P]),
        "fm_prepare_linear": (I, [_P, I64, I64, I, _P, _P, _P]),
        "fm_w8a8_gemm": (I, [_P, _P, I64, _P, _P, I64, I64, _P, _P, _P, _P]),
        "fm_in_proj": (I, [_P, _P, I64, _P, _P, sp, _P, _P, _P, _P, _P]),
        "fm_gemm_workspace_bytes": (SZ, [I64, I64, I64]),
        "fm_w8a8_gemm_ws": (I, [_P, _P, I64, _P, _P, I64, I64, _P, _P, _P, _P, SZ, _P]),
        "fm_in_proj_ws": (I, [_P, _P, I64, _P, _P, sp, _P, _P, _P, _P, _P, SZ, _P]),
        "fm_conv1d_pot": (I, [_P, I, I, sp, _P, _P, _P, _P, _P, _P]),
        "fm_ssm_scan_pot": (I, [_P, _P, I, I, sp, _P, _P, _P, _P, _P, _P, _P, SZ, _P]),
        "fm_scan_workspace_bytes": (SZ, [sp, I, I]),
        "fm_ssd_scan": (I, [_P, _P, I, I, sp, _P, _P, _P, _P, _P, _P, _P, SZ, _P]),
        "fm_ssd_workspace_bytes": (SZ, [sp, I, I]),
        "fm_set_scan_mode": (I, [I]),
        "fm_set_state_spec": (I, [I, I]),
        "fm_set_scan_tile": (I, [I, I, I]),
        "fm_gate_norm_quant": (I, [_P, _P, I64, sp, _P, _P, I, I, _P, _P, _P, _P, _P]),
        "fm_eval_pwl": (I, [I, _P, I64, _P, _P]),
        "fm_workspace_bytes": (SZ, [sp, I, I]),
        "fm_mixer_prefill": (I, [lp, _P, I, I, I, _P, _P, _P, _P, SZ, _P]),
        "fm_stack_prefill": (I, [_P, I, _P, I, I, _P, _P, I, _P, SZ, _P]),
        "fm_stack_prefill_host": (I, [_P, I, _P, _P, _P, I, I, _P, _P, I, _P, SZ, _P]),
        "fm_stack_workspace_bytes": (SZ, [sp, I, I, I, I]),
        "fm_decode_step": (I, [lp, _P, I, I, _P, _P, _P, _P, SZ, _P]),
        "fm_decode_step_noalloc": (I, [lp, _P, I, I, _P, _P, _P, _P]),
        "fm_prepare_mixer_params": (I, [sp, _P, _P, _P, _P, _P, _P, _P, _P]),
        "fm_calib_workspace_bytes": (SZ, [sp, I, I]),
        "fm_calibrate_layer": (I, [lp, _P, _P, _P, _P, _P, I, I, I, _P, _P, SZ, _P]),
        "fm_lq_conv1d": (I, [_P, I64, I, I, sp, _P, _P, _P, _P, _P]),
        "fm_lq_scan": (I, [_P, _P, I64, _P, I64, I, I, sp, _P, _P, _P, _P, _P, _P]),
        "fm_lq_workspace_bytes": (SZ, [sp, I, I]),
        "fm_set_fault_injection": (I, [I, C.c_uint64]),
        "fm_set_gemm_splitk": (I, [I]),
        "fm_set_gemm_tile": (I, [I]),
        "fm_set_pdl": (I, [I]),
        "fm_set_gemm_cluster": (I, [I]),
        "fm_set_lq_scan_cpw": (I, [I]),
        "fm_set_xbc_exponents": (I, [I]),
        "fm_conv1d_pot_tok": (I, [_P, I, I, sp, _P, _P, _P, _P, _P, _P, _P]),
        "fm_ssm_scan_pot_tok": (I, [_P, _P, I, I, sp, _P, _P, _P, _P, _P, _P, _P, _P, SZ, _P]),
        "fm_scan_workspace_bytes_tok": (SZ, [sp, I, I]),
        "fm_lq_mixer_prefill": (I, [lp, C.POINTER(fm_lq_params), _P, I, I, I, _P, _P, _P, _P,
                                    SZ, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libfastmamba takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("libfastmamba takes contiguous tensors only")
    return C.c_void_p(t.data_ptr())


def _s(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _check(status: int):
    if status != 0:
        raise FmError(status, load().fm_last_error().decode())


def shape_struct(shape) -> fm_shape:
    return fm_shape(shape.d_model, shape.d_inner, shape.headdim, shape.d_state, shape.ngroups,
                    shape.d_conv)


def exp_table_layout(shape) -> fm_exp_layout:
    return load().fm_exp_table_layout(C.byref(shape_struct(shape)))


def sync_status(stream=None):
    _check(load().fm_sync_status(_s(stream)))


STALL_GEMM, STALL_SCAN = 1, 2


def set_fault_injection(stall_mask: int, wait_limit_ns: int = 0):
    """Test hook: producers that issue nothing (STALL_GEMM, STALL_SCAN) and a
    shorter pipeline-wait limit; (0, 0) restores normal operation."""
    _check(load().fm_set_fault_injection(stall_mask, wait_limit_ns))


def hadamard_quant(x, K, prenorm_w, rotate, mode, static_amax, q, s_x, amax_row=None, stream=None):
    M = x.numel() // K
    _check(load().fm_hadamard_quant(_p(x), M, K, _p(prenorm_w), rotate, mode, _p(static_amax),
                                    _p(q), _p(s_x), _p(amax_row), _s(stream)))


def prepare_linear(W, rotate, Wq, s_w, stream=None):
    N, K = W.shape
    _check(load().fm_prepare_linear(_p(W), N, K, rotate, _p(Wq), _p(s_w), _s(stream)))


PDL_DEFAULT = True  # fm_set_pdl's default


def set_pdl(enable: bool):
    """Programmatic dependent launch of the hot kernels (on by default)."""
    _check(load().fm_set_pdl(int(bool(enable))))


GEMM_CLUSTER_DEFAULT = False


def set_gemm_cluster(enable: bool):
    """Split K over a thread-block cluster for decode-size GEMMs with fewer
    tiles than SMs (off by default: measured slower; the same bits either way)."""
    _check(load().fm_set_gemm_cluster(int(bool(enable))))


def set_gemm_tile(bn: int):
    """Tile width of the persistent GEMM: 0 (by the grid), 128 or 256."""
    _check(load().fm_set_gemm_tile(bn))


def set_gemm_splitk(enable: bool):
    """Split-K of the small-grid GEMMs (off by default); process-wide."""
    _check(load().fm_set_gemm_splitk(int(bool(enable))))


def gemm_workspace_bytes(M, N, K) -> int:
    """Bytes of workspace that let a small-grid GEMM split K (0: it would not)."""
    return load().fm_gemm_workspace_bytes(M, N, K)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def w8a8_gemm(A, s_x, Wq, s_w, Y, residual=None, acc_out=None, stream=None, ws=None):
    M, K = A.shape
    N = Wq.shape[0]
    if ws is None:
        _check(load().fm_w8a8_gemm(_p(A), _p(s_x), M, _p(Wq), _p(s_w), N, K, _p(residual), _p(Y),
                                   _p(acc_out), _s(stream)))
    else:
        _check(load().fm_w8a8_gemm_ws(_p(A), _p(s_x), M, _p(Wq), _p(s_w), N, K, _p(residual),
                                      _p(Y), _p(acc_out), _p(ws), _nbytes(ws), _s(stream)))


def in_proj(A, s_x, Wq, s_w, shape, exps, z, xbc, dt, stream=None, ws=None):
    sh = shape_struct(shape)
    if ws is None:
        _check(load().fm_in_proj(_p(A), _p(s_x), A.shape[0], _p(Wq), _p(s_w), C.byref(sh),
                                 _p(exps), _p(z), _p(xbc), _p(dt), _s(stream)))
    else:
        _check(load().fm_in_proj_ws(_p(A), _p(s_x), A.shape[0], _p(Wq), _p(s_w), C.byref(sh),
                                    _p(exps), _p(z), _p(xbc), _p(dt), _p(ws), _nbytes(ws),
                                    _s(stream)))


def conv1d_pot(u, B, T, shape, wq, bq, exps, conv_state, out, stream=None):
    sh = shape_struct(shape)
    _check(load().fm_conv1d_pot(_p(u), B, T, C.byref(sh), _p(wq), _p(bq), _p(exps),
                                _p(conv_state), _p(out), _s(stream)))


def conv1d_pot_tok(u, B, T, shape, wq, bq, exps, conv_state, out, e_tok, stream=None):
    sh = shape_struct(shape)
    _check(load().fm_conv1d_pot_tok(_p(u), B, T, C.byref(sh), _p(wq), _p(bq), _p(exps),
                                    _p(conv_state), _p(out), _p(e_tok), _s(stream)))


# (4, 0, 32): the default, channels per CTA chosen by the grid
SCAN_TILES = ((4, 0, 32), (4, 4, 32), (4, 8, 32), (4, 4, 16), (4, 2, 16), (4, 8, 16), (8, 4, 16),
              (8, 2, 16), (8, 8, 16))
SCAN_TILE_DEFAULT = (4, 0, 32)


def set_scan_tile(npt: int, pc: int, tch: int):
    _check(load().fm_set_scan_tile(npt, pc, tch))


STATE_BITS = 31  # the state spec in force (set_state_spec)


def set_state_spec(bits: int, guard: int):
    """(31, 0): the int32 state as built (default); (16, 7): the narrow state
    with the guard-bit increment, its state buffers int16.  Process-wide; set
    it before calibrating and allocating states."""
    global STATE_BITS
    _check(load().fm_set_state_spec(bits, guard))
    STATE_BITS = bits


XBC_EXPONENTS = "static"  # the conv-output exponent granularity in force


def set_xbc_exponents(kind: str):
    """'static' (per head / B / C, as built; default) or 'token' (per token);
    process-wide, set before calibrating and sizing workspaces."""
    global XBC_EXPONENTS
    _check(load().fm_set_xbc_exponents({"static": 0, "token": 1}[kind]))
    XBC_EXPONENTS = kind


def scan_workspace_bytes(shape, B, T) -> int:
    return load().fm_scan_workspace_bytes(C.byref(shape_struct(shape)), B, T)


def ssm_scan_pot(xbc, dt_raw, B, T, shape, dt_bias, A_q, D_q, exps, state, y, ws, stream=None):
    sh = shape_struct(shape)
    _check(load().fm_ssm_scan_pot(_p(xbc), _p(dt_raw), B, T, C.byref(sh), _p(dt_bias), _p(A_q),
                                  _p(D_q), _p(exps), _p(state), _p(y), _p(ws),
                                  ws.numel() * ws.element_size(), _s(stream)))


def scan_workspace_bytes_tok(shape, B, T) -> int:
    return load().fm_scan_workspace_bytes_tok(C.byref(shape_struct(shape)), B, T)


def ssm_scan_pot_tok(xbc, dt_raw, B, T, shape, dt_bias, A_q, D_q, exps, e_tok, state, y, ws,
                     stream=None):
    sh = shape_struct(shape)
    _check(load().fm_ssm_scan_pot_tok(_p(xbc), _p(dt_raw), B, T, C.byref(sh), _p(dt_bias),
                                      _p(A_q), _p(D_q), _p(exps), _p(e_tok), _p(state), _p(y),
                                      _p(ws), ws.numel() * ws.element_size(), _s(stream)))


SCAN_MODES = {"seq": 0, "ssd": 1}


def set_scan_mode(mode: str):
    """'seq' (the sequential fixed-point scan, default) or 'ssd' (the chunked
    tensor-core mode for prefills of more than one token)."""
    _check(load().fm_set_scan_mode(SCAN_MODES[mode]))


def ssd_workspace_bytes(shape, B, T) -> int:
    return load().fm_ssd_workspace_bytes(C.byref(shape_struct(shape)), B, T)


def ssd_scan(xbc, dt_raw, B, T, shape, dt_bias, A_q, D_q, exps, state, y, ws, stream=None):
    sh = shape_struct(shape)
    _check(load().fm_ssd_scan(_p(xbc), _p(dt_raw), B, T, C.byref(sh), _p(dt_bias), _p(A_q),
                              _p(D_q), _p(exps), _p(state), _p(y), _p(ws),
                              ws.numel() * ws.element_size(), _s(stream)))


def gate_norm_quant(y, z, shape, exps, norm_w, rotate, mode, static_amax, q, s_x, amax_row=None,
                    stream=None):
    sh = shape_struct(shape)
    M = y.numel() // shape.d_inner
    _check(load().fm_gate_norm_quant(_p(y), _p(z), M, C.byref(sh), _p(exps), _p(norm_w), rotate,
                                     mode, _p(static_amax), _p(q), _p(s_x), _p(amax_row),
                                     _s(stream)))


def eval_pwl(kind: int, inp, out, stream=None):
    _check(load().fm_eval_pwl(kind, _p(inp), inp.numel(), _p(out), _s(stream)))


def workspace_bytes(shape, B, T) -> int:
    return load().fm_workspace_bytes(C.byref(shape_struct(shape)), B, T)


def calib_workspace_bytes(shape, B, T) -> int:
    return load().fm_calib_workspace_bytes(C.byref(shape_struct(shape)), B, T)


def mixer_prefill(layer: fm_layer, x, B, T, residual, conv_state, ssm_state, out, ws,
                  stream=None):
    _check(load().fm_mixer_prefill(C.byref(layer), _p(x), B, T, residual, _p(conv_state),
                                   _p(ssm_state), _p(out), _p(ws), ws.numel() * ws.element_size(),
                                   _s(stream)))


def stack_workspace_bytes(shape, n_layers, B, T, n_chunks) -> int:
    return load().fm_stack_workspace_bytes(C.byref(shape_struct(shape)), n_layers, B, T, n_chunks)


def stack_prefill(layers, x, B, T, states, n_chunks, ws, stream=None):
    """layers: fm_layer structs; states: None or a list of (conv, ssm) tensors
    per layer.  The pointer arrays live for the call only (the library reads
    them while it queues the work)."""
    n = len(layers)
    larr = (C.POINTER(fm_layer) * n)(*[C.pointer(L) for L in layers])
    carr = sarr = None
    if states is not None:
        carr = (C.c_void_p * n)(*[_p(cs) for cs, _ in states])
        sarr = (C.c_void_p * n)(*[_p(ss) for _, ss in states])
    _check(load().fm_stack_prefill(C.cast(larr, C.c_void_p), n, _p(x), B, T,
                                   None if carr is None else C.cast(carr, C.c_void_p),
                                   None if sarr is None else C.cast(sarr, C.c_void_p), n_chunks,
                                   _p(ws), ws.numel() * ws.element_size(), _s(stream)))


def _host_ptr(t):
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("a contiguous host tensor is required")
    return C.c_void_p(t.data_ptr())


def stack_prefill_host(layers, x_host, out_host, x_dev, B, T, states, n_chunks, ws, stream=None):
    """fm_stack_prefill_host: x_host / out_host contiguous CPU tensors (pinned for
    the copies to overlap the compute), x_dev the device rows it works in."""
    n = len(layers)
    larr = (C.POINTER(fm_layer) * n)(*[C.pointer(L) for L in layers])
    carr = sarr = None
    if states is not None:
        carr = (C.c_void_p * n)(*[_p(cs) for cs, _ in states])
        sarr = (C.c_void_p * n)(*[_p(ss) for _, ss in states])
    _check(load().fm_stack_prefill_host(C.cast(larr, C.c_void_p), n, _host_ptr(x_host),
                                        _host_ptr(out_host), _p(x_dev), B, T,
                                        None if carr is None else C.cast(carr, C.c_void_p),
                                        None if sarr is None else C.cast(sarr, C.c_void_p),
                                        n_chunks, _p(ws), ws.numel() * ws.element_size(),
                                        _s(stream)))


def decode_step(layer: fm_layer, x, B, residual, conv_state, ssm_state, out, ws, stream=None):
    _check(load().fm_decode_step(C.byref(layer), _p(x), B, residual, _p(conv_state),
                                 _p(ssm_state), _p(out), _p(ws), ws.numel() * ws.element_size(),
                                 _s(stream)))


def decode_step_noalloc(layer: fm_layer, x, B, residual, conv_state, ssm_state, out,
                        stream=None):
    """fm_decode_step without a workspace: the library's fixed device scratch
    array is used instead (for callers that cannot allocate device memory)."""
    _check(load().fm_decode_step_noalloc(C.byref(layer), _p(x), B, residual, _p(conv_state),
                                         _p(ssm_state), _p(out), _s(stream)))


def prepare_mixer_params(shape, conv_w, a_log, D, conv_wq, A_q, D_q, exps, stream=None):
    sh = shape_struct(shape)
    _check(load().fm_prepare_mixer_params(C.byref(sh), _p(conv_w), _p(a_log), _p(D),
                                          _p(conv_wq), _p(A_q), _p(D_q), _p(exps), _s(stream)))


def calibrate_layer(layer: fm_layer, conv_b, exps, conv_bq, static_amax, xcal, B, T, residual,
                    out, ws, stream=None):
    _check(load().fm_calibrate_layer(C.byref(layer), _p(conv_b), _p(exps), _p(conv_bq),
                                     _p(static_amax), _p(xcal), B, T, residual, _p(out), _p(ws),
                                     ws.numel() * ws.element_size(), _s(stream)))


# ------------------------------------------------------------------ FastMamba-LQ
def _p_any(t):
    """A CUDA tensor's address without the contiguity check (strided row views)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libfastmamba takes CUDA tensors only")
    return C.c_void_p(t.data_ptr())


def _row_view(t, width):
    """(pointer, row stride) of a 2-D view whose rows are unit-stride."""
    if t.dim() != 2 or t.stride(1) != 1 or t.shape[1] != width:
        raise ValueError("expected a [rows, width] view with unit column stride")
    return _p_any(t), t.stride(0)


def lq_conv1d(u, B, T, shape, conv_w, conv_b, conv_state, out, stream=None):
    """u: [B*T, conv_ch] rows (may be a column slice of a wider buffer)."""
    sh = shape_struct(shape)
    pu, ldu = _row_view(u, shape.conv_ch)
    _check(load().fm_lq_conv1d(pu, ldu, B, T, C.byref(sh), _p(conv_w), _p(conv_b),
                               _p(conv_state), _p(out), _s(stream)))


def lq_scan(xo, dt_raw, z, B, T, shape, dt_bias, a_log, D, state, out, stream=None):
    """dt_raw: [B*T, nheads] rows, z: [B*T, d_inner] rows or None (slices allowed)."""
    sh = shape_struct(shape)
    pdt, lddt = _row_view(dt_raw, shape.nheads)
    pz, ldz = _row_view(z, shape.d_inner) if z is not None else (None, 0)
    _check(load().fm_lq_scan(_p(xo), pdt, lddt, pz, ldz, B, T, C.byref(sh), _p(dt_bias),
                             _p(a_log), _p(D), _p(state), _p(out), _s(stream)))


def set_lq_scan_cpw(cpw: int):
    """Channels per warp of the LQ scan: 0 (by the grid), 1, 2 or 4."""
    _check(load().fm_set_lq_scan_cpw(cpw))


def lq_workspace_bytes(shape, B, T) -> int:
    return load().fm_lq_workspace_bytes(C.byref(shape_struct(shape)), B, T)


def lq_mixer_prefill(layer: fm_layer, params: fm_lq_params, x, B, T, residual, conv_state,
                     ssm_state, out, ws, stream=None):
    _check(load().fm_lq_mixer_prefill(C.byref(layer), C.byref(params), _p(x), B, T, residual,
                                      _p(conv_state), _p(ssm_state), _p(out), _p(ws),
                                      ws.numel() * ws.element_size(), _s(stream)))
