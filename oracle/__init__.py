"""CPU oracle of the quantised Mamba2 mixer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and
its binding) never imports it, and it imports nothing from the product.

Two parts:
  * ``fm_oracle.c`` -- the quantised method step by step (plain C, fp32 /
    fp64 IEEE arithmetic with no FMA contraction, integer fixed point),
    loaded through ctypes; this module composes those steps into the
    mixer, the stack and the calibration.
  * ``ref_mixer_f64`` -- the unquantised Mamba2 mixer in numpy fp64 with
    exact exp / softplus / SiLU, the reference for SQNR and for the
    "naive double recurrence" check.
  * ``stages`` -- a mixer whose stages are each quantised or exact, for the
    per-stage error attribution and the linears-only FastMamba-LQ variant.

Sources are the web pages about FastMamba (arXiv 2505.18975); citations
use the page's section (see fm_oracle.c for the full list).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fm_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")

DYNAMIC, STATIC = 0, 1
E_ZERO = -30

_lib = None


def build(force: bool = False) -> str:
    """Compile fm_oracle.c into oracle/_build/liboracle.so (gcc, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _declare(_lib)
    return _lib


_P = C.c_void_p
_I64 = C.c_int64
_I = C.c_int
_F = C.c_float


def _declare(L):
    sig = {
        "fmo_rshr": (_I64, [_I64, _I]),
        "fmo_sat": (_I64, [_I64, _I]),
        "fmo_to_q16": (C.c_int32, [_F]),
        "fmo_pot_exponent": (_I, [C.c_double, C.c_double]),
        "fmo_fwht256_f32": (None, [_P]),
        "fmo_fwht256_f64": (None, [_P]),
        "fmo_hadamard_quant": (None, [_P, _I64, _I64, _P, _I, _I, _F, _P, _P, _P]),
        "fmo_prepare_linear": (None, [_P, _I64, _I64, _I, _P, _P]),
        "fmo_gemm_i8": (None, [_P, _P, _I64, _I64, _I64, _P]),
        "fmo_dequant": (None, [_P, _P, _P, _I64, _I64, _P, _P]),
        "fmo_in_proj_epilogue": (None, [_P, _P, _P, _I64, _I, _I, _I, _P, _P, _P, _P]),
        "fmo_pwl_coef": (_I64, [_I, _I]),
        "fmo_pow2_pwl": (_I64, [_I64]),
        "fmo_exp_pwl": (_I64, [_I64]),
        "fmo_softplus_pwl": (_I64, [_I64]),
        "fmo_silu_pwl": (_I64, [_I64]),
        "fmo_prepare_conv": (None, [_P, _P, _I, _P, _P, _P, _P]),
        "fmo_conv1d_pot": (None, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
        "fmo_prepare_ssm": (None, [_P, _P, _I, _P, _P, _P]),
        "fmo_ssm_scan_pot": (None, [_P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P,
                                    _I, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
        "fmo_ssm_scan_pot_x": (None, [_P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P,
                                      _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _P, _I]),
        "fmo_scan_state_amax": (None, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
        "fmo_scan_state_amax_x": (None, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _I]),
        "fmo_conv1d_pot_x": (None, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "fmo_requant_per_token": (None, [_P, _I64, _I, _I, _I, _P, _P, _P]),
        "fmo_gate_norm_quant": (None, [_P, _P, _I64, _I, _I, _P, _I, _P, _I, _I, _F,
                                       _P, _P, _P, _P]),
        "fmo_eval_array": (None, [_I, _P, _I64, _I, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def _c(a, dtype):
    """Contiguous array of dtype (no copy when already so)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


# ---------------------------------------------------------------- scalars / arrays

def rshr(a: int, s: int) -> int:
    return lib().fmo_rshr(int(a), int(s))


def pot_exponent(amax: float, Q: float) -> int:
    return lib().fmo_pot_exponent(float(amax), float(Q))


def pwl_coefficients():
    """(P[0..8], S[0..7], LOG2E_Q15) as the oracle derives them."""
    L = lib()
    return ([L.fmo_pwl_coef(0, i) for i in range(9)], [L.fmo_pwl_coef(1, i) for i in range(8)],
            L.fmo_pwl_coef(2, 0))


def eval_array(kind: str, x, shift: int = 0) -> np.ndarray:
    kinds = {"pow2": 0, "exp": 1, "softplus": 2, "silu": 3, "rshr": 4, "to_q16": 5}
    if kind == "to_q16":
        x = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.int64)
    x = _c(x, np.int64)
    out = np.empty_like(x)
    lib().fmo_eval_array(kinds[kind], _p(x), x.size, shift, _p(out))
    return out


def fwht256(v: np.ndarray) -> np.ndarray:
    """Block-diagonal (256) Sylvester Hadamard rotation of the last axis (fp32 or fp64)."""
    dt = np.float64 if v.dtype == np.float64 else np.float32
    out = np.array(v, dtype=dt, order="C", copy=True)
    fn = lib().fmo_fwht256_f64 if dt == np.float64 else lib().fmo_fwht256_f32
    flat = out.reshape(-1, 256)
    step = flat.strides[0]
    base = flat.ctypes.data
    for i in range(flat.shape[0]):
        fn(C.c_void_p(base + i * step))
    return out


# ---------------------------------------------------------------- stages

def hadamard_quant(x, prenorm_w=None, rotate=1, mode=DYNAMIC, static_amax=0.0, want_amax=False):
    x = _c(x, np.float32)
    M, K = x.reshape(-1, x.shape[-1]).shape
    q = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    am = np.empty(M, np.float32) if want_amax else None
    pw = None if prenorm_w is None else _c(prenorm_w, np.float32)
    lib().fmo_hadamard_quant(_p(x), M, K, _p(pw), rotate, mode, float(static_amax),
                             _p(q), _p(sx), _p(am))
    return (q, sx, am) if want_amax else (q, sx)


def prepare_linear(W, rotate=1):
    W = _c(W, np.float32)
    N, K = W.shape
    wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    lib().fmo_prepare_linear(_p(W), N, K, rotate, _p(wq), _p(sw))
    return wq, sw


def gemm_i8(A, W):
    A = _c(A, np.int8)
    W = _c(W, np.int8)
    M, K = A.shape
    N = W.shape[0]
    acc = np.empty((M, N), np.int32)
    lib().fmo_gemm_i8(_p(A), _p(W), M, N, K, _p(acc))
    return acc


def dequant(acc, sx, sw, residual=None):
    acc = _c(acc, np.int32)
    M, N = acc.shape
    Y = np.empty((M, N), np.float32)
    r = None if residual is None else _c(residual, np.float32).reshape(M, N)
    lib().fmo_dequant(_p(acc), _p(_c(sx, np.float32)), _p(_c(sw, np.float32)), M, N, _p(r), _p(Y))
    return Y


def in_proj_epilogue(acc, sx, sw, di, cc, nh, e_u):
    acc = _c(acc, np.int32)
    M = acc.shape[0]
    z = np.empty((M, di), np.float32)
    xbc = np.empty((M, cc), np.int8)
    dt = np.empty((M, nh), np.float32)
    lib().fmo_in_proj_epilogue(_p(acc), _p(_c(sx, np.float32)), _p(_c(sw, np.float32)), M,
                               di, cc, nh, _p(_c(e_u, np.int32)), _p(z), _p(xbc), _p(dt))
    return z, xbc, dt


def prepare_conv(w, b, e_u=None):
    w = _c(w, np.float32)
    cc = w.shape[0]
    wq = np.empty((cc, 4), np.int8)
    e_w = np.empty(cc, np.int32)
    bq = np.empty(cc, np.int32) if e_u is not None else None
    lib().fmo_prepare_conv(_p(w), _p(_c(b, np.float32)), cc,
                           _p(None if e_u is None else _c(e_u, np.int32)), _p(wq), _p(bq), _p(e_w))
    return wq, bq, e_w


def conv1d_pot(u, wq, bq, e_u, e_w, e_o, conv_state=None, want_amax=False, want_s16=False):
    """u: int8 [B, T, cc]; conv_state (int8 [B,3,cc]) is updated in place.
    want_s16 adds the Q.16 SiLU values before requantisation (int32 [B,T,cc])."""
    u = _c(u, np.int8)
    Bsz, T, cc = u.shape
    out = np.empty_like(u)
    am = np.zeros(cc, np.int64) if want_amax else None
    s16 = np.empty((Bsz, T, cc), np.int32) if want_s16 else None
    if conv_state is not None:
        assert conv_state.dtype == np.int8 and conv_state.flags.c_contiguous
    lib().fmo_conv1d_pot_x(_p(u), Bsz, T, cc, _p(_c(wq, np.int8)),
                           _p(None if bq is None else _c(bq, np.int32)), _p(_c(e_u, np.int32)),
                           _p(_c(e_w, np.int32)), _p(_c(e_o, np.int32)), _p(conv_state), _p(out),
                           _p(am), _p(s16))
    res = [out] + ([am] if want_amax else []) + ([s16] if want_s16 else [])
    return res[0] if len(res) == 1 else tuple(res)


def requant_per_token(s16, nh, hd, ds, e_o):
    """Per-token PoT requantisation of the conv's Q.16 SiLU values [B,T,cc]:
    returns (int8 codes [B,T,cc], exponents int32 [B,T,nh+2])."""
    s16 = _c(s16, np.int32)
    Bsz, T, cc = s16.shape
    codes = np.empty((Bsz, T, cc), np.int8)
    e_tok = np.empty((Bsz, T, nh + 2), np.int32)
    lib().fmo_requant_per_token(_p(s16), Bsz * T, nh, hd, ds, _p(_c(e_o, np.int32)), _p(e_tok),
                                _p(codes))
    return codes, e_tok


def prepare_ssm(a_log, D):
    nh = len(a_log)
    A_q = np.empty(nh, np.int32)
    D_q = np.empty(nh, np.int32)
    e_D = np.empty(nh, np.int32)
    lib().fmo_prepare_ssm(_p(_c(a_log, np.float32)), _p(_c(D, np.float32)), nh, _p(A_q), _p(D_q),
                          _p(e_D))
    return A_q, D_q, e_D


def ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D, hd, ds,
                 state=None, want_dt=False, want_ystat=False, state_bits=31, e_tok=None,
                 ub_guard=0):
    """xbc int8 [B,T,cc] (conv output), dt_raw fp32 [B,T,nh]; state int32 [B,nh,hd,ds]
    is updated in place.  Returns y int32 [B,T,nh*hd] (+ extras).  state_bits
    is the state word's width reading (31: the method as built; 16: int16);
    e_tok (int32 [B,T,nh+2]) gives per-token exponents of x, B, C; ub_guard
    (0 as built, else guard bits) rounds the increment after the u B product."""
    xbc = _c(xbc, np.int8)
    Bsz, T, cc = xbc.shape
    nh = len(A_q)
    y = np.empty((Bsz, T, nh * hd), np.int32)
    dtq = np.empty((Bsz, T, nh), np.int32) if want_dt else None
    dA = np.empty((Bsz, T, nh), np.int32) if want_dt else None
    ys = np.zeros(nh, np.int64) if want_ystat else None
    if state is not None:
        assert state.dtype == np.int32 and state.flags.c_contiguous
    if not 8 <= state_bits <= 31:
        raise ValueError("state_bits must be in [8, 31]")
    if not 0 <= ub_guard <= 7:
        raise ValueError("ub_guard must be in [0, 7]")
    if ub_guard and state_bits + ub_guard > 24:
        # u keeps its 24-bit saturation (u B inside 32 bits), so with g guard
        # bits an increment saturates at 2^(23-g) state LSBs per unit of B
        # code: harmless only when the state word itself is no wider
        raise ValueError("ub_guard needs state_bits + ub_guard <= 24")
    et = None if e_tok is None else _c(e_tok, np.int32)
    if et is not None:
        assert et.shape == (Bsz, T, nh + 2)
    lib().fmo_ssm_scan_pot_x(_p(xbc), _p(_c(dt_raw, np.float32)), _p(_c(dt_bias, np.float32)),
                             _p(_c(A_q, np.int32)), _p(_c(D_q, np.int32)), _p(_c(e_x, np.int32)),
                             int(e_B), int(e_C), _p(_c(e_h, np.int32)), _p(_c(e_y, np.int32)),
                             _p(_c(e_D, np.int32)), Bsz, T, nh, hd, ds, _p(state), _p(y), _p(dtq),
                             _p(dA), _p(ys), int(state_bits), _p(et), int(ub_guard))
    out = [y]
    if want_dt:
        out += [dtq, dA]
    if want_ystat:
        out += [ys]
    return out[0] if len(out) == 1 else tuple(out)


def scan_state_amax(xbc, dt_raw, dt_bias, A_q, hd, ds, e_tok=None, e_x=None, e_B=0):
    """Max |h| per head at the finest exponent e_x + e_B - 15; with per-token
    exponents e_tok, at that of the static e_x, e_B given."""
    xbc = _c(xbc, np.int8)
    Bsz, T, cc = xbc.shape
    nh = len(A_q)
    am = np.zeros(nh, np.int64)
    et = None if e_tok is None else _c(e_tok, np.int32)
    lib().fmo_scan_state_amax_x(_p(xbc), _p(_c(dt_raw, np.float32)), _p(_c(dt_bias, np.float32)),
                                _p(_c(A_q, np.int32)), Bsz, T, nh, hd, ds, _p(am), _p(et),
                                _p(None if e_x is None else _c(e_x, np.int32)), int(e_B))
    return am


def gate_norm_quant(y, z, hd, e_y, e_g, norm_w, rotate=1, mode=DYNAMIC, static_amax=0.0,
                    want_amax=False, want_gstat=False):
    y = _c(y, np.int32)
    di = y.shape[-1]
    M = y.size // di
    q = np.empty((M, di), np.int8)
    sx = np.empty(M, np.float32)
    am = np.empty(M, np.float32) if want_amax else None
    nh = di // hd
    gs = np.zeros(nh, np.int64) if want_gstat else None
    lib().fmo_gate_norm_quant(_p(y), _p(_c(z, np.float32)), M, di, hd, _p(_c(e_y, np.int32)),
                              int(e_g), _p(_c(norm_w, np.float32)), rotate, mode,
                              float(static_amax), _p(q), _p(sx), _p(am), _p(gs))
    out = [q, sx]
    if want_amax:
        out.append(am)
    if want_gstat:
        out.append(gs)
    return tuple(out)


# ---------------------------------------------------------------- the layer

@dataclass
class Layer:
    """A prepared (and, once calibrated, complete) quantised mixer layer."""
    shape: object
    rotate: int
    mode: int
    wq_in: np.ndarray
    sw_in: np.ndarray
    wq_out: np.ndarray
    sw_out: np.ndarray
    conv_wq: np.ndarray
    conv_e_w: np.ndarray
    conv_w: np.ndarray      # fp32 taps (kept to quantise the bias once e_u is known)
    conv_b: np.ndarray      # fp32 bias
    A_q: np.ndarray
    D_q: np.ndarray
    e_D: np.ndarray
    dt_bias: np.ndarray
    norm_w: np.ndarray
    prenorm_w: np.ndarray | None
    # calibrated
    e_u: np.ndarray | None = None
    conv_bq: np.ndarray | None = None
    e_x: np.ndarray | None = None
    e_B: int = 0
    e_C: int = 0
    e_h: np.ndarray | None = None
    e_y: np.ndarray | None = None
    e_g: int = 0
    amax_in: float = 0.0
    amax_out: float = 0.0
    state_bits: int = 31    # state word width reading (31 as built; 16 the int16 reading)
    xbc_exponents: str = "static"   # conv output exponents: "static" per head, or "token"
    ub_guard: int = 0       # 0 as built; g: the increment rounded after u B, u with g more bits
    scan_mode: str = "seq"  # "seq": the sequential fixed-point scan; "ssd": the chunked form
    ssd_chunk: int = 64
    extra: dict = field(default_factory=dict)

    def e_o(self) -> np.ndarray:
        """Per conv channel output exponent: e_x per head for x, e_B, e_C."""
        s = self.shape
        return np.concatenate([np.repeat(self.e_x, s.headdim),
                               np.full(s.d_state, self.e_B), np.full(s.d_state, self.e_C)]
                              ).astype(np.int32)

    def exponents(self) -> dict:
        return dict(e_u=self.e_u, e_w=self.conv_e_w, e_x=self.e_x, e_B=self.e_B, e_C=self.e_C,
                    e_h=self.e_h, e_y=self.e_y, e_D=self.e_D, e_g=self.e_g,
                    amax_in=self.amax_in, amax_out=self.amax_out)


def prepare_layer(params: dict, shape, rotate=1, mode=DYNAMIC, prenorm=False,
                  state_bits=31, xbc_exponents="static", ub_guard=0) -> Layer:
    if xbc_exponents not in ("static", "token"):
        raise ValueError("xbc_exponents is 'static' or 'token'")
    if ub_guard and state_bits + ub_guard > 24:
        raise ValueError("ub_guard needs state_bits + ub_guard <= 24")
    wq_in, sw_in = prepare_linear(params["w_in"], rotate)
    wq_out, sw_out = prepare_linear(params["w_out"], rotate)
    wq, _, e_w = prepare_conv(params["conv_w"], params["conv_b"])
    A_q, D_q, e_D = prepare_ssm(params["a_log"], params["D"])
    return Layer(shape=shape, rotate=rotate, mode=mode, wq_in=wq_in, sw_in=sw_in,
                 wq_out=wq_out, sw_out=sw_out, conv_wq=wq, conv_e_w=e_w,
                 conv_w=_c(params["conv_w"], np.float32), conv_b=_c(params["conv_b"], np.float32), A_q=A_q, D_q=D_q, e_D=e_D,
                 dt_bias=_c(params["dt_bias"], np.float32), norm_w=_c(params["norm_w"], np.float32),
                 prenorm_w=_c(params["prenorm_w"], np.float32) if prenorm else None,
                 state_bits=int(state_bits), xbc_exponents=xbc_exponents,
                 ub_guard=int(ub_guard))


def set_conv_input_exponents(L: Layer, e_u):
    """Fix the conv input exponents and quantise the conv bias at e_w + e_u."""
    L.e_u = _c(e_u, np.int32)
    _, L.conv_bq, _ = prepare_conv(L.conv_w, L.conv_b, L.e_u)


def conv_out(L: Layer, xbc, conv_state=None):
    """The conv stage's int8 output for the layer's exponent reading:
    (codes [B,T,cc], per-token exponents [B,T,nh+2] or None when static)."""
    s = L.shape
    if L.xbc_exponents == "static":
        return conv1d_pot(xbc, L.conv_wq, L.conv_bq, L.e_u, L.conv_e_w, L.e_o(), conv_state), None
    _, s16 = conv1d_pot(xbc, L.conv_wq, L.conv_bq, L.e_u, L.conv_e_w, L.e_o(), conv_state,
                        want_s16=True)
    return requant_per_token(s16, s.nheads, s.headdim, s.d_state, L.e_o())


def mixer_prefill(L: Layer, x, residual=False, conv_state=None, ssm_state=None, trace=None):
    """One layer on x fp32 [B,T,dm].  Stacks pass residual=True (and a layer
    prepared with prenorm): out = x + mixer(RMSNorm(x)).  States update in place."""
    s = L.shape
    Bsz, T, dm = x.shape
    M = Bsz * T
    di, cc, nh, hd, ds = s.d_inner, s.conv_ch, s.nheads, s.headdim, s.d_state
    q, sx = hadamard_quant(x.reshape(M, dm), L.prenorm_w, L.rotate, L.mode, L.amax_in)
    acc = gemm_i8(q, L.wq_in)
    z, xbc, dt = in_proj_epilogue(acc, sx, L.sw_in, di, cc, nh, L.e_u)
    xo, e_tok = conv_out(L, xbc.reshape(Bsz, T, cc), conv_state)
    if L.scan_mode == "ssd" and T > 1:   # single steps stay sequential
        from .ssd import ssd_scan
        if e_tok is not None or L.state_bits != 31:
            raise ValueError("the chunked scan follows static exponents and the 31-bit state")
        y = ssd_scan(xo, dt.reshape(Bsz, T, nh), L.dt_bias, L.A_q, L.D_q, L.e_x, L.e_B, L.e_C,
                     L.e_h, L.e_y, L.e_D, hd, ds, Q=L.ssd_chunk, state=ssm_state)
    else:
        y = ssm_scan_pot(xo, dt.reshape(Bsz, T, nh), L.dt_bias, L.A_q, L.D_q, L.e_x, L.e_B,
                         L.e_C, L.e_h, L.e_y, L.e_D, hd, ds, ssm_state,
                         state_bits=L.state_bits, e_tok=e_tok, ub_guard=L.ub_guard)
    q2, sx2 = gate_norm_quant(y.reshape(M, di), z, hd, L.e_y, L.e_g, L.norm_w, L.rotate, L.mode,
                              L.amax_out)
    acc2 = gemm_i8(q2, L.wq_out)
    out = dequant(acc2, sx2, L.sw_out, x.reshape(M, dm) if residual else None)
    if trace is not None:
        trace.update(q_in=q, sx_in=sx, acc_in=acc, z=z, xbc=xbc, dt=dt, conv_out=xo, y=y,
                     q_out=q2, sx_out=sx2, acc_out=acc2)
    return out.reshape(Bsz, T, dm)


def calibrate_layer(L: Layer, xcal, residual=False):
    """Stage-by-stage calibration on the quantised pipeline (16 seeded sequences
    in the workloads).  Each stage's exponent comes from the max of that
    stage's pre-quantisation value over the calibration tokens, with the
    exponents of earlier stages already fixed.  Fills L in place and returns
    the layer's output on xcal (the next layer's calibration input)."""
    s = L.shape
    Bsz, T, dm = xcal.shape
    M = Bsz * T
    di, cc, nh, hd, ds = s.d_inner, s.conv_ch, s.nheads, s.headdim, s.d_state
    x2 = xcal.reshape(M, dm)
    # in_proj input: static amax = max of the rotated (normed) input
    q, sx, am = hadamard_quant(x2, L.prenorm_w, L.rotate, DYNAMIC, 0.0, want_amax=True)
    L.amax_in = float(am.max())
    if L.mode == STATIC:
        q, sx = hadamard_quant(x2, L.prenorm_w, L.rotate, STATIC, L.amax_in)
    acc = gemm_i8(q, L.wq_in)
    Y = dequant(acc, sx, L.sw_in)
    amax_u = np.abs(Y[:, di:di + cc]).max(axis=0)
    set_conv_input_exponents(L, [pot_exponent(a, 127.0) for a in amax_u])
    z, xbc, dt = in_proj_epilogue(acc, sx, L.sw_in, di, cc, nh, L.e_u)
    xbc = xbc.reshape(Bsz, T, cc)
    # conv output exponents (per head for x, one each for B and C)
    _, am_s = conv1d_pot(xbc, L.conv_wq, L.conv_bq, L.e_u, L.conv_e_w, np.zeros(cc, np.int32),
                         want_amax=True)
    L.e_x = np.array([pot_exponent(am_s[h * hd:(h + 1) * hd].max(), 127.0) - 16
                      for h in range(nh)], np.int32)
    L.e_B = pot_exponent(am_s[di:di + ds].max(), 127.0) - 16
    L.e_C = pot_exponent(am_s[di + ds:].max(), 127.0) - 16
    xo, e_tok = conv_out(L, xbc)
    dt3 = dt.reshape(Bsz, T, nh)
    # state exponent: 64-bit run at the finest exponent, headroom 2^29 of the
    # 2^30 clamp (2^(bits-2) of 2^(bits-1) for a narrower state word)
    am_h = scan_state_amax(xo, dt3, L.dt_bias, L.A_q, hd, ds, e_tok, L.e_x, L.e_B)
    e_f = L.e_x + L.e_B - 15
    head = 2.0 ** (L.state_bits - 2)
    L.e_h = np.array([max(pot_exponent(float(am_h[h]), head) + int(e_f[h]), int(e_f[h]))
                      for h in range(nh)], np.int32)
    # output exponent from max |y| at the finer term exponent
    _, ys = ssm_scan_pot(xo, dt3, L.dt_bias, L.A_q, L.D_q, L.e_x, L.e_B, L.e_C, L.e_h,
                         np.zeros(nh, np.int32), L.e_D, hd, ds, want_ystat=True,
                         state_bits=L.state_bits, e_tok=e_tok, ub_guard=L.ub_guard)
    e_f = np.minimum(L.e_C + L.e_h, L.e_D + L.e_x)
    lo = np.maximum(L.e_C + L.e_h, L.e_D + L.e_x) - 16
    L.e_y = np.array([max(pot_exponent(float(ys[h]), 2.0 ** 29) + int(e_f[h]), int(lo[h]))
                      for h in range(nh)], np.int32)
    y = ssm_scan_pot(xo, dt3, L.dt_bias, L.A_q, L.D_q, L.e_x, L.e_B, L.e_C, L.e_h, L.e_y, L.e_D,
                     hd, ds, state_bits=L.state_bits, e_tok=e_tok, ub_guard=L.ub_guard)
    # gate exponent (int16 g), then the out_proj input amax
    # (the statistic does not depend on e_g; the pass uses its lower bound so
    # that every gate shift is a right shift)
    _, _, gs = gate_norm_quant(y.reshape(M, di), z, hd, L.e_y, int(L.e_y.max()) - 16, L.norm_w,
                               L.rotate, DYNAMIC, 0.0, want_gstat=True)
    L.e_g = int(max(max(pot_exponent(float(gs[h]), 32767.0) + int(L.e_y[h]) - 16
                        for h in range(nh)), int(L.e_y.max()) - 16))
    q2, sx2, am2 = gate_norm_quant(y.reshape(M, di), z, hd, L.e_y, L.e_g, L.norm_w, L.rotate,
                                   DYNAMIC, 0.0, want_amax=True)
    L.amax_out = float(am2.max())
    if L.mode == STATIC:
        q2, sx2 = gate_norm_quant(y.reshape(M, di), z, hd, L.e_y, L.e_g, L.norm_w, L.rotate,
                                  STATIC, L.amax_out)
    acc2 = gemm_i8(q2, L.wq_out)
    out = dequant(acc2, sx2, L.sw_out, x2 if residual else None)
    return out.reshape(Bsz, T, dm)


# ---------------------------------------------------------------- fp64 reference

def _silu(v):
    return v / (1.0 + np.exp(-v))


def _softplus(v):
    return np.logaddexp(0.0, v)


def ref_conv_f64(xBC, w, b):
    """Causal depthwise conv, kernel 4: out[t,c] = b[c] + sum_k w[c,k] x[t-3+k, c]."""
    Bsz, T, cc = xBC.shape
    xp = np.concatenate([np.zeros((Bsz, 3, cc)), xBC], axis=1)
    return b + sum(w[:, k] * xp[:, k:k + T] for k in range(4))


def ref_scan_f64(xs, Bm, Cm, dt, A, D, h0=None):
    """Mamba2 selective scan, one group, zero-order hold (the paper's references
    [2], [14]): dA = exp(dt A); h = dA h + dt x B^T; y = h C + D x.
    xs [B,T,nh,hd], Bm/Cm [B,T,ds], dt [B,T,nh]; returns y [B,T,nh,hd], h."""
    Bsz, T, nh, hd = xs.shape
    ds = Bm.shape[-1]
    dA = np.exp(dt * A)
    h = np.zeros((Bsz, nh, hd, ds)) if h0 is None else np.array(h0, np.float64)
    y = np.empty((Bsz, T, nh, hd))
    for t in range(T):
        h = dA[:, t, :, None, None] * h + (dt[:, t, :, None] * xs[:, t])[..., None] \
            * Bm[:, t, None, None, :]
        y[:, t] = np.einsum("bhpn,bn->bhp", h, Cm[:, t]) + D[None, :, None] * xs[:, t]
    return y, h


def ref_mixer_f64(params: dict, shape, x, prenorm=False, residual=False, return_state=False,
                  stats=None):
    """Unquantised Mamba2 mixer (the paper's reference [2]; flow of Fig. 2) in
    fp64 with exact nonlinearities: in_proj -> causal depthwise conv + SiLU ->
    selective scan (dt = softplus(dt_raw + dt_bias), dA = exp(dt A),
    h = dA h + dt x B, y = C.h + D x) -> y * SiLU(z) -> RMSNorm -> out_proj.
    ``stats`` (a dict, optional) receives the per-channel max |.| of the two
    linears' inputs over all tokens ("in_absmax", "out_absmax")."""
    s = shape
    di, ds, nh, hd, cc = s.d_inner, s.d_state, s.nheads, s.headdim, s.conv_ch
    x = np.asarray(x, np.float64)
    Bsz, T, dm = x.shape
    u = x
    if prenorm:
        u = u / np.sqrt((u * u).mean(-1, keepdims=True) + 1e-5) * params["prenorm_w"]
    Y = u @ params["w_in"].astype(np.float64).T
    if stats is not None:
        stats["in_absmax"] = np.abs(u).reshape(-1, dm).max(axis=0)
    z, xBC, dt_raw = Y[..., :di], Y[..., di:di + cc], Y[..., di + cc:]
    xc = _silu(ref_conv_f64(xBC, params["conv_w"].astype(np.float64),
                             params["conv_b"].astype(np.float64)))
    xs, Bm, Cm = xc[..., :di].reshape(Bsz, T, nh, hd), xc[..., di:di + ds], xc[..., di + ds:]
    dt = _softplus(dt_raw + params["dt_bias"].astype(np.float64))
    A = -np.exp(params["a_log"].astype(np.float64))
    y, h = ref_scan_f64(xs, Bm, Cm, dt, A, params["D"].astype(np.float64))
    g = y.reshape(Bsz, T, di) * _silu(z)
    g = g / np.sqrt((g * g).mean(-1, keepdims=True) + 1e-5) * params["norm_w"]
    if stats is not None:
        stats["out_absmax"] = np.abs(g).reshape(-1, di).max(axis=0)
    out = g @ params["w_out"].astype(np.float64).T
    if residual:
        out = out + x
    return (out, h) if return_state else out


def sqnr_db(ref, q) -> float:
    ref = np.asarray(ref, np.float64)
    err = np.asarray(q, np.float64) - ref
    return float(10.0 * np.log10((ref * ref).sum() / max((err * err).sum(), 1e-300)))
