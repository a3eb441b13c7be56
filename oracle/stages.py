"""Stage-by-stage error attribution and the FastMamba-LQ variant -- TEST
INFRASTRUCTURE ONLY (same rules as the rest of ``oracle``).

``staged_mixer`` runs one Mamba2 mixer layer in which each stage of the
quantised method is, independently, either the oracle's quantised step or
the exact fp64 computation of ``ref_mixer_f64``:

  ``lin``   the two linears as Hadamard-rotated W8A8 (FastMamba, arXiv
            2505.18975, "Hadamard-based 8-bit quantization of the linear
            layers"; Algorithm 1)
  ``conv``  the causal conv1d on power-of-two int8 codes with the PWL SiLU
            (the "power-of-two quantization" of the conv1d)
  ``pwl``   dt = SoftPlus and dA = exp(dt A) through the 8-segment 2^v unit
            (Eq. (5) and its symmetric form for x > 0; dA as a shift-based
            exponential)
  ``scan``  the fixed-point selective scan on int8 x / B / C codes (the
            "power-of-two quantization" of the SSM block); implies ``pwl``,
            which the fixed-point scan always uses
  ``gate``  the PWL-SiLU gate with the int16 gated value and the integer
            RMSNorm sum; implies ``lin`` (its output is the out_proj's int8
            input)

One more switch, ``eq5``, is not a pipeline stage: it takes dt from the
first-order SoftPlus form of Eq. (5) (e^x for x <= 0, x + e^-x above) in
exact fp64 arithmetic, to separate the error of that form from the error of
the 8-segment 2^v chords and the Q.16 words (``pwl``, which overrides it).

Where an exact stage feeds a quantised one, the exact value is quantised at
the calibrated exponent of that boundary (sat(rint(v 2^-e)), in fp64); where
a quantised stage feeds an exact one, its codes are dequantised exactly
(code 2^e).  With every stage quantised the function is ``mixer_prefill``
bit for bit; with none it is ``ref_mixer_f64`` up to fp64 summation order.

FastMamba-LQ -- the variant with only the linear layers quantised, which
the paper's Table II reports beside the fully quantised model (pith.science
review of FastMamba, "Desk Editor's Note": LQ at the FP16 average accuracy
on Mamba2-130M, the full model about half a point below) -- is the
``lin``-only case (``lq_mixer``).  The linears' static activation scales are
those the full pipeline calibrated.
"""
from __future__ import annotations

import numpy as np

from . import (conv1d_pot, dequant, gate_norm_quant, gemm_i8, hadamard_quant, in_proj_epilogue,
               ref_conv_f64, ssm_scan_pot, _silu, _softplus)

STAGES = ("lin", "conv", "pwl", "scan", "gate")


def _codes(v, e, bits):
    """sat_bits(rint(v 2^-e)) of fp64 values, e broadcast over the last axis."""
    lim = 2.0 ** (bits - 1) - 1
    return np.clip(np.rint(np.asarray(v, np.float64) * np.exp2(-np.asarray(e, np.float64))),
                   -lim, lim)


def _scan_f64(xs, Bm, Cm, dt, dA, D):
    """h = dA h + dt x B^T; y = h C + D x (one group), fp64, dA given."""
    Bsz, T, nh, hd = xs.shape
    h = np.zeros((Bsz, nh, hd, Bm.shape[-1]))
    y = np.empty((Bsz, T, nh, hd))
    for t in range(T):
        h = dA[:, t, :, None, None] * h + (dt[:, t, :, None] * xs[:, t])[..., None] \
            * Bm[:, t, None, None, :]
        y[:, t] = np.einsum("bhpn,bn->bhp", h, Cm[:, t]) + D[None, :, None] * xs[:, t]
    return y


def staged_mixer(L, params: dict, x, quant=(), residual=False):
    """One layer on x [B,T,dm] with the stages named in ``quant`` quantised
    (L a calibrated oracle layer, params its fp32 weights).  Returns fp64
    [B,T,dm] (the fp32 output of the quantised steps, widened)."""
    if L.xbc_exponents != "static":
        raise ValueError("the staged mixer follows the static conv-output exponents")
    quant = set(quant)
    bad = quant - set(STAGES) - {"eq5"}
    if bad:
        raise ValueError(f"unknown stages {sorted(bad)}")
    if "scan" in quant:
        quant.add("pwl")
    if "gate" in quant and "lin" not in quant:
        raise ValueError("a quantised gate writes the out_proj's int8 input: it needs 'lin'")
    s = L.shape
    di, cc, nh, hd, ds = s.d_inner, s.conv_ch, s.nheads, s.headdim, s.d_state
    x32 = np.ascontiguousarray(x, np.float32)
    Bsz, T, dm = x32.shape
    M = Bsz * T
    x64 = x32.astype(np.float64)
    e_o = L.e_o()
    e_y = np.repeat(L.e_y, hd)                                  # per channel of y

    # ---- in_proj: z, the conv input (codes or fp64) and dt_raw (fp32)
    xbc_q = xbc_f = None
    if "lin" in quant:
        q, sx = hadamard_quant(x32.reshape(M, dm), L.prenorm_w, L.rotate, L.mode, L.amax_in)
        acc = gemm_i8(q, L.wq_in)
        if "conv" in quant:
            z, xbc_q, dt_raw = in_proj_epilogue(acc, sx, L.sw_in, di, cc, nh, L.e_u)
        else:
            Y = dequant(acc, sx, L.sw_in)
            z, xbc_f, dt_raw = Y[:, :di], Y[:, di:di + cc].astype(np.float64), Y[:, di + cc:]
        z = z.astype(np.float64)
    else:
        u = x64.reshape(M, dm)
        if L.prenorm_w is not None:
            u = u / np.sqrt((u * u).mean(-1, keepdims=True) + 1e-5) * L.prenorm_w
        Y = u @ params["w_in"].astype(np.float64).T
        z, xbc_f, dt_raw = Y[:, :di], Y[:, di:di + cc], Y[:, di + cc:]
        if "conv" in quant:
            xbc_q = _codes(xbc_f, L.e_u, 8).astype(np.int8)

    # ---- conv + SiLU: x / B / C as codes at e_o or as fp64
    xo_q = xo_f = None
    if "conv" in quant:
        xo_q = conv1d_pot(xbc_q.reshape(Bsz, T, cc), L.conv_wq, L.conv_bq, L.e_u, L.conv_e_w, e_o)
        if "scan" not in quant:
            xo_f = xo_q.astype(np.float64) * np.exp2(e_o.astype(np.float64))
    else:
        xo_f = _silu(ref_conv_f64(xbc_f.reshape(Bsz, T, cc), params["conv_w"].astype(np.float64),
                                  params["conv_b"].astype(np.float64)))
        if "scan" in quant:
            xo_q = _codes(xo_f, e_o, 8).astype(np.int8)
    dt3 = np.ascontiguousarray(dt_raw, np.float32).reshape(Bsz, T, nh)   # the PWL unit's input
    dt_f = np.asarray(dt_raw, np.float64).reshape(Bsz, T, nh)

    # ---- dt, dA and the scan: y as int32 codes at e_y or as fp64
    if "scan" in quant:
        y_q = ssm_scan_pot(xo_q, dt3, L.dt_bias, L.A_q, L.D_q, L.e_x, L.e_B, L.e_C, L.e_h, L.e_y,
                           L.e_D, hd, ds, state_bits=L.state_bits).reshape(M, di)
        y_f = y_q.astype(np.float64) * np.exp2(e_y.astype(np.float64))
    else:
        if "pwl" in quant:
            # the oracle's own dt / dA (they do not depend on the x / B / C codes)
            _, dtq, dAq = ssm_scan_pot(np.zeros((Bsz, T, cc), np.int8), dt3, L.dt_bias, L.A_q,
                                       L.D_q, L.e_x, L.e_B, L.e_C, L.e_h, L.e_y, L.e_D, hd, ds,
                                       want_dt=True)
            dt, dA = dtq / 65536.0, dAq / 65536.0
        else:
            v = dt_f + params["dt_bias"].astype(np.float64)
            if "eq5" in quant:
                dt = np.where(v <= 0.0, np.exp(np.minimum(v, 0.0)), v + np.exp(-np.abs(v)))
            else:
                dt = _softplus(v)
            dA = np.exp(dt * -np.exp(params["a_log"].astype(np.float64)))
        y_f = _scan_f64(xo_f[..., :di].reshape(Bsz, T, nh, hd), xo_f[..., di:di + ds],
                        xo_f[..., di + ds:], dt, dA,
                        params["D"].astype(np.float64)).reshape(M, di)
        y_q = _codes(y_f, e_y, 32).astype(np.int32) if "gate" in quant else None

    # ---- gate + gated RMSNorm + out_proj
    res = x32.reshape(M, dm) if residual else None
    if "gate" in quant:
        q2, sx2 = gate_norm_quant(y_q, z.astype(np.float32), hd, L.e_y, L.e_g, L.norm_w, L.rotate,
                                  L.mode, L.amax_out)
        out = dequant(gemm_i8(q2, L.wq_out), sx2, L.sw_out, res).astype(np.float64)
    else:
        g = y_f * _silu(z)
        g = g / np.sqrt((g * g).mean(-1, keepdims=True) + 1e-5) * params["norm_w"]
        if "lin" in quant:
            q2, sx2 = hadamard_quant(g.astype(np.float32), None, L.rotate, L.mode, L.amax_out)
            out = dequant(gemm_i8(q2, L.wq_out), sx2, L.sw_out, res).astype(np.float64)
        else:
            out = g @ params["w_out"].astype(np.float64).T
            if residual:
                out = out + x64.reshape(M, dm)
    return out.reshape(Bsz, T, dm)


def lq_mixer(L, params: dict, x, residual=False):
    """FastMamba-LQ: rotated W8A8 linears, everything else exact (fp64)."""
    return staged_mixer(L, params, x, ("lin",), residual)
