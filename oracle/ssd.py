"""Chunked (state-space-dual) form of the power-of-two selective scan -- TEST
INFRASTRUCTURE ONLY (same rules as the rest of ``oracle``).

The FastMamba pages run the scan as a sequential fixed-point recurrence (the
SSM module of Fig. 7, one step per token).  Mamba2's own algorithm (the
paper's reference [2], "Transformers are SSMs") computes the same
recurrence chunk by chunk as matrix products, which is what a GPU's tensor
cores can run.  This module defines that chunked form on the method's
quantised inputs, as a separate scan mode with its own error budget (it
cannot reproduce the sequential form's per-step roundings):

inputs (per sequence and head, as in the sequential scan)
  X[t, p], Bq[t, n], Cq[t, n]   the conv's int8 codes (exponents e_x, e_B, e_C)
  dt_q[t]                       the PWL SoftPlus of dt_raw + dt_bias (Q.16)
  w[t] = -rshr(dt_q[t] A_q, 12) the step's log2 decay (Q.16), as the
                                sequential scan feeds its 2^v unit
chunks of Q tokens from the first token of the call; inside chunk c
(tokens t0 .. t0+Q-1):
  W[t]     = sum_{k=t0..t} w[k]                     (exact integer)
  a(s, t)  = fl32(2^(fl32((W[t] - W[s]) 2^-16)))    decay from after s to t
  a0(t)    = fl32(2^(fl32(W[t] 2^-16)))             from the chunk's start
  dtf[s]   = dt_q[s] 2^-16                          (exact in fp32)
  intra:  G = Cq Bq^T (exact integer), for s <= t
          M[t, s] = op(fl32(G[t, s] * fl32(a(s, t) dtf[s])))
  inter:  Ca[t, n] = op(fl32(a0(t) Cq[t, n]))
  both in one sum (one accumulator on the tensor cores):
          Y[t, p] = fl32(sum_s M[t, s] X[s, p] + sum_n Ca[t, n] op(H[p, n]))
  state:  K[s] = fl32(a(s, end) dtf[s]);  U[s, n] = op(fl32(K[s] Bq[s, n]))
          H <- fl32(fl32(a0(end) H) + fl32(sum_s X[s, p] U[s, n]))
  output: y[t, p] = sat32(rint(Y[t, p] 2^(e_C+e_x+e_B-e_y)) + rshr(D_q X[t, p], s_D))
A layer in this mode (``scan_mode = "ssd"``) runs it for calls of more than
one token; single decode steps stay sequential.
H is the state in code units (2^(e_x+e_B)); it enters from and leaves to the
sequential scan's int32 word at e_h: H = h 2^(e_h-e_x-e_B), h =
sat31(rint(H 2^(e_x+e_B-e_h))), so a chunked prefill hands over to the
sequential decode step.  op() is the tensor-core operand rounding: bf16
(round to nearest even) or none ("fp32").  Sums are formed exactly (fp64
over exact products) and rounded once to fp32; a GPU's fp32 accumulation
differs from that by at most its own rounding, which the parity tolerance
of this mode covers.

With op = none and one chunk the mode is the exact recurrence
h_t = 2^(w_t) h_{t-1} + dt_t x_t B_t^T on the codes, up to fp32 rounding;
the tests pin it to the fp64 recurrence with the same decays.
"""
from __future__ import annotations

import numpy as np

from . import ssm_scan_pot

F32 = np.float32


def bf16(v):
    """Round fp32 values to bfloat16 (nearest, ties to even), returned as fp32."""
    v = np.ascontiguousarray(v, F32)
    u = v.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(F32)


def _op(v, operand):
    return bf16(v) if operand == "bf16" else np.asarray(v, F32)


def _pow2(e_q16):
    """fl32(2^(fl32(e 2^-16))) for integer exponents e <= 0 (Q.16)."""
    ef = (np.asarray(e_q16, np.float64) * 2.0 ** -16).astype(F32)
    return np.exp2(ef.astype(np.float64)).astype(F32)


def decay_exponents(xbc, dt_raw, dt_bias, A_q, hd, ds):
    """dt_q [B,T,nh] from the oracle's fixed-point unit and the log2 decay
    w = -rshr(dt_q A_q, 12) [B,T,nh] (Q.16)."""
    nh = len(A_q)
    z = np.zeros(nh, np.int32)
    _, dtq, _ = ssm_scan_pot(xbc, dt_raw, dt_bias, A_q, z, z, 0, 0, z, z, z, hd, ds,
                             want_dt=True)
    v = dtq.astype(np.int64) * np.asarray(A_q, np.int64)[None, None, :]
    w = -((v + (1 << 11)) >> 12)
    return dtq, w


def ssd_scan(xbc, dt_raw, dt_bias, A_q, D_q, e_x, e_B, e_C, e_h, e_y, e_D, hd, ds, Q=64,
             state=None, operand="bf16", want_f32=False):
    """The chunked scan: xbc int8 [B,T,cc], dt_raw fp32 [B,T,nh]; state int32
    [B,nh,hd,ds] at e_h (updated in place).  Returns y int32 [B,T,nh*hd]
    (and the fp32 SSM part before the skip term, in code units, if want_f32)."""
    if operand not in ("bf16", "fp32"):
        raise ValueError("operand is 'bf16' or 'fp32'")
    xbc = np.ascontiguousarray(xbc, np.int8)
    Bsz, T, cc = xbc.shape
    nh = len(A_q)
    di = nh * hd
    dtq, w = decay_exponents(xbc, dt_raw, dt_bias, A_q, hd, ds)
    y = np.empty((Bsz, T, di), np.int32)
    yf_all = np.empty((Bsz, T, di), F32) if want_f32 else None
    for b in range(Bsz):
        Bq = xbc[b, :, di:di + ds].astype(np.float64)
        Cq = xbc[b, :, di + ds:].astype(np.float64)
        for h in range(nh):
            X = xbc[b, :, h * hd:(h + 1) * hd].astype(np.float64)
            u_sh = int(e_h[h]) - int(e_x[h]) - int(e_B)          # state word -> code units
            H = np.zeros((hd, ds), F32)
            if state is not None:
                H = (state[b, h].astype(np.float64) * 2.0 ** u_sh).astype(F32)
            dtf = (dtq[b, :, h].astype(np.float64) * 2.0 ** -16).astype(F32)
            for t0 in range(0, T, Q):
                t1 = min(T, t0 + Q)
                W = np.cumsum(w[b, t0:t1, h])                     # exact int64
                n = t1 - t0
                # intra-chunk
                G = Cq[t0:t1] @ Bq[t0:t1].T                       # exact integers
                diff = W[:, None] - W[None, :]                    # W[t] - W[s]
                low = np.tril(np.ones((n, n), bool))
                a = np.where(low, _pow2(np.where(low, diff, 0)), F32(0))
                ad = (a * dtf[None, t0:t1]).astype(F32)           # fl32(a(s,t) dtf[s])
                M = _op((G.astype(F32) * ad).astype(F32), operand)
                # inter-chunk, from the state entering the chunk: the decay
                # from the chunk's start scales C before the operand rounding
                a0 = _pow2(W)
                Ca = _op((a0[:, None] * Cq[t0:t1].astype(F32)).astype(F32), operand)
                yf = (M.astype(np.float64) @ X[t0:t1] +
                      Ca.astype(np.float64) @ _op(H, operand).astype(np.float64).T).astype(F32)
                # state leaving the chunk
                K = (_pow2(W[-1] - W) * dtf[t0:t1]).astype(F32)
                U = _op((K[:, None] * Bq[t0:t1].astype(F32)).astype(F32), operand)
                dH = (X[t0:t1].T @ U.astype(np.float64)).astype(F32)
                H = ((a0[-1] * H).astype(F32) + dH).astype(F32)
                # output codes
                s_y = int(e_C) + int(e_x[h]) + int(e_B) - int(e_y[h])
                ycode = np.rint((yf.astype(np.float64) * 2.0 ** s_y).astype(F32).astype(np.float64))
                s_D = int(e_y[h]) - int(e_D[h]) - int(e_x[h])
                dx = np.asarray(D_q[h], np.int64) * X[t0:t1].astype(np.int64)
                skip = _rshr_vec(dx, s_D)
                tot = ycode + skip.astype(np.float64)
                y[b, t0:t1, h * hd:(h + 1) * hd] = np.clip(tot, -2147483647, 2147483647)
                if want_f32:
                    yf_all[b, t0:t1, h * hd:(h + 1) * hd] = yf
            if state is not None:
                hs = np.rint(H.astype(np.float64) * 2.0 ** -u_sh)
                state[b, h] = np.clip(hs, -(2 ** 30 - 1), 2 ** 30 - 1).astype(np.int32)
    return (y, yf_all) if want_f32 else y


def _rshr_vec(a, s):
    """rshr on int64 arrays: floor((a + 2^(s-1)) / 2^s) for s > 0, a 2^-s for s <= 0."""
    a = np.asarray(a, np.int64)
    if s > 0:
        return (a + (1 << (s - 1))) >> s
    return a << (-s)
