"""Seeded synthetic inputs for the quantised Mamba2 mixer.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no rotation, quantisation, fixed point or recurrence).
Both the CPU oracle (through the tests) and the CUDA path consume what it
returns, so the two sides always see the same inputs.

Distributions follow the synthetic workloads used for the FastMamba
(arXiv 2505.18975) Mamba2-130M / Mamba2-2.7B shapes:
  * linear weights ~ N(0, 0.02);
  * A_log = log U[1, 16];
  * dt_bias = inverse-softplus of dt ~ U[1e-3, 1e-1];
  * depthwise conv taps ~ N(0, 0.2), conv bias 0;
  * D = 1, norm weights = 1;
  * activations ~ N(0, 1) with a few seed-chosen outlier channels scaled
    up (Mamba has attention-like outlier channels: Mamba-PTQ, arXiv
    2407.12397, abstract).
Every tensor gets its own PCG64 stream: seed = base + tensor id.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import numpy as np


@dataclass(frozen=True)
class MixerShape:
    d_model: int
    d_inner: int
    headdim: int
    d_state: int
    ngroups: int = 1
    d_conv: int = 4

    @property
    def nheads(self) -> int:
        return self.d_inner // self.headdim

    @property
    def conv_ch(self) -> int:  # channels of the causal conv: x, B, C
        return self.d_inner + 2 * self.ngroups * self.d_state

    @property
    def n_in(self) -> int:  # in_proj output width: z, x, B, C, dt
        return 2 * self.d_inner + 2 * self.ngroups * self.d_state + self.nheads

    def as_dict(self):
        d = asdict(self)
        d.update(nheads=self.nheads, conv_ch=self.conv_ch, n_in=self.n_in)
        return d


MAMBA2_130M = MixerShape(d_model=768, d_inner=1536, headdim=64, d_state=128)
MAMBA2_2P7B = MixerShape(d_model=2560, d_inner=5120, headdim=64, d_state=128)

# tensor ids inside one layer's seed block
_T_WIN, _T_WOUT, _T_CONVW, _T_ALOG, _T_DT = 1, 2, 3, 4, 5


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def layer_params(shape: MixerShape, seed: int, conv_bias_std: float = 0.0) -> dict:
    """Random-init fp32 parameters of one Mamba2 mixer layer.

    `seed` identifies the layer; each tensor draws from seed*16 + tensor id.
    `conv_bias_std` > 0 draws a non-zero conv bias (unit tests only).
    """
    s = shape
    base = seed * 16
    w_in = _rng(base + _T_WIN).normal(0.0, 0.02, (s.n_in, s.d_model))
    w_out = _rng(base + _T_WOUT).normal(0.0, 0.02, (s.d_model, s.d_inner))
    r = _rng(base + _T_CONVW)
    conv_w = r.normal(0.0, 0.2, (s.conv_ch, s.d_conv))
    conv_b = (r.normal(0.0, conv_bias_std, s.conv_ch) if conv_bias_std > 0
              else np.zeros(s.conv_ch))
    a_log = np.log(_rng(base + _T_ALOG).uniform(1.0, 16.0, s.nheads))
    dt = _rng(base + _T_DT).uniform(1e-3, 1e-1, s.nheads)
    dt_bias = dt + np.log(-np.expm1(-dt))  # softplus(dt_bias) == dt
    f32 = lambda a: np.ascontiguousarray(a, dtype=np.float32)
    return dict(
        w_in=f32(w_in), w_out=f32(w_out), conv_w=f32(conv_w), conv_b=f32(conv_b),
        a_log=f32(a_log), dt_bias=f32(dt_bias), D=np.ones(s.nheads, np.float32),
        norm_w=np.ones(s.d_inner, np.float32), prenorm_w=np.ones(s.d_model, np.float32),
    )


def outlier_channels(d: int, n_outliers: int, seed: int) -> np.ndarray:
    """Seed-chosen outlier channel indices (without replacement), sorted."""
    if n_outliers <= 0:
        return np.zeros(0, np.int64)
    return np.sort(_rng(seed).choice(d, n_outliers, replace=False))


def activations(batch: int, seqlen: int, d: int, seed: int, n_outliers: int = 8,
                outlier_scale: float = 50.0, outlier_seed: int | None = None) -> np.ndarray:
    """fp32 [batch, seqlen, d] ~ N(0,1); the same outlier channels for every token
    are multiplied by `outlier_scale` after sampling."""
    x = _rng(seed).standard_normal((batch, seqlen, d))
    ch = outlier_channels(d, n_outliers, seed + 7 if outlier_seed is None else outlier_seed)
    x[..., ch] *= outlier_scale
    return np.ascontiguousarray(x, dtype=np.float32)


def uniform_ints(shape, lo: int, hi: int, seed: int, dtype=np.int32) -> np.ndarray:
    """Integers uniform in [lo, hi] (both ends included) for stage-level unit tests."""
    return np.ascontiguousarray(_rng(seed).integers(lo, hi + 1, size=shape), dtype=dtype)


def normal(shape, std: float, seed: int, mean: float = 0.0) -> np.ndarray:
    return np.ascontiguousarray(_rng(seed).normal(mean, std, shape), dtype=np.float32)


# The five workloads (sizes only).  Calibration uses 16 seeded sequences of
# min(seqlen, 512) tokens drawn like the workload's own inputs.
WORKLOADS = {
    "mixer130m_b1_t256": dict(shape=MAMBA2_130M, layers=1, batch=1, seqlen=256,
                              n_outliers=8, outlier_scale=50.0),
    "stack130m_24l_b1_t2048": dict(shape=MAMBA2_130M, layers=24, batch=1, seqlen=2048,
                                   n_outliers=8, outlier_scale=50.0),
    "gemm2p7b_inproj": dict(shape=MAMBA2_2P7B, m_list=(2048, 8192, 32768),
                            n_outliers=16, outlier_scale=100.0),
    "stack2p7b_64l_b2_t4096": dict(shape=MAMBA2_2P7B, layers=64, batch=2, seqlen=4096,
                                   n_outliers=8, outlier_scale=50.0),
    "decode2p7b_64l_b64": dict(shape=MAMBA2_2P7B, layers=64, batch=64, seqlen=1,
                               prefill_len=512, n_outliers=8, outlier_scale=50.0),
}
CALIB_SEQS = 16
CALIB_MAX_LEN = 512
CALIB_SEED0 = 10000


def calibration_batch(d: int, seqlen: int, n_outliers: int, outlier_scale: float,
                      outlier_seed: int, n_seqs: int = CALIB_SEQS) -> np.ndarray:
    """[n_seqs, min(seqlen, 512), d] calibration inputs (seeds 10000..), with the
    same outlier channels as the workload they calibrate for."""
    t = min(seqlen, CALIB_MAX_LEN)
    return np.concatenate([
        activations(1, t, d, CALIB_SEED0 + i, n_outliers, outlier_scale, outlier_seed)
        for i in range(n_seqs)], axis=0)
