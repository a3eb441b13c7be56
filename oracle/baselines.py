"""Comparison arms for the rotated W8A8 linears -- TEST INFRASTRUCTURE ONLY
(same rules as the rest of ``oracle``).

The pages compare FastMamba's Hadamard-rotated 8-bit linears with plain
("normal") per-token / per-channel W8A8 and with SmoothQuant (pith.science
review of FastMamba, forward implications and supporting citation [7]: the
rotated quantiser beats both on perplexity and seven zero-shot tasks for
Mamba2-130M).  Both arms run on the same quantised steps as the method with
the rotation switched off:

  * normal W8A8: ``prepare_layer(..., rotate=0)``;
  * SmoothQuant (reference [7] of the paper): each input channel j of a
    linear is divided by s_j = max|X_j|^alpha / max_n |W[n, j]|^(1 - alpha)
    and the weight's column j multiplied by s_j, so X W^T is unchanged while
    the activation outliers move into the weights.  In a Mamba2 block both
    linears follow an RMSNorm with a per-channel weight (the pre-norm before
    in_proj, the gated norm before out_proj), so 1/s folds into that weight
    and the quantised kernels run unchanged.  max|X_j| comes from the
    unquantised fp64 mixer on the calibration set, as SmoothQuant takes it
    from the floating-point model; alpha = 0.5 is its default.
"""
from __future__ import annotations

import numpy as np

from . import ref_mixer_f64


def activation_absmax(params: dict, shape, xcal):
    """Per input channel max |activation| of in_proj and out_proj over the
    calibration tokens (fp64 mixer, pre-norm form)."""
    st = {}
    ref_mixer_f64(params, shape, xcal, prenorm=True, residual=True, stats=st)
    return st["in_absmax"], st["out_absmax"]


def smoothing_factors(act_absmax, W, alpha=0.5):
    """s_j = max|X_j|^alpha / max_n |W[n, j]|^(1 - alpha); 1 where either max is 0."""
    a = np.asarray(act_absmax, np.float64)
    w = np.abs(np.asarray(W, np.float64)).max(axis=0)
    s = np.ones_like(a)
    ok = (a > 0) & (w > 0)
    s[ok] = a[ok] ** alpha / w[ok] ** (1.0 - alpha)
    return s


def smooth_params(params: dict, shape, xcal, alpha=0.5) -> dict:
    """The layer's fp32 parameters with SmoothQuant folded in (pre-norm form:
    1/s into prenorm_w and norm_w, s into the weight columns)."""
    a_in, a_out = activation_absmax(params, shape, xcal)
    s_in = smoothing_factors(a_in, params["w_in"], alpha)
    s_out = smoothing_factors(a_out, params["w_out"], alpha)
    q = dict(params)
    q["prenorm_w"] = (params["prenorm_w"].astype(np.float64) / s_in).astype(np.float32)
    q["w_in"] = (params["w_in"].astype(np.float64) * s_in).astype(np.float32)
    q["norm_w"] = (params["norm_w"].astype(np.float64) / s_out).astype(np.float32)
    q["w_out"] = (params["w_out"].astype(np.float64) * s_out).astype(np.float32)
    return q
