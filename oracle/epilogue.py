"""Output epilogue of a KDA layer in float64 (numpy).

TEST INFRASTRUCTURE ONLY.  Shares no code with ``ref`` or the CUDA path.

Kimi Linear summary, §4 "The Kimi Linear Model Architecture": the attention
output of each head is normalised by its root mean square over the head's
features (head-wise RMSNorm), then scaled feature by feature into (0, 1) by a
data-dependent sigmoid gate; the output projection comes after and is not part
of the operator.  §5.2 (ablations) fixes the gate's nonlinearity as a sigmoid,
not Swish.

Per token t and head h, over the dv features j of that head:

    y[t,h,j] = o[t,h,j] / sqrt(mean_j' o[t,h,j']^2 + eps) * w[j] * sigmoid(r[t,h,j])

The pages name neither a gain nor an epsilon: ``w`` is an optional per-feature
gain shared by the heads (ones when absent) and ``eps`` is the caller's.  The
gate input ``r`` comes from the layer's low-rank projection, outside the
operator; tests draw it at random.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    """numpy float64 copy of an array or a CPU torch tensor (exact widening)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, np.float64)


def sigmoid(x):
    """1 / (1 + e^{-x}), split by sign so neither branch overflows."""
    x = _f64(x)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    e = np.exp(x[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def rms_normalise(o, eps):
    """o / sqrt(mean of o^2 over the last axis + eps), float64."""
    o = _f64(o)
    return o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)


def norm_gate(o, r, weight=None, eps=1e-6):
    """y = RMSNorm(o) * w * sigmoid(r) over the last axis (a head's features).

    o, r: [..., dv] (any float dtype, widened to float64); weight: [dv] or None."""
    y = rms_normalise(o, eps)
    if weight is not None:
        y = y * _f64(weight)
    return y * sigmoid(r)
