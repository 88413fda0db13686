"""Input prologue of a KDA layer in float64 (numpy).

TEST INFRASTRUCTURE ONLY.  Shares no code with ``ref`` or the CUDA path.

Kimi Linear summary, §4 "The Kimi Linear Model Architecture": KDA captures
dependencies between neighbouring tokens with a short convolution and applies
a Swish nonlinearity to the queries, keys and values; queries and keys are then
normalised to unit length (that last step is inside the operator itself).

The pages give neither the width nor the form of the convolution.  The
reading taken here is the plainest one: a causal depthwise convolution along
the token axis, one filter of ``width`` taps per channel, no bias, that never
reaches across a sequence boundary (inputs before a sequence's first token are
zeros).  Per channel c of token t in a sequence that starts at token a:

    u[t,c] = sum_{i=0}^{width-1} w[c,i] * x[t-(width-1)+i, c]   (x[s,c] = 0 for s < a)
    y[t,c] = u[t,c] * sigmoid(u[t,c])                            (Swish / SiLU)

so w[c, width-1] weighs the current token and w[c, 0] the oldest one.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, np.float64)


def swish(u):
    """u * sigmoid(u), split by sign so nothing overflows."""
    u = _f64(u)
    e = np.exp(-np.abs(u))
    sig = np.where(u >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return u * sig


def causal_conv(x, w, cu_seqlens=None, num_seqs=1):
    """u = the causal depthwise convolution above, before the Swish.

    x: [T, ..., C] (the channel axes after the token axis are flattened);
    w: [C_total, width] with C_total the product of x's trailing axes;
    cu_seqlens: [N+1] token offsets, or None for ``num_seqs`` equal sequences."""
    x = _f64(x)
    w = _f64(w)
    T = x.shape[0]
    xf = x.reshape(T, -1)
    width = w.shape[1]
    if cu_seqlens is None:
        L = T // num_seqs if num_seqs else 0
        cu = np.arange(num_seqs + 1) * L
    else:
        cu = np.asarray(_f64(cu_seqlens), np.int64)
    u = np.zeros_like(xf)
    for n in range(len(cu) - 1):
        a, b = int(cu[n]), int(cu[n + 1])
        for t in range(a, b):
            for i in range(width):
                s = t - (width - 1) + i
                if s >= a:
                    u[t] += w[:, i] * xf[s]
    return u.reshape(x.shape)


def short_conv_swish(x, w, cu_seqlens=None, num_seqs=1):
    """y = Swish(causal depthwise convolution of x), float64."""
    return swish(causal_conv(x, w, cu_seqlens, num_seqs))
