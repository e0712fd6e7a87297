"""fp64 oracle of the per-head steps around the KDA operator (test infrastructure).

Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
algorithm", the paragraph on what each KDA head applies: a short depthwise
convolution of kernel size 4 followed by a Swish activation on the queries,
keys and values; L2 normalisation of the queries and keys; and, on the
output, a head-wise RMSNorm followed by a sigmoid output gate.

Readings (the pages give no formulas):
  * the convolution is causal, over time, one 4-tap filter per channel
    (depthwise), without bias; tap 3 multiplies the current token and tap 0
    the token three positions back; tokens before a sequence's first token
    count as zero (a packed batch never convolves across sequences);
  * Swish is x * sigmoid(x);
  * the L2 normalisation of q and k is over the dk channels of one (token,
    head): x / sqrt(sum x^2 + eps);
  * the head-wise RMSNorm is over the dv channels of one (token, head):
    o / sqrt(mean o^2 + eps), times a weight vector of length dv shared by
    the heads, and the output gate multiplies by sigmoid(gate) elementwise,
    gate being a tensor of the output's shape.

Only ``tests/`` may import this module.  Plain numpy in fp64, written from the
definitions above; no blocking or reordering.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def _seq_starts(total: int, cu_seqlens) -> np.ndarray:
    """Index of the first token of the sequence that each token belongs to."""
    start = np.zeros(total, dtype=np.int64)
    if cu_seqlens is None:
        return start
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    for s in range(len(cu) - 1):
        start[cu[s]:cu[s + 1]] = cu[s]
    return start


def causal_conv4(x, w, cu_seqlens=None) -> np.ndarray:
    """Depthwise causal convolution over time.

    x [total, H, d]; w [H * d, 4] (tap 3 = current token).  Returns
    y[t, h, c] = sum_{i=0..3} w[h d + c, i] * x[t - 3 + i, h, c], with x taken
    as zero before the first token of t's sequence."""
    x = _f64(x)
    w = _f64(w)
    total, H, d = x.shape
    start = _seq_starts(total, cu_seqlens)
    wt = w.reshape(H, d, 4)
    y = np.zeros_like(x)
    for t in range(total):
        for i in range(4):
            src = t - 3 + i
            if src >= start[t]:
                y[t] += wt[:, :, i] * x[src]
    return y


def swish(x) -> np.ndarray:
    x = _f64(x)
    return x / (1.0 + np.exp(-x))


def l2_normalize(x, eps: float) -> np.ndarray:
    """x / sqrt(sum over the last axis of x^2 + eps)."""
    x = _f64(x)
    return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)


def qkv_conv_norm(xq, xk, xv, wq, wk, wv, cu_seqlens=None, eps: float = 1e-6):
    """q, k, v as the operator takes them: conv + Swish on each, then L2 norm
    of q and k (in fp64)."""
    q = l2_normalize(swish(causal_conv4(xq, wq, cu_seqlens)), eps)
    k = l2_normalize(swish(causal_conv4(xk, wk, cu_seqlens)), eps)
    v = swish(causal_conv4(xv, wv, cu_seqlens))
    return q, k, v


def output_norm_gate(o, gate, w, eps: float = 1e-6) -> np.ndarray:
    """Head-wise RMSNorm of o over its last axis, times w, times sigmoid(gate)."""
    o = _f64(o)
    gate = _f64(gate)
    w = _f64(w)
    rms = np.sqrt((o * o).mean(axis=-1, keepdims=True) + eps)
    return o / rms * w / (1.0 + np.exp(-gate))
