"""Float64 short causal convolution of the KDA inputs, with packed-document resets, an optional
SiLU and an optional per-group L2 normalisation (the input prologue of the recurrence).

TEST INFRASTRUCTURE ONLY: part of the independent checker (see oracle/__init__.py for who may
import it). Plain NumPy in float64; shares no code with gated_delta_rule_144_b200.

Passages it follows:
- NeMo glm5_next layers, ``_TorchShortConvolution``: a depthwise causal Conv1d over
  [batch, sequence, channels] that resets at packed boundaries, with one ``weight`` parameter
  (``kernel_size`` taps per channel) and no bias named; ``Glm5NextLinearAttention`` holds one for
  each of q, k and v (``q_conv1d``, ``k_conv1d``, ``v_conv1d``), of size
  ``linear_conv_kernel_dim``.
- The workloads of this recurrence: q and k arrive L2-normalised per head vector.

Readings (the formula is not printed):
- causal Conv1d with W taps as PyTorch applies it with W - 1 positions of left padding:
  y[t, c] = sum_{j < W} w[c, j] x[t - (W - 1) + j, c]; the last tap multiplies the current token;
  positions before the start of the token's document contribute zero (the reset);
- the page names no activation; an optional SiLU, y * sigmoid(y), is offered (the FLA module it
  matches takes one), off unless asked for;
- L2 normalisation of each group of g consecutive channels (a head vector when g = head_dim):
  y / sqrt(sum over the group of y^2 + eps).
Pinned in tests/test_oracle_short_conv.py.
"""

from __future__ import annotations

import numpy as np


def short_conv(x, weight, cu_seqlens=None, activation: str = "none", norm_group: int = 0,
               eps: float = 1e-6):
    """x: [B, T, C]; weight: [C, W]; cu_seqlens: None or int [N + 1] (then B = 1): documents
    x[0, cu[d]:cu[d + 1]]. Returns y [B, T, C] in float64."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    B, T, C = x.shape
    W = w.shape[1]
    if w.shape[0] != C:
        raise ValueError("weight must be [C, W]")
    if cu_seqlens is None:
        spans = [(b, 0, T) for b in range(B)]
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        if B != 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
            raise ValueError("cu_seqlens must be non-decreasing from 0 to T with B = 1")
        spans = [(0, int(cu[d]), int(cu[d + 1])) for d in range(len(cu) - 1)]
    y = np.zeros((B, T, C))
    for b, t0, t1 in spans:
        for t in range(t0, t1):
            for j in range(W):
                p = t - (W - 1) + j
                if p >= t0:
                    y[b, t] += w[:, j] * x[b, p]
    if activation == "silu":
        y = y / (1.0 + np.exp(-y))
    elif activation != "none":
        raise ValueError("activation must be 'none' or 'silu'")
    if norm_group:
        if C % norm_group:
            raise ValueError("norm_group must divide C")
        g = y.reshape(B, T, C // norm_group, norm_group)
        g = g / np.sqrt(np.sum(g * g, axis=-1, keepdims=True) + eps)
        y = g.reshape(B, T, C)
    return y
