"""Float64 gated per-head RMSNorm of the KDA output.

TEST INFRASTRUCTURE ONLY: part of the independent checker (see oracle/__init__.py for who may
import it). Plain NumPy in float64; shares no code with gated_delta_rule_144_b200.

Passages it follows:
- NeMo glm5_next layers, ``_TorchRMSNormGated.forward``: normalise
  [batch, sequence, heads, head_dim], then gate the result with a sigmoid of ``gate``.
- NeMo glm5_next layers, ``Glm5NextRMSNorm`` (its base): RMSNorm with the variance accumulated
  in fp32, and a weight of ``hidden_size`` entries initialised to ones.
- metrale glm5next_layer, decoder-layer invariants: every norm computes x * w / rms, never a
  1 + w scaling.

Reading (the formula is not printed): per (token, head), rms = sqrt(mean over head_dim of x^2 +
eps) and y = x / rms * w * sigmoid(gate), with w of head_dim entries shared by all heads and
gate of the same shape as x. Pinned in tests/test_oracle_out_norm.py.
"""

from __future__ import annotations

import numpy as np


def out_norm_gated(o, gate, weight, eps: float):
    """y = o / sqrt(mean(o^2 over the last axis) + eps) * weight * sigmoid(gate), in float64."""
    o = np.asarray(o, dtype=np.float64)
    g = np.asarray(gate, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + float(eps)) * w * (1.0 / (1.0 + np.exp(-g)))
