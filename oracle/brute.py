"""Brute-force, loop-free evaluation of the KDA recurrence for tiny inputs (T <= 8).

TEST INFRASTRUCTURE ONLY: used to pin the float64 oracle, never by the product.

The per-token steps of the GLM-5.3-Flash model card's Kimi Delta Attention snippet
(decay, read k^T S, delta = beta (v - k^T S), rank-one write) compose to one affine map per token:

    S_t = A_t S_{t-1} + beta_t k_t v_t^T,      A_t = (I - beta_t k_t k_t^T) diag(g_t),

so the state after t tokens is the unrolled sum

    S_t = (A_t ... A_1) S_0 + sum_{s <= t} (A_t ... A_{s+1}) beta_s k_s v_s^T,

and the read-out is o_t = S_t^T q_t. This module evaluates that sum with explicit dk x dk
matrices and no state loop, so that a mistake in the oracle's loop (an index, a transposed
operand, the order of decay, read and write) shows up as a disagreement.
"""

from __future__ import annotations

import numpy as np


def transition(k_t, log_g_t, beta_t):
    """A_t = (I - beta k k^T) diag(exp(log_g)) as a dense float64 matrix."""
    k_t = np.asarray(k_t, dtype=np.float64)
    dk = k_t.shape[0]
    return (np.eye(dk) - float(beta_t) * np.outer(k_t, k_t)) @ np.diag(
        np.exp(np.asarray(log_g_t, dtype=np.float64)))


def kda_unrolled(q, k, v, log_g, beta, S0):
    """One (sequence, head): q, k, log_g [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv].

    Returns (o [T, dv], S_T [dk, dv]) from the unrolled sum, every prefix evaluated afresh.
    """
    q, k, v, log_g, beta, S0 = (np.asarray(x, dtype=np.float64)
                                for x in (q, k, v, log_g, beta, S0))
    T, dk = q.shape
    if T > 8:
        raise ValueError("brute force is for T <= 8")
    A = [transition(k[t], log_g[t], beta[t]) for t in range(T)]

    def prod(hi, lo):
        """A_hi ... A_lo (identity when hi < lo), indices 0-based and inclusive."""
        M = np.eye(dk)
        for s in range(lo, hi + 1):
            M = A[s] @ M
        return M

    o = np.zeros((T, v.shape[1]))
    S_t = S0
    for t in range(T):
        S_t = prod(t, 0) @ S0 + sum(
            (prod(t, s + 1) @ (beta[s] * np.outer(k[s], v[s])) for s in range(t + 1)),
            np.zeros_like(S0))
        o[t] = S_t.T @ q[t]
    return o, S_t
