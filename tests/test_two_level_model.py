"""The algebra of the two-level state pass, in float64 on the chunk model (tests/chunk_model.py),
against the pinned per-token oracle.

The chunked state pass maps each chunk's initial state to its final state affinely:
S -> (diag(e^{Gamma_end}) - K_end^T W) S + K_end^T U~. A segment of chunks therefore maps
S -> A S + B. A is the segment run from S = I with the values taken as 0, which makes U~ = 0;
B is the segment run from S = 0. The two-level pass does three things:
- it runs segment 0 from h0;
- it chains the initial states S_{p+1} = A_p S_p + B_p;
- it runs every other segment from its initial state.

The result must be the recurrence: the o and final state of the oracle, to float64 rounding, for
any segment count (segments of ceil(chunks / P) chunks, the last one partial).
"""

import numpy as np
import pytest

import oracle
from chunk_model import C, chunk_forward


def _inputs(T, d, mu, seed, beta_scale=1.0):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((T, d))).astype(np.float32)
    k = unit(rng.standard_normal((T, d))).astype(np.float32)
    v = rng.standard_normal((T, d)).astype(np.float32)
    lg = (-np.logaddexp(0.0, rng.standard_normal((T, d)) + mu)).astype(np.float32)
    beta = (beta_scale / (1.0 + np.exp(-rng.standard_normal(T)))).astype(np.float32)
    h0 = (rng.standard_normal((d, d)) * 0.5).astype(np.float32)
    return q, k, v, lg, beta, h0


def two_level(q, k, v, lg, beta, h0, P):
    """o and the final state by the two-level pass with P segments."""
    T, d = q.shape
    nc = -(-T // C)
    m = -(-nc // P)
    bounds = [min(T, C * m * p) for p in range(-(-nc // m) + 1)]
    seg = lambda x, p: x[bounds[p]:bounds[p + 1]]
    zeros_v = np.zeros_like(v)
    # segment 0 from h0; the maps of the inner segments
    _, S = chunk_forward(seg(q, 0), seg(k, 0), seg(v, 0), seg(lg, 0), seg(beta, 0), h0)
    states = [np.asarray(h0, dtype=np.float64), S]
    for p in range(1, len(bounds) - 2):
        args = (seg(q, p), seg(k, p))
        _, A = chunk_forward(*args, seg(zeros_v, p), seg(lg, p), seg(beta, p), np.eye(d))
        _, B = chunk_forward(*args, seg(v, p), seg(lg, p), seg(beta, p), np.zeros((d, d)))
        states.append(A @ states[-1] + B)
    # every segment from its initial state
    o = np.zeros((T, v.shape[1]))
    for p in range(len(bounds) - 1):
        o_p, S = chunk_forward(seg(q, p), seg(k, p), seg(v, p), seg(lg, p), seg(beta, p),
                               states[p])
        o[bounds[p]:bounds[p + 1]] = o_p
    return o, S, len(bounds) - 1


@pytest.mark.parametrize("P", [3, 4, 8])
@pytest.mark.parametrize("mu,beta_scale", [(0.0, 1.0), (-5.0, 1.0), (-5.0, 0.05)])
def test_two_level_pass_equals_the_oracle(P, mu, beta_scale):
    """8 chunks, the last partial (T = 7 x 64 + 19), d = 16, h0 given; fast gates, slow gates,
    and slow gates with weak writes (the state, and so every segment map, persists)."""
    T, d = 7 * C + 19, 16
    q, k, v, lg, beta, h0 = _inputs(T, d, mu, 60 + P, beta_scale)
    o, S, segs = two_level(q, k, v, lg, beta, h0, P)
    assert segs == P
    o_ref, h_ref = oracle.kda_fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                                  lg[None, :, None], beta[None, :, None], h0=h0[None, None])
    eo = np.linalg.norm(o - o_ref[0, :, 0]) / np.linalg.norm(o_ref[0, :, 0])
    eh = np.linalg.norm(S - h_ref[0, 0]) / np.linalg.norm(h_ref[0, 0])
    assert eo < 1e-11 and eh < 1e-11, (eo, eh)


def test_segment_map_without_writes_is_the_decay_product():
    """beta = 0: W = U~ = 0, so a segment's map is A = diag(prod of its decays) and B = 0, and
    the chain carries h0 by the decays alone (the oracle pin beta = 0 => S_T = diag(prod g) S_0)."""
    T, d = 3 * C + 5, 16
    q, k, v, lg, beta, h0 = _inputs(T, d, -2.0, 70)
    beta[:] = 0.0
    _, A = chunk_forward(q, k, np.zeros_like(v), lg, beta, np.eye(d))
    _, B = chunk_forward(q, k, v, lg, beta, np.zeros((d, d)))
    decay = np.exp(lg.astype(np.float64).sum(axis=0))
    assert np.allclose(A, np.diag(decay), rtol=1e-12, atol=1e-300)
    assert np.abs(B).max() == 0.0
    o, S, _ = two_level(q, k, v, lg, beta, h0, 3)
    assert np.allclose(S, decay[:, None] * h0, rtol=1e-12, atol=0)


def test_a_wrong_map_is_caught():
    """The check has teeth: the segment map A S + B reproduces the segment run from S, while
    dropping B, or applying A twice, does not (slow gates and weak writes, so both terms
    matter)."""
    T, d = 7 * C + 19, 16
    q, k, v, lg, beta, h0 = _inputs(T, d, -5.0, 71, 0.05)
    nc = -(-T // C)
    m = -(-nc // 4)
    b1, b2 = C * m, min(T, 2 * C * m)
    sl = lambda x: x[b1:b2]
    _, S1 = chunk_forward(q[:b1], k[:b1], v[:b1], lg[:b1], beta[:b1], h0)
    _, A = chunk_forward(sl(q), sl(k), np.zeros_like(sl(v)), sl(lg), sl(beta), np.eye(d))
    _, B = chunk_forward(sl(q), sl(k), sl(v), sl(lg), sl(beta), np.zeros((d, d)))
    _, S2 = chunk_forward(sl(q), sl(k), sl(v), sl(lg), sl(beta), S1)
    assert np.allclose(A @ S1 + B, S2, rtol=1e-11, atol=1e-14)
    assert not np.allclose(A @ S1, S2, rtol=1e-3)
    assert not np.allclose(A @ (A @ S1) + B, S2, rtol=1e-3)
