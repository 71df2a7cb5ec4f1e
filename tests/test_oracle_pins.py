"""Pins for the float64 oracle: checks against facts the recurrence fixes, not against itself.

Each test is chosen so that a plausible mistake in the oracle (decaying the value axis instead of
the key axis, reading out before the write, a dropped beta, a transposed write, state leaking
across documents) fails at least one of them. See tests/test_oracle_mutants.py for the planted
mistakes that demonstrate it.
"""

import json
import os

import numpy as np
import pytest

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, B, T, H, dk, dv, h0=True, decay_scale=1.0):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    log_g = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk)))) * decay_scale
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.5 * rng.standard_normal((B, H, dk, dv)) if h0 else None
    f = lambda x: None if x is None else x.astype(np.float32)
    return tuple(map(f, (q, k, v, log_g, beta, S0)))


def check_unrolled_brute_force(orc, seed=0, T=8, dk=6, dv=5):
    rng = np.random.default_rng(seed)
    B, H = 2, 2
    q, k, v, lg, b, S0 = _rand_case(rng, B, T, H, dk, dv)
    o, hT = orc.kda_fwd(q, k, v, lg, b, h0=S0)
    for n in range(B):
        for h in range(H):
            ob, Sb = brute.kda_unrolled(q[n, :, h], k[n, :, h], v[n, :, h], lg[n, :, h],
                                        b[n, :, h], S0[n, h])
            np.testing.assert_allclose(o[n, :, h], ob, rtol=0, atol=1e-12)
            np.testing.assert_allclose(hT[n, h], Sb, rtol=0, atol=1e-12)


def check_hand_worked_example(orc):
    with open(os.path.join(GOLDEN, "kda_hand_d2_t2.json")) as fh:
        gold = json.load(fh)
    g = np.array(gold["g"])
    q = np.array(gold["q"])[None, :, None, :]
    k = np.array(gold["k"])[None, :, None, :]
    v = np.array(gold["v"])[None, :, None, :]
    lg = np.log(g)[None, :, None, :]
    beta = np.array(gold["beta"])[None, :, None]
    S0 = np.array(gold["S0"])[None, None]
    o, hT = orc.kda_fwd(q, k, v, lg, beta, h0=S0)
    # inputs pass through float32 (0.6, 0.8, ln 0.5 are not exact there): 1e-6 absolute
    np.testing.assert_allclose(o[0, :, 0], np.array(gold["o"]), rtol=0, atol=1e-6)
    np.testing.assert_allclose(hT[0, 0], np.array(gold["ST"]), rtol=0, atol=1e-6)
    assert np.abs(o[0, :, 0] - np.array(gold["o_if_read_before_write"])).max() > 0.1
    # the unrolled form reproduces the hand values too
    ob, Sb = brute.kda_unrolled(q[0, :, 0], k[0, :, 0], v[0, :, 0], lg[0, :, 0], beta[0, :, 0],
                                S0[0, 0])
    np.testing.assert_allclose(ob, np.array(gold["o"]), rtol=0, atol=1e-6)
    np.testing.assert_allclose(Sb, np.array(gold["ST"]), rtol=0, atol=1e-6)


def check_beta_zero_is_pure_decay(orc):
    """beta = 0: S_T = diag(prod_t g_t) S_0 and o_t = S_0^T diag(prod_{s<=t} g_s) q_t."""
    rng = np.random.default_rng(7)
    B, T, H, dk, dv = 1, 40, 3, 6, 5
    q, k, v, lg, b, S0 = _rand_case(rng, B, T, H, dk, dv)
    b = np.zeros_like(b)
    o, hT = orc.kda_fwd(q, k, v, lg, b, h0=S0)
    cum = np.cumsum(lg.astype(np.float64), axis=1)          # [B, T, H, dk]
    for h in range(H):
        np.testing.assert_allclose(hT[0, h], np.exp(cum[0, -1, h])[:, None] * S0[0, h],
                                   rtol=1e-12, atol=1e-14)
        for t in range(T):
            ref = S0[0, h].astype(np.float64).T @ (np.exp(cum[0, t, h]) * q[0, t, h])
            np.testing.assert_allclose(o[0, t, h], ref, rtol=1e-11, atol=1e-13)


def check_exact_recall_with_orthonormal_keys(orc, T=5, dk=8):
    """g = 1, beta = 1, S_0 = 0 and orthonormal keys: k_i^T S_T = v_i for every i."""
    rng = np.random.default_rng(T * 100 + dk)
    dv = 7
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T.astype(np.float32)[None, :, None, :]    # rows are orthonormal keys
    v = rng.standard_normal((1, T, 1, dv)).astype(np.float32)
    q = rng.standard_normal((1, T, 1, dk)).astype(np.float32)
    lg = np.zeros((1, T, 1, dk), np.float32)
    b = np.ones((1, T, 1), np.float32)
    o, hT = orc.kda_fwd(q, k, v, lg, b)
    kf = k[0, :, 0].astype(np.float64)
    # float32 keys are orthonormal to ~1e-7
    np.testing.assert_allclose(kf @ hT[0, 0], v[0, :, 0], rtol=0, atol=5e-6)
    # and the read-out with q = k_i right after writing i returns v_i
    o2, _ = orc.kda_fwd(k, k, v, lg, b)
    np.testing.assert_allclose(o2[0, :, 0], v[0, :, 0], rtol=0, atol=5e-6)


def check_linearity_in_values_and_initial_state(orc):
    rng = np.random.default_rng(11)
    q, k, v, lg, b, S0 = _rand_case(rng, 2, 9, 2, 5, 4)
    # dyadic values so that the float32 sums below are exact
    dy = lambda x: (np.round(x * 1024) / 1024).astype(np.float32)
    v, S0 = dy(v), dy(S0)
    o1, h1 = orc.kda_fwd(q, k, v, lg, b, h0=S0)
    o2, h2 = orc.kda_fwd(q, k, 2 * v, lg, b, h0=2 * S0)
    np.testing.assert_allclose(o2, 2 * o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h2, 2 * h1, rtol=1e-12, atol=1e-13)
    _, _, v2, _, _, S02 = _rand_case(np.random.default_rng(12), 2, 9, 2, 5, 4)
    v2, S02 = dy(v2), dy(S02)
    o3, h3 = orc.kda_fwd(q, k, v2, lg, b, h0=S02)
    o4, h4 = orc.kda_fwd(q, k, v + v2, lg, b, h0=S0 + S02)
    np.testing.assert_allclose(o4, o1 + o3, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(h4, h1 + h3, rtol=1e-10, atol=1e-12)


def check_value_columns_evolve_independently(orc):
    rng = np.random.default_rng(13)
    q, k, v, lg, b, S0 = _rand_case(rng, 1, 12, 2, 6, 5)
    perm = np.array([3, 0, 4, 1, 2])
    o1, h1 = orc.kda_fwd(q, k, v, lg, b, h0=S0)
    o2, h2 = orc.kda_fwd(q, k, v[..., perm], lg, b, h0=S0[..., perm])
    np.testing.assert_allclose(o2, o1[..., perm], rtol=0, atol=1e-13)
    np.testing.assert_allclose(h2, h1[..., perm], rtol=0, atol=1e-13)


def check_packed_documents_equal_separate_runs(orc):
    rng = np.random.default_rng(17)
    lengths = [5, 0, 1, 9, 3]
    T = sum(lengths)
    H, dk, dv = 2, 4, 3
    q, k, v, lg, b, _ = _rand_case(rng, 1, T, H, dk, dv, h0=False)
    S0 = (0.5 * rng.standard_normal((len(lengths), H, dk, dv))).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    o, hT = orc.kda_fwd(q, k, v, lg, b, h0=S0, cu_seqlens=cu)
    for n, L in enumerate(lengths):
        s = slice(cu[n], cu[n + 1])
        if L == 0:
            np.testing.assert_array_equal(hT[n], S0[n].astype(np.float64))
            continue
        for h in range(H):
            if L <= 8:
                ob, Sb = brute.kda_unrolled(q[0, s, h], k[0, s, h], v[0, s, h], lg[0, s, h],
                                            b[0, s, h], S0[n, h])
                np.testing.assert_allclose(o[0, s, h], ob, rtol=0, atol=1e-12)
                np.testing.assert_allclose(hT[n, h], Sb, rtol=0, atol=1e-12)
        o1, h1 = orc.kda_fwd(q[:, s], k[:, s], v[:, s], lg[:, s], b[:, s], h0=S0[n:n + 1])
        np.testing.assert_array_equal(o[:, s], o1)
        np.testing.assert_array_equal(hT[n], h1[0])


def check_batched_rows_equal_separate_runs(orc):
    rng = np.random.default_rng(19)
    q, k, v, lg, b, S0 = _rand_case(rng, 3, 6, 2, 4, 3)
    o, hT = orc.kda_fwd(q, k, v, lg, b, h0=S0)
    for n in range(3):
        o1, h1 = orc.kda_fwd(q[n:n + 1], k[n:n + 1], v[n:n + 1], lg[n:n + 1], b[n:n + 1],
                                h0=S0[n:n + 1])
        np.testing.assert_array_equal(o[n:n + 1], o1)
        np.testing.assert_array_equal(hT[n:n + 1], h1)


def check_decode_equals_one_token_prefill_and_brute_force(orc):
    rng = np.random.default_rng(23)
    N, H, dk, dv = 3, 2, 5, 4
    q, k, v, lg, b, S = _rand_case(rng, N, 1, H, dk, dv)
    o_d, S_new = orc.kda_decode(q[:, 0], k[:, 0], v[:, 0], lg[:, 0], b[:, 0], S)
    o_p, hT = orc.kda_fwd(q, k, v, lg, b, h0=S)
    np.testing.assert_array_equal(o_d, o_p[:, 0])
    np.testing.assert_array_equal(S_new, hT)
    for n in range(N):
        for h in range(H):
            ob, Sb = brute.kda_unrolled(q[n, :, h], k[n, :, h], v[n, :, h], lg[n, :, h],
                                        b[n, :, h], S[n, h])
            np.testing.assert_allclose(o_d[n, h], ob[0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(S_new[n, h], Sb, rtol=0, atol=1e-12)


def check_decode_iterated_equals_prefill(orc):
    rng = np.random.default_rng(29)
    T, H, dk, dv = 7, 2, 4, 3
    q, k, v, lg, b, S0 = _rand_case(rng, 1, T, H, dk, dv)
    o_p, hT = orc.kda_fwd(q, k, v, lg, b, h0=S0)
    S = S0.astype(np.float64)
    for t in range(T):
        o_d, S = orc.kda_decode(q[:, t], k[:, t], v[:, t], lg[:, t], b[:, t], S)
        # the decode state passes through float32 between calls
        np.testing.assert_allclose(o_d, o_p[:, t], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(S, hT, rtol=1e-5, atol=1e-6)


def check_malformed_cu_seqlens_rejected(orc):
    rng = np.random.default_rng(31)
    q, k, v, lg, b, _ = _rand_case(rng, 1, 6, 1, 2, 2, h0=False)
    for cu in ([0, 4, 3, 6], [0, 2, 5], [1, 3, 6]):
        with pytest.raises(ValueError):
            orc.kda_fwd(q, k, v, lg, b, cu_seqlens=np.array(cu, np.int32))


CHECKS = [
    check_unrolled_brute_force,
    check_hand_worked_example,
    check_beta_zero_is_pure_decay,
    check_exact_recall_with_orthonormal_keys,
    check_linearity_in_values_and_initial_state,
    check_value_columns_evolve_independently,
    check_packed_documents_equal_separate_runs,
    check_batched_rows_equal_separate_runs,
    check_decode_equals_one_token_prefill_and_brute_force,
    check_decode_iterated_equals_prefill,
    check_malformed_cu_seqlens_rejected,
]


@pytest.mark.parametrize("seed,T,dk,dv", [(0, 1, 3, 2), (1, 5, 4, 3), (2, 8, 6, 5), (3, 8, 5, 7)])
def test_oracle_matches_unrolled_brute_force(seed, T, dk, dv):
    check_unrolled_brute_force(oracle.default(), seed, T, dk, dv)


@pytest.mark.parametrize("T,dk", [(4, 4), (5, 8), (16, 16)])
def test_exact_recall_with_orthonormal_keys(T, dk):
    check_exact_recall_with_orthonormal_keys(oracle.default(), T, dk)


@pytest.mark.parametrize("check", [c for c in CHECKS if c not in (
    check_unrolled_brute_force, check_exact_recall_with_orthonormal_keys)],
    ids=lambda c: c.__name__[len("check_"):])
def test_pin(check):
    check(oracle.default())
