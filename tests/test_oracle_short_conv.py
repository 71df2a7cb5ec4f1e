"""Pins for the float64 short convolution of the inputs (oracle/short_conv.py).

Each check uses a fact the definition fixes: a hand-worked packed example, numpy's convolution on
one channel of one document, shifted-delta filters, packed documents equal to separate rows,
linearity, the SiLU at known points and unit group norms. The planted mistakes show that each
plausible slip fails at least one check: taps reversed, no reset at document boundaries, the
current token left out, the taps applied across channels instead of along time, a sigmoid instead
of a SiLU, the norm over the whole row, eps outside the root.
"""

import json
import os

import numpy as np
import pytest

from oracle.short_conv import short_conv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "short_conv_w3.json")


def check_hand_worked_example(f):
    d = json.load(open(GOLDEN))
    y = f(np.array(d["x"]), np.array(d["weight"]), np.array(d["cu_seqlens"]))
    return np.array_equal(y, np.array(d["y"]))


def check_numpy_convolution(f):
    # one channel, one document: y = (x * h)[:T] with h the taps in time order reversed
    rng = np.random.default_rng(5)
    x = rng.standard_normal(40)
    w = rng.standard_normal(4)
    y = f(x[None, :, None], w[None, :])
    return np.allclose(y[0, :, 0], np.convolve(x, w[::-1])[:40], rtol=1e-13, atol=1e-14)


def check_shifted_deltas(f):
    # taps e_{W-1-s}: y[t] = x[t - s], zero for the first s tokens of every document
    rng = np.random.default_rng(6)
    x = rng.standard_normal((1, 11, 3))
    cu = np.array([0, 4, 11])
    ok = True
    for s in range(4):
        w = np.zeros((3, 4))
        w[:, 3 - s] = 1.0
        y = f(x, w, cu)
        for a, b in ((0, 4), (4, 11)):
            ref = np.zeros((b - a, 3))
            ref[s:] = x[0, a:b - s] if b - a > s else ref[s:]
            ok &= np.array_equal(y[0, a:b], ref)
    return ok


def check_packed_equals_separate(f):
    rng = np.random.default_rng(7)
    lens = [5, 1, 0, 9, 3]
    x = rng.standard_normal((1, sum(lens), 6))
    w = rng.standard_normal((6, 4))
    cu = np.concatenate([[0], np.cumsum(lens)])
    y = f(x, w, cu, activation="silu", norm_group=3)
    ok = True
    for d in range(len(lens)):
        a, b = cu[d], cu[d + 1]
        if b > a:
            ok &= np.allclose(y[0, a:b], f(x[:, a:b], w, activation="silu", norm_group=3)[0],
                              rtol=0, atol=0)
    return ok


def check_linearity(f):
    rng = np.random.default_rng(8)
    x1, x2 = rng.standard_normal((2, 2, 7, 4))
    w = rng.standard_normal((4, 3))
    return np.allclose(f(2.5 * x1 - x2, w), 2.5 * f(x1, w) - f(x2, w), rtol=1e-13, atol=1e-13)


def check_silu_points(f):
    # one tap of weight 1: y = silu(x); silu(0) = 0, silu(ln 3) = ln 3 * 3/4, silu(-ln 3) = -ln 3/4
    x = np.array([[[0.0], [np.log(3.0)], [-np.log(3.0)]]])
    y = f(x, np.ones((1, 1)), activation="silu")
    return np.allclose(y[0, :, 0], [0.0, 0.75 * np.log(3.0), -0.25 * np.log(3.0)], rtol=1e-15,
                       atol=1e-16)


def check_group_norm(f):
    # eps = 0: every group of 4 channels has unit L2 norm, and its direction is kept
    rng = np.random.default_rng(9)
    x = rng.standard_normal((2, 6, 8)) * 3
    w = rng.standard_normal((8, 2))
    y = f(x, w, norm_group=4, eps=0.0)
    raw = f(x, w)
    n = np.sqrt(np.sum(y.reshape(2, 6, 2, 4) ** 2, axis=-1))
    ok = np.allclose(n, 1.0, rtol=1e-13, atol=0)
    cos = np.sum((y * raw).reshape(2, 6, 2, 4), -1) / np.linalg.norm(raw.reshape(2, 6, 2, 4), axis=-1)
    # eps enters under the root: a group with sum of squares 16 and eps 9 is scaled by 1/5
    z = f(np.array([[[4.0, 0.0]]]), np.ones((2, 1)), norm_group=2, eps=9.0)
    return ok and np.allclose(cos, 1.0, rtol=1e-13) and np.allclose(z, [[[0.8, 0.0]]], rtol=1e-15)


CHECKS = [check_hand_worked_example, check_numpy_convolution, check_shifted_deltas,
          check_packed_equals_separate, check_linearity, check_silu_points, check_group_norm]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__[6:])
def test_pin(check):
    assert check(short_conv)


def _mut(kind):
    def f(x, weight, cu_seqlens=None, activation="none", norm_group=0, eps=1e-6):
        x = np.asarray(x, dtype=np.float64)
        w = np.asarray(weight, dtype=np.float64)
        B, T, C = x.shape
        W = w.shape[1]
        spans = ([(b, 0, T) for b in range(B)] if cu_seqlens is None or kind == "no reset"
                 else [(0, int(cu_seqlens[d]), int(cu_seqlens[d + 1]))
                       for d in range(len(cu_seqlens) - 1)])
        y = np.zeros((B, T, C))
        for b, t0, t1 in spans:
            for t in range(t0, t1):
                for j in range(W):
                    jj = W - 1 - j if kind == "taps reversed" else j
                    p = t - (W - 1) + j - (1 if kind == "current token left out" else 0)
                    if p >= t0:
                        if kind == "taps across channels":
                            y[b, t] += w[:, jj] * np.roll(x[b, p], j)
                        else:
                            y[b, t] += w[:, jj] * x[b, p]
        if activation == "silu":
            y = 1.0 / (1.0 + np.exp(-y)) if kind == "sigmoid instead of silu" else y / (1 + np.exp(-y))
        if norm_group:
            gs = C if kind == "norm over the row" else norm_group
            g = y.reshape(B, T, C // gs, gs)
            den = (np.sqrt(np.sum(g * g, -1, keepdims=True)) + eps if kind == "eps outside the root"
                   else np.sqrt(np.sum(g * g, -1, keepdims=True) + eps))
            with np.errstate(invalid="ignore", divide="ignore"):   # a mutant may divide 0 by 0
                y = (g / den).reshape(B, T, C)
        return y
    return f


MUTANTS = ["taps reversed", "no reset", "current token left out", "taps across channels",
           "sigmoid instead of silu", "norm over the row", "eps outside the root"]


@pytest.mark.parametrize("name", MUTANTS)
def test_planted_mistake_fails_a_pin(name):
    f = _mut(name)
    failed = []
    for check in CHECKS:
        try:
            ok = bool(check(f))
        except Exception:
            ok = False
        if not ok:
            failed.append(check.__name__)
    assert failed, name
