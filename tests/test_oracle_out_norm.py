"""Pins for the float64 gated per-head RMSNorm (oracle/out_norm.py).

Each check uses a fact the definition fixes (a hand-worked value, a closed form, an identity of
the sigmoid gate, independence of heads and channels), and the planted mistakes below show that
every plausible slip fails at least one of them: the mean taken over the wrong axis, eps outside
the square root, a (1 + w) weight, a SiLU instead of a sigmoid gate, the gate dropped, the root
of the sum instead of the mean.
"""

import json
import os

import numpy as np
import pytest

from oracle.out_norm import out_norm_gated

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "out_norm_gated_d2.json")


def check_hand_worked_example(f):
    d = json.load(open(GOLDEN))
    y = f(np.array(d["x"]), np.array(d["gate"]), np.array(d["weight"]), d["eps"])
    return np.allclose(y, d["y"], rtol=1e-14, atol=0)


def check_constant_rows_closed_form(f):
    # x = 3 everywhere, eps = 7: rms = sqrt(9 + 7) = 4; gate 0 -> 1/2; y = 3/4 * w / 2
    x = np.full((2, 5, 3, 8), 3.0)
    w = np.linspace(0.5, 2.0, 8)
    y = f(x, np.zeros_like(x), w, 7.0)
    return np.allclose(y, np.broadcast_to(0.375 * w, x.shape), rtol=1e-15, atol=0)


def check_unit_mean_square(f):
    # w = 1, eps = 0, gate saturated: every (token, head) row of y has mean square 1
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 4, 2, 16)) * rng.uniform(0.1, 10, (3, 4, 2, 1))
    y = f(x, np.full_like(x, 60.0), np.ones(16), 0.0)
    return np.allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-12, atol=0)


def check_sigmoid_gate_identity(f):
    # sigmoid(g) + sigmoid(-g) = 1, so y(g) + y(-g) is the ungated normalised row x * w / rms
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 3, 4, 8))
    g = rng.standard_normal(x.shape) * 3
    w = rng.uniform(0.5, 1.5, 8)
    eps = 1e-3
    ungated = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * w
    return np.allclose(f(x, g, w, eps) + f(x, -g, w, eps), ungated, rtol=1e-12, atol=1e-15)


def check_heads_and_channels_independent(f):
    # permuting heads permutes the output; the weight scales its own channel only
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 3, 5, 8))
    g = rng.standard_normal(x.shape)
    w = rng.uniform(0.5, 1.5, 8)
    perm = [3, 0, 4, 1, 2]
    ok = np.allclose(f(x, g, w, 1e-5)[:, :, perm], f(x[:, :, perm], g[:, :, perm], w, 1e-5),
                     rtol=1e-14, atol=0)
    e = np.zeros(8)
    e[5] = 2.0
    y = f(x, g, e, 1e-5)
    return ok and np.all(y[..., :5] == 0) and np.all(y[..., 6:] == 0) and np.all(y[..., 5] != 0)


CHECKS = [check_hand_worked_example, check_constant_rows_closed_form, check_unit_mean_square,
          check_sigmoid_gate_identity, check_heads_and_channels_independent]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__[6:])
def test_pin(check):
    assert check(out_norm_gated)


def _sig(g):
    return 1.0 / (1.0 + np.exp(-g))


MUTANTS = {
    "mean over heads": lambda o, g, w, e: o / np.sqrt(np.mean(o * o, axis=-2, keepdims=True) + e)
    * w * _sig(g),
    "eps outside the root": lambda o, g, w, e: o / (np.sqrt(np.mean(o * o, -1, keepdims=True)) + e)
    * w * _sig(g),
    "1 + w scaling": lambda o, g, w, e: o / np.sqrt(np.mean(o * o, -1, keepdims=True) + e)
    * (1 + w) * _sig(g),
    "silu gate": lambda o, g, w, e: o / np.sqrt(np.mean(o * o, -1, keepdims=True) + e)
    * w * g * _sig(g),
    "gate dropped": lambda o, g, w, e: o / np.sqrt(np.mean(o * o, -1, keepdims=True) + e) * w,
    "root of the sum": lambda o, g, w, e: o / np.sqrt(np.sum(o * o, -1, keepdims=True) + e)
    * w * _sig(g),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    f = MUTANTS[name]
    failed = []
    for check in CHECKS:
        try:
            ok = bool(check(f))
        except Exception:
            ok = False
        if not ok:
            failed.append(check.__name__)
    assert failed, name
