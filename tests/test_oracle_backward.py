"""Pins for the float64 gradients of the KDA recurrence (oracle/backward.py).

The gradients are checked against facts that do not go through their own formulas:
- central finite differences of the loop-free, brute-force forward (oracle/brute.py), element by
  element on a tiny case;
- PyTorch float64 autograd of the forward recurrence written as plain tensor operations;
- the adjoint identity: o and the final state are jointly linear in (v, h0), so
  <do, o> + <dhT, hT> = <dv, v> + <dh0, h0> with o, hT from the C++ forward oracle;
- a closed form at beta = 0, g = 1 (the state stays h0);
- packed documents equal separate runs.
The planted mistakes below (a dropped term, a sign, a wrong operand, a missing decay, the final-
state gradient ignored) each fail at least one of them.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle.backward import kda_bwd
from oracle.brute import kda_unrolled


def _case(rng, B=1, T=5, H=1, dk=3, dv=2, N=None, f32=False):
    N = B if N is None else N
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    c = dict(q=rng.standard_normal((B, T, H, dk)) * 0.7, k=k,
             v=rng.standard_normal((B, T, H, dv)),
             log_g=-np.logaddexp(0.0, rng.standard_normal((B, T, H, dk))),
             beta=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))),
             h0=rng.standard_normal((N, H, dk, dv)) * 0.5,
             do=rng.standard_normal((B, T, H, dv)), dhT=rng.standard_normal((N, H, dk, dv)))
    if f32:   # values the float32-input forward oracle takes exactly
        c = {n: x.astype(np.float32).astype(np.float64) for n, x in c.items()}
    return c


NAMES = ("q", "k", "v", "log_g", "beta", "h0")


def _grads(bwd, c, cu=None):
    return dict(zip(NAMES, bwd(c["q"], c["k"], c["v"], c["log_g"], c["beta"], c["do"],
                               dhT=c["dhT"], h0=c["h0"], cu_seqlens=cu)))


def check_finite_differences(bwd):
    rng = np.random.default_rng(5)
    c = _case(rng)
    g = _grads(bwd, c)

    def loss(x):
        o, S = kda_unrolled(x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0],
                            x["log_g"][0, :, 0], x["beta"][0, :, 0], x["h0"][0, 0])
        return float((x["do"][0, :, 0] * o).sum() + (x["dhT"][0, 0] * S).sum())

    h = 1e-6
    for name in NAMES:
        for idx in np.ndindex(c[name].shape):
            xp = {n: a.copy() for n, a in c.items()}
            xm = {n: a.copy() for n, a in c.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            fd = (loss(xp) - loss(xm)) / (2 * h)
            if abs(fd - g[name][idx]) > 1e-7 * max(1.0, abs(fd)):
                return False
    return True


def _torch_forward(c, cu=None):
    """The forward recurrence as plain float64 torch operations (differentiated by autograd)."""
    t = {n: torch.tensor(c[n], dtype=torch.float64, requires_grad=n in NAMES) for n in c}
    B, T, H, dk = c["q"].shape
    spans = [(n, 0, T) for n in range(B)] if cu is None else \
        [(0, int(cu[d]), int(cu[d + 1])) for d in range(len(cu) - 1)]
    loss = torch.zeros((), dtype=torch.float64)
    for doc, (row, t0, t1) in enumerate(spans):
        for h in range(H):
            S = t["h0"][doc, h]
            for s in range(t0, t1):
                S = torch.exp(t["log_g"][row, s, h])[:, None] * S
                d = t["beta"][row, s, h] * (t["v"][row, s, h] - S.T @ t["k"][row, s, h])
                S = S + torch.outer(t["k"][row, s, h], d)
                loss = loss + (t["do"][row, s, h] * (S.T @ t["q"][row, s, h])).sum()
            loss = loss + (t["dhT"][doc, h] * S).sum()
    loss.backward()
    return {n: t[n].grad.numpy() for n in NAMES}


def check_autograd(bwd):
    rng = np.random.default_rng(6)
    c = _case(rng, B=2, T=7, H=2, dk=4, dv=3)
    g, ref = _grads(bwd, c), _torch_forward(c)
    ok = all(np.allclose(g[n], ref[n], rtol=1e-11, atol=1e-12) for n in NAMES)
    cp = _case(rng, B=1, T=9, H=2, dk=4, dv=3, N=3)   # packed: lengths 4, 0, 5
    cu = np.array([0, 4, 4, 9])
    g, ref = _grads(bwd, cp, cu), _torch_forward(cp, cu)
    return ok and all(np.allclose(g[n], ref[n], rtol=1e-11, atol=1e-12) for n in NAMES)


def check_adjoint_identity(bwd):
    rng = np.random.default_rng(7)
    c = _case(rng, B=2, T=11, H=3, dk=8, dv=5, f32=True)
    o, hT = oracle.kda_fwd(c["q"], c["k"], c["v"], c["log_g"], c["beta"], h0=c["h0"])
    g = _grads(bwd, c)
    lhs = (c["do"] * o).sum() + (c["dhT"] * hT).sum()
    rhs = (g["v"] * c["v"]).sum() + (g["h0"] * c["h0"]).sum()
    return abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def check_beta_zero_closed_form(bwd):
    # beta = 0 and g = 1: S_t = h0 for every t, o_t = h0^T q_t. With dS_t = dhT + sum_{s>=t}
    # q_s do_s^T: dq_t = h0 do_t, dk = dv = 0, dh0 = dS_1, dbeta_t = <dS_t^T k_t, v_t - h0^T k_t>,
    # dlog_g_t = rowsum(dS_t * h0).
    rng = np.random.default_rng(8)
    c = _case(rng, T=6, dk=4, dv=3)
    c["beta"][:] = 0.0
    c["log_g"][:] = 0.0
    g = _grads(bwd, c)
    q, k, v, do = (c[n][0, :, 0] for n in ("q", "k", "v", "do"))
    h0, dhT = c["h0"][0, 0], c["dhT"][0, 0]
    outer = np.einsum("tc,tj->tcj", q, do)
    dS = dhT + np.cumsum(outer[::-1], axis=0)[::-1]        # dS_t for t = 1..T
    want = dict(q=do @ h0.T, k=np.zeros_like(q), v=np.zeros_like(v),
                log_g=np.einsum("tcj,cj->tc", dS, h0),
                beta=np.einsum("tcj,tc,tj->t", dS, k, v - k @ h0), h0=dS[0])
    return all(np.allclose(g[n][0, :, 0] if n != "h0" else g[n][0, 0], want[n], rtol=1e-12,
                           atol=1e-13) for n in NAMES)


def check_packed_equals_separate(bwd):
    rng = np.random.default_rng(9)
    c = _case(rng, B=1, T=10, H=2, dk=4, dv=3, N=2)
    cu = np.array([0, 6, 10])
    g = _grads(bwd, c, cu)
    for d, (t0, t1) in enumerate([(0, 6), (6, 10)]):
        sub = {n: c[n][:, t0:t1] for n in ("q", "k", "v", "log_g", "beta", "do")}
        sub["h0"], sub["dhT"] = c["h0"][d:d + 1], c["dhT"][d:d + 1]
        gs = _grads(bwd, sub)
        for n in NAMES:
            got = g[n][d:d + 1] if n == "h0" else g[n][:, t0:t1]
            if not np.array_equal(got, gs[n]):
                return False
    return True


CHECKS = [check_finite_differences, check_autograd, check_adjoint_identity,
          check_beta_zero_closed_form, check_packed_equals_separate]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__[6:])
def test_pin(check):
    assert check(kda_bwd)


MUTANTS = {
    "read-out term of dk dropped": lambda *a, **kw: kda_bwd(*a, **kw, mutant=1),
    "sign of dm": lambda *a, **kw: kda_bwd(*a, **kw, mutant=2),
    "v + m in dbeta": lambda *a, **kw: kda_bwd(*a, **kw, mutant=3),
    "decayed state in dlog_g": lambda *a, **kw: kda_bwd(*a, **kw, mutant=4),
    "state gradient not decayed": lambda *a, **kw: kda_bwd(*a, **kw, mutant=5),
    "final-state gradient ignored": lambda *a, **kw: kda_bwd(*a, **{**kw, "dhT": None}),
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
