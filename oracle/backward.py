"""Float64 gradients of the KDA recurrence (the training direction).

TEST INFRASTRUCTURE ONLY: part of the independent checker (see oracle/__init__.py for who may
import it). Plain NumPy in float64; shares no code with gated_delta_rule_144_b200.

Passage it follows: NeMo AutoModel glm5_next layers page, ``_torch_recurrent_kda`` -- a
differentiable reference KDA (its gradients are what training back-propagates through; FLA owns
the GPU training kernel). The forward is the per-token recurrence of the GLM-5.3-Flash model
card's Kimi Delta Attention snippet, per (sequence or document, head), with g_t = exp(log_g_t):

    S'_t = diag(g_t) S_{t-1}
    m_t  = S'_t^T k_t
    d_t  = beta_t (v_t - m_t)
    S_t  = S'_t + k_t d_t^T
    o_t  = S_t^T q_t

starting from h0 (or zero) and restarting at every packed-document boundary. Given the upstream
gradients do (of o) and dhT (of the final states), the gradients of the scalar
L = sum_t <do_t, o_t> + <dhT, S_T> are the plain reverse-mode derivative of those five lines,
taken one token at a time from the last to the first (the forward states are recomputed and
kept):

    dS    += q_t do_t^T                     dq_t   = S_t do_t
    dk_t  += dS d_t                         dd     = dS^T k_t
    dbeta_t = <dd, v_t - m_t>               dv_t   = beta_t dd        dm = -beta_t dd
    dk_t  += S'_t dm                        dS'    = dS + k_t dm^T
    dlog_g_t = g_t * rowsum(dS' * S_{t-1})  dS     = diag(g_t) dS'    (becomes dS_{t-1})

and dh0 = dS after the first token. Pinned in tests/test_oracle_backward.py against central
finite differences of the forward oracle, PyTorch float64 autograd of the forward recurrence,
the adjoint identity of the part linear in (v, h0), and a closed form at beta = 0, g = 1.
"""

from __future__ import annotations

import numpy as np


def _chain(q, k, v, lg, b, h0, do, dhT, mutant=0):
    """One (sequence or document, head) chain: q, k, lg [T, dk]; v, do [T, dv]; b [T];
    h0, dhT [dk, dv] (dhT may be None). Returns dq, dk, dv, dlg, db, dh0."""
    T, dk = q.shape
    dv = v.shape[1]
    g = np.exp(lg)
    S = h0.copy()
    prev, dec, mem, dlt, post = [], [], [], [], []
    for t in range(T):
        prev.append(S)
        Sp = g[t][:, None] * S
        m = Sp.T @ k[t]
        d = b[t] * (v[t] - m)
        S = Sp + np.outer(k[t], d)
        dec.append(Sp)
        mem.append(m)
        dlt.append(d)
        post.append(S)
    dq = np.zeros((T, dk))
    dkk = np.zeros((T, dk))
    dvv = np.zeros((T, dv))
    dlg = np.zeros((T, dk))
    db = np.zeros(T)
    dS = np.zeros((dk, dv)) if dhT is None else dhT.copy()
    for t in range(T - 1, -1, -1):
        dq[t] = post[t] @ do[t]
        dS = dS + np.outer(q[t], do[t])
        dkk[t] = dS @ dlt[t]
        dd = dS.T @ k[t]
        db[t] = dd @ ((v[t] + mem[t]) if mutant == 3 else (v[t] - mem[t]))
        dvv[t] = b[t] * dd
        dm = (b[t] * dd) if mutant == 2 else (-b[t] * dd)
        if mutant != 1:
            dkk[t] += dec[t] @ dm
        dSp = dS + np.outer(k[t], dm)
        dlg[t] = (dSp * (dec[t] if mutant == 4 else prev[t])).sum(axis=1) * g[t]
        dS = dSp if mutant == 5 else g[t][:, None] * dSp
    return dq, dkk, dvv, dlg, db, dS


def kda_bwd(q, k, v, log_g, beta, do, dhT=None, h0=None, cu_seqlens=None, mutant: int = 0):
    """Gradients of L = sum <do, o> + <dhT, hT> for the forward of oracle.kda_fwd.

    q, k, log_g: [B, T, H, dk]; v, do: [B, T, H, dv]; beta: [B, T, H]; h0, dhT:
    [N, H, dk, dv] or None; cu_seqlens: int [N + 1] or None (then N = B). Values are taken as
    float64. Returns (dq, dk, dv, dlog_g, dbeta, dh0) with the shapes of (q, k, v, log_g, beta,
    h0). ``mutant`` > 0 plants one mistake, for the pin tests only.
    """
    f = lambda x: np.asarray(x, dtype=np.float64)
    q, k, v, log_g, beta, do = (f(x) for x in (q, k, v, log_g, beta, do))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        N = B
        spans = [(n, 0, T) for n in range(B)]
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        if B != 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
            raise ValueError("cu_seqlens must be non-decreasing from 0 to T with B = 1")
        N = len(cu) - 1
        spans = [(0, int(cu[d]), int(cu[d + 1])) for d in range(N)]
    h0 = np.zeros((N, H, dk, dv)) if h0 is None else f(h0)
    dhT = None if dhT is None else f(dhT)
    out = [np.zeros_like(x) for x in (q, k, v, log_g, beta)] + [np.zeros((N, H, dk, dv))]
    for doc, (row, t0, t1) in enumerate(spans):
        for h in range(H):
            sl = (row, slice(t0, t1), h)
            r = _chain(q[sl], k[sl], v[sl], log_g[sl], beta[sl], h0[doc, h], do[sl],
                       None if dhT is None else dhT[doc, h], mutant)
            for dst, src in zip(out[:5], r[:5]):
                dst[sl] = src
            out[5][doc, h] = r[5]
    return tuple(out)
