"""NumPy model of the gradients of the chunked form: the algebra a chunked backward kernel follows.

Test infrastructure and a design aid, like chunk_model.py for the forward: float64 throughout, it
is checked against the pinned gradient oracle (oracle/backward.py) in
tests/test_chunk_bwd_model.py, where it must agree to rounding. It shares nothing with the CUDA
sources.

Forward per chunk of L <= C tokens (one head), with Gamma the within-chunk inclusive cumulative
log decay, K+ = k e^Gamma, K- = k e^-Gamma, Q+ = q e^Gamma, K_end = k e^(Gamma_end - Gamma):
  A_kk = strict_lower(K+ K-^T),  A_qk = lower(Q+ K-^T),  M = (I + diag(beta) A_kk)^-1,
  T = M diag(beta),  W = T K+,  U~ = T V,  Q~ = Q+ - A_qk W,  O~ = A_qk U~,
  U = U~ - W S,  o = O~ + Q~ S,  S_next = diag(e^Gamma_end) S + K_end^T U.
Backward, chunks from the last (dS: gradient of S_next; S: the chunk's starting state, kept by
the forward):
  state part   dU = K_end dS;  dK_end = U dS^T;  d(e^Gamma_end) = rowsum(dS * S);
               dS <- diag(e^Gamma_end) dS + Q~^T do - W^T dU   (passed to the previous chunk);
               dQ~ = do S^T;  dO~ = do;  dU~ = dU;  dW = -dU S^T
  intra part   dQ+ = dQ~;  dA_qk = -dQ~ W^T + dO~ U~^T;  dW -= A_qk^T dQ~;  dU~ += A_qk^T dO~;
               dT = dW K+^T + dU~ V^T;  dK+ = T^T dW;  dV = T^T dU~;
               dbeta = diag(M^T dT) + rowsum(dX * A_kk) with dX = -M^T (dT diag(beta)) M^T;
               dA_kk = strict_lower(diag(beta) dX);  dA_qk = lower(dA_qk);
               dK+ += dA_kk K-;  dK- = dA_kk^T K+ + dA_qk^T Q+;  dQ+ += dA_qk K-;
               then through the exponentials to dk, dq and dGamma, and dlog_g as the reverse
               cumulative sum of dGamma plus the gradient of Gamma_end.
The explicit inverse and the unanchored e^-Gamma are fine in float64 at the test's sizes; a
kernel would use the UT structure and anchored factors as the forward does.
"""

from __future__ import annotations

import numpy as np


def _chain(q, k, v, lg, b, h0, do, dhT, C):
    T = q.shape[0]
    chunks = []
    S = h0.copy()
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        qc, kc, vc, lc, bc = q[sl], k[sl], v[sl], lg[sl], b[sl]
        L = qc.shape[0]
        G = np.cumsum(lc, axis=0)
        Ge = G[-1]
        eG, emG, eE = np.exp(G), np.exp(-G), np.exp(Ge[None, :] - G)
        Kp, Km, Qp, Ke = kc * eG, kc * emG, qc * eG, kc * eE
        dec = np.exp(Ge)
        Akk = np.tril(Kp @ Km.T, -1)
        Aqk = np.tril(Qp @ Km.T, 0)
        M = np.linalg.inv(np.eye(L) + bc[:, None] * Akk)
        Tm = M * bc[None, :]
        W, Ut = Tm @ Kp, Tm @ vc
        Qt, Ot = Qp - Aqk @ W, Aqk @ Ut
        U = Ut - W @ S
        chunks.append(dict(sl=sl, S=S, G=G, eG=eG, emG=emG, eE=eE, Kp=Kp, Km=Km, Qp=Qp, Ke=Ke,
                           dec=dec, Akk=Akk, Aqk=Aqk, M=M, Tm=Tm, W=W, Ut=Ut, Qt=Qt, U=U, b=bc,
                           v=vc))
        S = dec[:, None] * S + Ke.T @ U
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dlg, db = np.zeros_like(lg), np.zeros_like(b)
    dS = np.zeros_like(h0) if dhT is None else dhT.copy()
    for ch in reversed(chunks):
        sl, S0 = ch["sl"], ch["S"]
        doc = do[sl]
        # state part
        dU = ch["Ke"] @ dS
        dKe = ch["U"] @ dS.T
        ddec = (dS * S0).sum(axis=1)
        dS_prev = ch["dec"][:, None] * dS + ch["Qt"].T @ doc - ch["W"].T @ dU
        dQt, dOt, dUt, dW = doc @ S0.T, doc, dU.copy(), -dU @ S0.T
        # intra part
        Aqk, Akk, M, Tm, bc = ch["Aqk"], ch["Akk"], ch["M"], ch["Tm"], ch["b"]
        dQp = dQt.copy()
        dAqk = -dQt @ ch["W"].T + dOt @ ch["Ut"].T
        dW = dW - Aqk.T @ dQt
        dUt = dUt + Aqk.T @ dOt
        dT = dW @ ch["Kp"].T + dUt @ ch["v"].T
        dKp = Tm.T @ dW
        dv[sl] = Tm.T @ dUt
        dX = -M.T @ (dT * bc[None, :]) @ M.T
        db[sl] = np.einsum("ij,ij->j", M, dT) + (dX * Akk).sum(axis=1)
        dAkk = np.tril(bc[:, None] * dX, -1)
        dAqk = np.tril(dAqk, 0)
        dKp = dKp + dAkk @ ch["Km"]
        dKm = dAkk.T @ ch["Kp"] + dAqk.T @ ch["Qp"]
        dQp = dQp + dAqk @ ch["Km"]
        dk[sl] = dKp * ch["eG"] + dKm * ch["emG"] + dKe * ch["eE"]
        dq[sl] = dQp * ch["eG"]
        dG = dKp * ch["Kp"] - dKm * ch["Km"] + dQp * ch["Qp"] - dKe * ch["Ke"]
        dGe = (dKe * ch["Ke"]).sum(axis=0) + ddec * ch["dec"]
        dlg[sl] = np.cumsum(dG[::-1], axis=0)[::-1] + dGe[None, :]
        dS = dS_prev
    return dq, dk, dv, dlg, db, dS


def chunked_bwd(q, k, v, log_g, beta, do, dhT=None, h0=None, C=64):
    """Gradients of the chunked form for B equal-length sequences: the same outputs as
    oracle.backward.kda_bwd (q, k, log_g [B, T, H, dk]; v, do [B, T, H, dv]; beta [B, T, H];
    h0, dhT [B, H, dk, dv] or None)."""
    f = lambda x: np.asarray(x, dtype=np.float64)
    q, k, v, log_g, beta, do = (f(x) for x in (q, k, v, log_g, beta, do))
    B, T, H, dk = q.shape
    dv_ = v.shape[-1]
    h0 = np.zeros((B, H, dk, dv_)) if h0 is None else f(h0)
    dhT = None if dhT is None else f(dhT)
    out = [np.zeros_like(x) for x in (q, k, v, log_g, beta)] + [np.zeros((B, H, dk, dv_))]
    for n in range(B):
        for h in range(H):
            sl = (n, slice(None), h)
            r = _chain(q[sl], k[sl], v[sl], log_g[sl], beta[sl], h0[n, h], do[sl],
                       None if dhT is None else dhT[n, h], C)
            for dst, src in zip(out[:5], r[:5]):
                dst[sl] = src
            out[5][n, h] = r[5]
    return tuple(out)
