"""NumPy model of the chunked prefill exactly as libkda's tcgen05 kernel organises it.

Test infrastructure: it checks the kernel's algebra against the oracle in float64 (where it must
agree to rounding), and, with bf16=True, rounds every tensor-core operand to bf16 where the
kernel does, to predict the kernel's error. It shares nothing with the CUDA sources.

Per chunk of C = 64 tokens (rows r) and one head, with a_t = exp(log_g_t) per key channel,
16-token blocks b and the within-chunk cumulative log decay Gamma:

  A_kk[r, i] = sum_c k_rc k_ic exp(Gamma_rc - Gamma_ic)  (i < r),  A_qk the same with q_r (i <= r)

are formed as one product R C^T of separable factors that never exceed the float32 range:
  - rows of R: x_r * exp(Gamma_r - Gamma_m(b(r))), m(b) = the middle of block b (after row 7)
  - diagonal-block columns of C: k_i * exp(Gamma_m(b(i)) - Gamma_i)
  - columns for a later row block a > b(i): k_i * exp(Gamma_m(a) - Gamma_i)  (<= 1)
Then T = (I + diag(beta) A_kk)^-1 diag(beta), W = T K+, U~ = T V with K+ = k exp(Gamma),
Q~ = Q+ - A_qk W, O~ = A_qk U~, and the state pass
  U = U~ - W S,  O = O~ + Q~ S,  S <- diag(exp(Gamma_end)) S + K_end^T U,
K_end = k exp(Gamma_end - Gamma).
"""

from __future__ import annotations

import numpy as np

C = 64
BLK = 16


def bf16(x):
    """Round to bfloat16 (round to nearest even), returned as float64."""
    x32 = np.asarray(x, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def tf32(x):
    """Round toward zero to tf32 (10 explicit mantissa bits), returned as float64."""
    x32 = np.asarray(x, dtype=np.float32)
    u = x32.view(np.uint32) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


def _factors(a):
    """Per-block products for one chunk. a: [64, d] decay factors. Returns a dict of arrays."""
    d = a.shape[1]
    ppre = np.empty_like(a)   # inclusive prefix product within the block
    sig = np.empty_like(a)    # exclusive suffix product to the block end
    rho = np.empty_like(a)    # exp(Gamma_r - Gamma_m(b))
    kap = np.empty_like(a)    # exp(Gamma_m(b) - Gamma_r)
    Lo = np.empty((4, d))
    Up = np.empty((4, d))
    for b in range(4):
        blk = a[b * BLK:(b + 1) * BLK]
        p = np.cumprod(blk, axis=0)
        ppre[b * BLK:(b + 1) * BLK] = p
        s = np.ones_like(blk)
        for lr in range(BLK - 2, -1, -1):
            s[lr] = s[lr + 1] * blk[lr + 1]
        sig[b * BLK:(b + 1) * BLK] = s
        Lo[b] = p[7]
        Up[b] = np.prod(blk[8:], axis=0)
        for lr in range(BLK):
            r = b * BLK + lr
            if lr >= 8:
                pfx = np.prod(blk[8:lr + 1], axis=0)
                rho[r] = pfx
                kap[r] = 1.0 / pfx
            else:
                sfx = np.prod(blk[lr + 1:8], axis=0)
                rho[r] = 1.0 / sfx
                kap[r] = sfx
    P = Lo * Up
    return dict(ppre=ppre, sig=sig, rho=rho, kap=kap, Lo=Lo, Up=Up, P=P)


def cross_factor(f, a_blk, b_blk):
    """exp(Gamma_m(a) - Gamma_end(b)) per channel for row block a > column block b."""
    P, Lo = f["P"], f["Lo"]
    x = Lo[a_blk].copy()
    for bb in range(b_blk + 1, a_blk):
        x = x * P[bb]
    return x


CROSS_OFF = {1: 0, 2: 16, 3: 48}   # row offset of row block a's cross columns inside C[64:]


def chunk_step(q, k, v, lg, beta, S, L, bf=False, only=None):
    """One chunk (rows >= L are padding). q, k, lg: [64, dk]; v: [64, dv]; beta: [64]."""
    ident = lambda x: np.asarray(x, dtype=np.float64)
    def R_(name):
        if not bf:
            return ident
        if isinstance(only, dict):
            return {"bf16": bf16, "tf32": tf32, "f32": ident}[only.get(name, "bf16")]
        if only is None or name in only:
            return bf16
        return ident
    q = q.copy(); k = k.copy(); lg = lg.copy(); beta = beta.copy()
    k[L:] = 0.0
    lg[L:] = 0.0
    beta[L:] = 0.0
    a = np.exp(lg)
    f = _factors(a)
    R = np.concatenate([k * f["rho"], q * f["rho"]], axis=0)          # [128, dk]
    Cm = np.zeros((160, k.shape[1]))
    Cm[:64] = k * f["kap"]
    for a_blk in (1, 2, 3):
        for b_blk in range(a_blk):
            rows = slice(b_blk * BLK, (b_blk + 1) * BLK)
            dst = 64 + CROSS_OFF[a_blk] + b_blk * BLK
            Cm[dst:dst + BLK] = k[rows] * f["sig"][rows] * cross_factor(f, a_blk, b_blk)
    D = (bf16(R) @ bf16(Cm).T) if only == "stacked" else R_("RC")(R) @ R_("RC")(Cm).T                                              # [128, 160] fp32 acc
    Akk = np.zeros((64, 64))
    Aqk = np.zeros((64, 64))
    for r in range(64):
        ab = r // BLK
        for i in range(r + 1):
            bb = i // BLK
            if bb == ab:
                col = i
            else:
                col = 64 + CROSS_OFF[ab] + i
            if i < r:
                Akk[r, i] = D[r, col]
            Aqk[r, i] = D[64 + r, col]
    Lm = beta[:, None] * Akk
    M = np.linalg.inv(np.eye(64) + Lm)                                 # fp32 solve in the kernel
    Tm = M * beta[None, :]
    P = f["P"]
    F = np.ones((4, k.shape[1]))
    G = np.ones((4, k.shape[1]))
    for b in range(1, 4):
        F[b] = F[b - 1] * P[b - 1]
    for b in range(2, -1, -1):
        G[b] = G[b + 1] * P[b + 1]
    blk_of = np.arange(64) // BLK
    eG = F[blk_of] * f["ppre"]
    Kp = k * eG
    Qp = q * eG
    Kend = k * f["sig"] * G[blk_of]
    decay = F[3] * P[3]
    if only is not None and not isinstance(only, (set, dict)) and only == "stacked":
        # the kernel's association: T' = A_qk T (bf16 operands, rounded to bf16), then
        # [W; A_qk W] = [T; T'] K+ and [U~; O~] = [T; T'] V in one product
        Tb = bf16(Tm)
        Tp = bf16(bf16(Aqk) @ Tb)
        W = Tb @ bf16(Kp)
        Ut = Tb @ v
        Wb = bf16(W)
        Qt = bf16(Qp) - Tp @ bf16(Kp)
        Ot = Tp @ v
        Sb = bf16(S)
        U = Ut - Wb @ Sb
        O = Ot + bf16(Qt) @ Sb
        S = decay[:, None] * S + bf16(Kend).T @ bf16(U)
        return O[:L], S
    W = R_("T")(Tm) @ R_("Kp")(Kp)
    Ut = R_("T")(Tm) @ v
    Wb = R_("W")(W)
    Qt = R_("Qp")(Qp) - R_("Aqk")(Aqk) @ Wb
    Ot = R_("Aqk")(Aqk) @ R_("Utb")(Ut)
    Sb = R_("S")(S)
    U = Ut - Wb @ Sb
    O = Ot + R_("Qt")(Qt) @ Sb
    S = decay[:, None] * S + R_("Kend")(Kend).T @ R_("U")(U)
    return O[:L], S


def chunk_forward(q, k, v, lg, beta, S0, bf=False, only=None):
    """One (sequence, head): q, k, lg [T, dk]; v [T, dv]; beta [T]; S0 [dk, dv]."""
    T = q.shape[0]
    dv = v.shape[1]
    S = np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        L = min(C, T - c0)
        pad = lambda x: np.concatenate([x[c0:c0 + L], np.zeros((C - L,) + x.shape[1:])], 0)
        O, S = chunk_step(pad(q), pad(k), pad(v), pad(lg), pad(beta), S, L, bf=bf, only=only)
        o[c0:c0 + L] = O
    return o, S
