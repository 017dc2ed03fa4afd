"""Independent fp64 numpy restatement of the chunkwise (WY) algorithm, used only as a pin.

It is written from "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention", review page
section "Chunkwise Parallel Training via WY Representation":
  Step 1  G_r = sum_{i<=r} g_i inside the chunk, gamma = exp(G), kbar = k / gamma, ebar = gamma*b*k
  Step 2  T = tril(Ebar Kbar^T, -1), A = (I + T)^-1, Y = A Ebar, U = A Z, Z = W * V   (Eq. 20)
  Step 3  S_C = Diag(gamma_C) S_0 + K_tail^T (U - Y S_0),  O = Q_gamma S_0 + A_qk (U - Y S_0)
          K_tail[r] = (gamma_C / gamma_r) * k_r, Q_gamma[r] = gamma_r * q_r,
          (A_qk)_rs = 1[r >= s] q_r^T Diag(gamma_r / gamma_s) k_s          (Eqs. 23-24)
and, for the backward, from section "Gate-Aware Backward Pass" (Eqs. 64-65: dA = dU Z^T + dY Ebar^T;
dT = -tril(A^T dA A^T, -1); dEbar += dT Kbar, dKbar += dT^T Ebar; dB = dEbar*gamma*K, dW = dZ*V,
dV = dZ*W with dZ = A^T dU; dg by a reverse cumulative sum inside the chunk). The output/state
vector-Jacobian products that the page only names are the chain rule applied to Step 3.

It is deliberately plain: per chain, per chunk, dense numpy matrices, a true matrix inverse.

relative=True restates the same algebra with the decay factors of the T and A_qk products taken relative
to each channel's mid-chunk log-decay m = G_C / 2 (Q' = q e^{G-m}, K' = k e^{m-G}, E' = b k e^{G-m}, whose
products equal those of Q_gamma, Kbar, Ebar; Y = A E' e^{m}), and the backward with the matching scaled
accumulators (dQ' = dQ_gamma e^{m}, dE' = dEbar e^{m}, dK' = dKbar e^{-m}, dY' = dY e^{m}). No factor then
exceeds e^{|G_C| / 2}, which keeps fp32 arithmetic finite where the absolute factors e^{+-G} overflow.
"""
from __future__ import annotations

import numpy as np


def _chunk_terms_relative(q, k, v, la, b, w):
    G = np.cumsum(la, axis=0)
    m = 0.5 * G[-1]
    ep, en = np.exp(G - m), np.exp(m - G)
    gam = np.exp(G)
    gC = gam[-1]
    Kp = k * en
    Ep = b * k * ep
    Qp = q * ep
    Z = w * v
    Kt = k * np.exp(G[-1] - G)
    n = q.shape[0]
    A = np.linalg.inv(np.eye(n, dtype=q.dtype) + np.tril(Ep @ Kp.T, -1))
    Aqk = np.tril(Qp @ Kp.T)
    Y = (A @ Ep) * np.exp(m)[None, :]
    U = A @ Z
    return dict(gam=gam, gC=gC, m=m, ep=ep, en=en, Kp=Kp, Ep=Ep, Qp=Qp, Z=Z, Qg=q * gam, Kt=Kt, A=A, Aqk=Aqk,
                Y=Y, U=U)


def _chunk_terms(q, k, v, la, b, w):
    G = np.cumsum(la, axis=0)
    gam = np.exp(G)
    gC = gam[-1]
    Kb = k / gam
    Eb = b * k * gam
    Z = w * v
    Qg = q * gam
    Kt = k * (gC / gam)
    n = q.shape[0]
    Tm = np.tril(Eb @ Kb.T, -1)
    A = np.linalg.inv(np.eye(n) + Tm)
    Aqk = np.tril(Qg @ Kb.T)
    Y = A @ Eb
    U = A @ Z
    return dict(gam=gam, gC=gC, Kb=Kb, Eb=Eb, Z=Z, Qg=Qg, Kt=Kt, A=A, Aqk=Aqk, Y=Y, U=U)


def chunk_fwd(q, k, v, la, b, w, S0, C=64, relative=False):
    """One chain: q,k,la,b [T,dk]; v,w [T,dv]; S0 [dk,dv]. Returns o [T,dv], S_T, chunk states."""
    T = q.shape[0]
    S = S0.copy()
    o = np.zeros_like(v)
    states = []
    terms = _chunk_terms_relative if relative else _chunk_terms
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        m = terms(q[sl], k[sl], v[sl], la[sl], b[sl], w[sl])
        states.append(S.copy())
        R = m["U"] - m["Y"] @ S
        o[sl] = m["Qg"] @ S + m["Aqk"] @ R
        S = m["gC"][:, None] * S + m["Kt"].T @ R
    return o, S, states


def chunk_bwd(q, k, v, la, b, w, S0, dO, dST, C=64, relative=False):
    """One chain. Returns dq, dk, dv, dla, db, dw, dS0."""
    if relative:
        return _chunk_bwd_relative(q, k, v, la, b, w, S0, dO, dST, C)
    T = q.shape[0]
    _, _, states = chunk_fwd(q, k, v, la, b, w, S0, C)
    out = {n: np.zeros_like(q) for n in ("dq", "dk", "dla", "db")}
    out.update({n: np.zeros_like(v) for n in ("dv", "dw")})
    dS = dST.copy()
    starts = list(range(0, T, C))
    for ci in reversed(range(len(starts))):
        c0 = starts[ci]
        sl = slice(c0, min(c0 + C, T))
        m = _chunk_terms(q[sl], k[sl], v[sl], la[sl], b[sl], w[sl])
        S0c = states[ci]
        gam, gC, Kb, Eb, Z, Qg, Kt, A, Aqk, Y, U = (m[x] for x in
                                                    ("gam", "gC", "Kb", "Eb", "Z", "Qg", "Kt", "A", "Aqk", "Y", "U"))
        R = U - Y @ S0c
        dOc = dO[sl]
        # state/output VJP (chain rule on S_C and O)
        dR = Aqk.T @ dOc + Kt @ dS
        dS0c = gC[:, None] * dS + Qg.T @ dOc - Y.T @ dR
        dQg = dOc @ S0c.T
        dAqk = np.tril(dOc @ R.T)
        dKt = R @ dS.T
        dgC = np.sum(dS * S0c, axis=1)
        dU = dR
        dY = -dR @ S0c.T
        dQg = dQg + dAqk @ Kb
        dKb = dAqk.T @ Qg
        # gate-aware WY VJP (Eqs. 64-65)
        dA = dU @ Z.T + dY @ Eb.T
        dZ = A.T @ dU
        dEb = A.T @ dY
        dT = -np.tril(A.T @ dA @ A.T, -1)
        dEb = dEb + dT @ Kb
        dKb = dKb + dT.T @ Eb
        # elementwise gradients
        kk, bb, vv, ww, qq = k[sl], b[sl], v[sl], w[sl], q[sl]
        out["dw"][sl] = dZ * vv
        out["dv"][sl] = dZ * ww
        out["db"][sl] = dEb * kk * gam
        out["dk"][sl] = dEb * bb * gam + dKb / gam + dKt * (gC / gam)
        out["dq"][sl] = dQg * gam
        dG = dQg * Qg + dEb * Eb - dKb * Kb - dKt * Kt
        dG[-1] += np.sum(dKt * Kt, axis=0) + dgC * gC
        out["dla"][sl] = np.cumsum(dG[::-1], axis=0)[::-1]
        dS = dS0c
    out["dS0"] = dS
    return out


def _chunk_bwd_relative(q, k, v, la, b, w, S0, dO, dST, C):
    T = q.shape[0]
    _, _, states = chunk_fwd(q, k, v, la, b, w, S0, C, relative=True)
    out = {n: np.zeros_like(q) for n in ("dq", "dk", "dla", "db")}
    out.update({n: np.zeros_like(v) for n in ("dv", "dw")})
    dS = dST.copy()
    starts = list(range(0, T, C))
    for ci in reversed(range(len(starts))):
        c0 = starts[ci]
        sl = slice(c0, min(c0 + C, T))
        t = _chunk_terms_relative(q[sl], k[sl], v[sl], la[sl], b[sl], w[sl])
        S0c = states[ci]
        em = np.exp(t["m"])[None, :]
        R = t["U"] - t["Y"] @ S0c
        dOc = dO[sl]
        dR = t["Aqk"].T @ dOc + t["Kt"] @ dS
        dS0c = t["gC"][:, None] * dS + t["Qg"].T @ dOc - t["Y"].T @ dR
        dAqk = np.tril(dOc @ R.T)
        dKt = R @ dS.T
        dgC = np.sum(dS * S0c, axis=1)
        dYp = -(dR @ S0c.T) * em                                  # dY' = dY e^{m}
        dQp = (dOc @ S0c.T) * em + dAqk @ t["Kp"]                 # dQ' = dQ_gamma e^{m}
        dA = dR @ t["Z"].T + dYp @ t["Ep"].T                      # = dU Z^T + dY Ebar^T
        dZ = t["A"].T @ dR
        dT = -np.tril(t["A"].T @ dA @ t["A"].T, -1)
        dEp = t["A"].T @ dYp + dT @ t["Kp"]                       # dE' = dEbar e^{m}
        dKp = dAqk.T @ t["Qp"] + dT.T @ t["Ep"]                   # dK' = dKbar e^{-m}
        kk, bb, vv, ww = k[sl], b[sl], v[sl], w[sl]
        ep, en = t["ep"], t["en"]
        G = np.cumsum(la[sl], axis=0)
        gt = np.exp(G[-1] - G)                                    # gamma_C / gamma
        out["dw"][sl] = dZ * vv
        out["dv"][sl] = dZ * ww
        out["db"][sl] = dEp * kk * ep
        out["dk"][sl] = dEp * bb * ep + dKp * en + dKt * gt
        out["dq"][sl] = dQp * ep
        dG = dQp * t["Qp"] + dEp * t["Ep"] - dKp * t["Kp"] - dKt * t["Kt"]
        dG[-1] += np.sum(dKt * t["Kt"], axis=0) + dgC * t["gC"]
        out["dla"][sl] = np.cumsum(dG[::-1], axis=0)[::-1]
        dS = dS0c
    out["dS0"] = dS
    return out

