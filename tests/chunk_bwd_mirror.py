"""The chunked backward's arithmetic in fp64 (NumPy): a mirror of the order
and factorisation the CUDA kernels use, checked against the oracle's autograd
gradients.  It is test infrastructure and never runs on the product path.

Forward, per 64-token chunk with start state S0 (Kimi K3 report digest,
section "KDA": per-channel decay with a floor, delta-rule write, sigmoid
output gate), in the chunk's own frame:
    lG_t = sum_{s <= t} max(g_s, floor)   (per channel),  lgam = lG_{C-1}
    Qbar = q e^{lG},  Kbar = k e^{lG},  Kbrev = k e^{-lG},  Khat = k e^{lgam - lG}
    A_qk = Qbar Kbrev^T (j <= i),  At = Kbar Kbrev^T (j < i),  A_kk = Diag(beta) At
    T = (I + A_kk)^-1,  Z = V - Kbar S0,  Y = Diag(beta) Z,  nu = T Y
    Oraw = scale (Qbar S0 + A_qk nu),  o = Oraw sigmoid(z),  S_C = e^{lgam} S0 + Khat^T nu
Every pair factor e^{lG_i - lG_j} (i >= j) is taken as
    a_i  m[b(i), b(j)]  bf_j,   a_i = e^{lG_i - r_b(i)},  bf_j = e^{r_b(j) - lG_j},
    m[bi, bj] = e^{r_bi - r_bj},   r_b = lG at the end of block b - 1 (r_0 = 0)
over 16-token blocks, so no factor leaves fp32's range (|floor| <= 5.45).

Backward (gradient dS_C of the chunk-end state, do of the outputs):
    go = do sigmoid(z),  dz = do Oraw sigmoid(z) (1 - sigmoid(z))
    dnu = scale A_qk^T go + Khat dS_C,  dY = T^T dnu,  dZ = Diag(beta) dY,  dv = dZ
    dT = dnu Y^T,  dA_kk = -T^T dT T^T (j < i),  dAt = Diag(beta) dA_kk
    dA_qk = scale go nu^T (j <= i)
    dS0 = scale Qbar^T go + e^{lgam} dS_C - Kbar^T dZ
The chain over chunks needs only dS0 from dS_C, which is affine:
    dZ = Et + Wt dS_C,   dS0 = F + e^{lgam} dS_C - Kbar^T dZ,
    Et = Diag(beta) T^T (scale A_qk^T go),  Wt = Diag(beta) T^T Khat,  F = scale Qbar^T go
(stage 1 forms Et, Wt, F, Kbar per chunk; stage 2 runs the chain; stage 3
forms every gradient of a chunk from its S0 and dS_C).  The key-side
gradients in the bounded form:
    dq  = a (eR scale go S0^T + sum_j dA_qk m bf k_j)
    dk1 = a (-eR dZ S0^T + sum_j dAt m bf k_j)                      (through Kbar)
    dk2 = bf (sum_i dA_qk m a q_i + sum_i dAt m a k_i + eG nu dS_C^T)  (through Kbrev, Khat)
    dk = dk1 + dk2,   dlG_t = q dq + k (dk1 - dk2)
    dlgam = e^{lgam} rowsum(dS_C o S0) + sum_t k_t dkh_t  (dkh = bf eG nu dS_C^T: the Khat part of dk2,
            i.e. rowsum(dS_C o S_C) written with the terms dlG holds, so that their
            cancellation inside sum_t is exact in the kernel's rounding as well)
    dg_s = [g_s >= floor] (sum_{t >= s} dlG_t + dlgam)
    dbeta = rowsum(dY o Z) + rowsum(dA_kk o At)
with eR[b] = e^{r_b} and eG[b] = e^{lgam - r_b}.
"""
from __future__ import annotations

import numpy as np

C = 64
BLK = 16


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _tables(g, floor):
    """Per-chunk decay tables from g [C, dk] (rows past the chunk's end are
    zero): lG, a, bf, m[4, 4, dk], eR[4, dk], eG[4, dk], lgam."""
    gc = np.maximum(g, floor)
    lG = np.cumsum(gc, axis=0)
    nb = C // BLK
    r = np.zeros((nb, g.shape[1]))
    for b in range(1, nb):
        r[b] = lG[BLK * b - 1]
    blk = np.arange(C) // BLK
    a = np.exp(lG - r[blk])
    bf = np.exp(r[blk] - lG)
    m = np.zeros((nb, nb, g.shape[1]))
    for bi in range(nb):
        for bj in range(bi + 1):
            m[bi, bj] = np.exp(r[bi] - r[bj])
    lgam = lG[C - 1]
    eR = np.exp(r)
    eG = np.exp(lgam[None, :] - r)
    return dict(lG=lG, a=a, bf=bf, m=m, eR=eR, eG=eG, lgam=lgam, blk=blk)


def _pair(M, x, tb, rows_out):
    """sum over the contraction index of M[i, j] m[b(i), b(j)] x[.] with the
    pair factor's middle term: rows_out = 'i' gives out[i] = sum_j M[i, j]
    m[bi, bj] x[j]; 'j' gives out[j] = sum_i M[i, j] m[bi, bj] x[i]."""
    m, blk = tb["m"], tb["blk"]
    out = np.zeros_like(x)
    for i in range(C):
        for j in range(i + 1):
            f = M[i, j] * m[blk[i], blk[j]]
            if rows_out == "i":
                out[i] += f * x[j]
            else:
                out[j] += f * x[i]
    return out


def _chunk_forward(q, k, v, beta, g, S0, scale, floor):
    tb = _tables(g, floor)
    a, bf, eR, eG, blk = tb["a"], tb["bf"], tb["eR"], tb["eG"], tb["blk"]
    qa, ka, kb = q * a, k * a, k * bf
    Aqk = np.zeros((C, C))
    At = np.zeros((C, C))
    for i in range(C):
        for j in range(i + 1):
            w = tb["m"][blk[i], blk[j]]
            Aqk[i, j] = np.sum(qa[i] * w * kb[j])
            if j < i:
                At[i, j] = np.sum(ka[i] * w * kb[j])
    Akk = beta[:, None] * At
    T = np.linalg.inv(np.eye(C) + Akk)
    Qbar, Kbar, Khat = qa * eR[blk], ka * eR[blk], kb * eG[blk]
    Z = v - Kbar @ S0
    Y = beta[:, None] * Z
    nu = T @ Y
    Oraw = scale * (Qbar @ S0 + Aqk @ nu)
    S_C = np.exp(tb["lgam"])[:, None] * S0 + Khat.T @ nu
    return dict(tb=tb, qa=qa, ka=ka, kb=kb, Aqk=Aqk, At=At, T=T, Qbar=Qbar, Kbar=Kbar, Khat=Khat,
                Z=Z, Y=Y, nu=nu, Oraw=Oraw, S_C=S_C)


def _pad(x, L):
    out = np.zeros((C,) + x.shape[1:])
    out[:L] = x
    return out


def head_backward(q, k, v, g, beta, do, gate, S0, dS_T, scale, floor):
    """Gradients of one (sequence, head): q, k, g [L, dk], v, do, gate [L, dv]
    (gate may be None), beta [L], S0 / dS_T [dk, dv] (may be None).  Returns
    dq, dk, dv, dg, dbeta, dgate (or None), dS0, and the forward's o."""
    L, dk = q.shape
    dv = v.shape[1]
    nch = (L + C - 1) // C
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, np.float64)
    chunks = []
    o = np.zeros((L, dv))
    for c in range(nch):
        t0, Lc = c * C, min(C, L - c * C)
        sl = slice(t0, t0 + Lc)
        ch = dict(t0=t0, Lc=Lc, q=_pad(q[sl], Lc), k=_pad(k[sl], Lc), v=_pad(v[sl], Lc),
                  g=_pad(g[sl], Lc), beta=_pad(beta[sl], Lc), do=_pad(do[sl], Lc),
                  gate=None if gate is None else _pad(gate[sl], Lc), S0=S)
        f = _chunk_forward(ch["q"], ch["k"], ch["v"], ch["beta"], ch["g"], S, scale, floor)
        ch.update(f)
        sg = np.ones((C, dv)) if gate is None else _sig(ch["gate"])
        o[sl] = (f["Oraw"] * sg)[:Lc]
        S = f["S_C"]
        chunks.append(ch)

    # stage 1: the chain's per-chunk constants
    for ch in chunks:
        sg = np.ones((C, dv)) if ch["gate"] is None else _sig(ch["gate"])
        go = ch["do"] * sg
        E = scale * ch["Aqk"].T @ go
        ch["Et"] = ch["beta"][:, None] * (ch["T"].T @ E)
        ch["Wt"] = ch["beta"][:, None] * (ch["T"].T @ ch["Khat"])
        ch["F"] = scale * ch["Qbar"].T @ go
    # stage 2: the chain, last chunk first
    dS = np.zeros((dk, dv)) if dS_T is None else np.array(dS_T, np.float64)
    for ch in reversed(chunks):
        ch["dS_C"] = dS
        dZ = ch["Et"] + ch["Wt"] @ dS
        dS = ch["F"] + np.exp(ch["tb"]["lgam"])[:, None] * dS - ch["Kbar"].T @ dZ
    dS0 = dS

    # stage 3: every chunk's gradients
    out = {n: np.zeros((L, d)) for n, d in (("dq", dk), ("dk", dk), ("dv", dv), ("dg", dk), ("dgate", dv))}
    out["dbeta"] = np.zeros(L)
    for ch in chunks:
        tb = ch["tb"]
        a, bf, eR, eG, blk = tb["a"], tb["bf"], tb["eR"], tb["eG"], tb["blk"]
        S0c, dSC, beta_c = ch["S0"], ch["dS_C"], ch["beta"]
        sg = np.ones((C, dv)) if ch["gate"] is None else _sig(ch["gate"])
        go = ch["do"] * sg
        dgate = ch["do"] * ch["Oraw"] * sg * (1.0 - sg)
        dnu = scale * ch["Aqk"].T @ go + ch["Khat"] @ dSC
        dY = ch["T"].T @ dnu
        dZ = beta_c[:, None] * dY
        dT = dnu @ ch["Y"].T
        dAkk = np.tril(-ch["T"].T @ dT @ ch["T"].T, -1)
        dAt = beta_c[:, None] * dAkk
        dAqk = np.tril(scale * go @ ch["nu"].T)
        acc_q = eR[blk] * (scale * go @ S0c.T) + _pair(dAqk, ch["kb"], tb, "i")
        acc_k1 = -eR[blk] * (dZ @ S0c.T) + _pair(dAt, ch["kb"], tb, "i")
        dkh = bf * (eG[blk] * (ch["nu"] @ dSC.T))
        dk2 = bf * (_pair(dAqk, ch["qa"], tb, "j") + _pair(dAt, ch["ka"], tb, "j")) + dkh
        dq = a * acc_q
        dk1 = a * acc_k1
        dlG = ch["q"] * dq + ch["k"] * (dk1 - dk2)
        # d/dlgam of S_C = e^{lgam} S0 + Khat^T nu, with the Khat part taken from dkh itself
        dlgam = np.exp(tb["lgam"]) * np.sum(dSC * S0c, axis=1) + np.sum(ch["k"] * dkh, axis=0)
        dgc = np.cumsum(dlG[::-1], axis=0)[::-1] + dlgam[None, :]
        dg = np.where(ch["g"] >= floor, dgc, 0.0)
        dbeta = np.sum(dY * ch["Z"], axis=1) + np.sum(dAkk * ch["At"], axis=1)
        sl, Lc = slice(ch["t0"], ch["t0"] + ch["Lc"]), ch["Lc"]
        out["dq"][sl] = dq[:Lc]
        out["dk"][sl] = (dk1 + dk2)[:Lc]
        out["dv"][sl] = dZ[:Lc]
        out["dg"][sl] = dg[:Lc]
        out["dbeta"][sl] = dbeta[:Lc]
        out["dgate"][sl] = dgate[:Lc]
    if gate is None:
        out["dgate"] = None
    out["dS0"] = dS0
    out["o"] = o
    return out
