"""NumPy model of the chunked (WY / UT-transform) algorithm the CUDA kernels
run, used on the CPU to check the factorisation against the oracle before and
independently of any kernel.  Test-side only; neither the oracle nor the
product imports it.

Per chunk of C tokens (C a multiple of 16; a ragged tail is zero-padded,
which is exact: g = 0, beta = 0, k = 0 make a padded token the identity):

  G     = inclusive cumulative sum of max(g, floor) inside the chunk
  r_b   = G at the last token before 16-token block b (0 for b = 0); r_nb = G_{C-1}
  Gt_i  = exp(G_i - r_{b(i)})             in [e^{16 floor}, 1]
  Kbar_j= k_j exp(r_{b(j)} - G_j)          <= e^{-16 floor} |k_j|
  D[b,b'] = exp(r_b - r_b')  (b >= b')     <= 1
  K^(b)_j = Kbar_j * D[b, b(j)]   for j in blocks <= b  (= k_j exp(r_b - G_j))

  A_qk[i,j] = sum_c q_ic Gt_ic K^(b(i))_jc           j <= i
  A_kk[i,j] = beta_i sum_c k_ic Gt_ic K^(b(i))_jc    j <  i
  T = (I + A_kk)^-1   (16x16 diagonal blocks by substitution, then block merges)
  W = T (beta * k * Gt * D[b(i),0]),   U = T (beta * v)
  per chunk, with the carried state S:
     Vn = U - W S                        (form "wy")
        = T' (V - (k Gt D[b(i),0]) S)    (form "z", T' = T Diag(beta))
        = T' V - T' ((k Gt D[b(i),0]) S) (form "split": the two products with their
                                          own operand precisions, as the
                                          tensor-core kernel accumulates them)
     O  = scale ((q * Gt * D[b(i),0]) S + A_qk Vn)
     S  = Diag(D[nb,0]) S + K^(nb)^T Vn        (K^(nb) = k_j exp(G_{C-1} - G_j))

The 16-token blocks are where the per-step floor matters: within a block
every factor is bounded by e^{-16 floor}, inside bf16/fp32 range for floor >= -5.45
(fupanwang.com Kimi K3 report digest, KDA section, Fig. 3).

``prec`` (a dict operand -> "bf16" | "tf32" | "tf32t" | "fp16" | "fp16x256" |
"fp16d256" | "bf16x2" | "tf32x2")
rounds the tensor-core operands the way a kernel stores them ("tf32t": fp32
stored whole, the MMA reading only its leading 19 bits, i.e. truncation;
"...x2": a leading part plus a low part in that type, the product issued once
per part); ``KERNEL_PREC`` with ``KERNEL_FORM`` is the plan of the tcgen05
kernel: tf32 for the operands the output is sensitive to (the diagonal A
operands, T', Z), fp16 (the same 11-bit significand) for the off-diagonal A
operands and for the last product (2^8 A_qk, 2^8 K^ and 2^-8 V_new), the state
as two bf16 parts, bf16 for Q e^G / K e^G and T' in T' V.  beta is folded into the columns of T
(T' = T Diag(beta)).
"""
from __future__ import annotations

import numpy as np


def _bf16(x):
    """Round fp64 -> bf16 (round to nearest even) -> fp64."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _tf32(x):
    """Round fp64 -> fp32 -> tf32 (10-bit mantissa, nearest even) -> fp64."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 13) & 1
    u = (u + 0xFFF + lsb) & 0xFFFFE000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _tf32_trunc(x):
    """fp64 -> fp32, keeping the leading 19 bits (what a tf32 MMA reads of an
    unrounded fp32 operand) -> fp64."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


def _split2(rnd):
    """An operand carried as a leading part plus a low part, both in the same
    storage type (the product is issued once per part into one accumulator)."""
    def f(x):
        x = np.asarray(x, np.float32).astype(np.float64)
        hi = rnd(x)
        return hi + rnd(x - hi)
    return f


def _fp16(x):
    """Round fp64 -> fp16 (nearest even; subnormals kept, smaller values to 0) -> fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def _fp16_scaled(scale):
    """fp16 storage of scale * x (a power of two), read back as x: the scale moves
    the values away from fp16's subnormal and overflow ranges."""
    return lambda x: _fp16(np.asarray(x, np.float64) * scale) / scale


_ROUND = {"bf16": _bf16, "tf32": _tf32, "tf32t": _tf32_trunc, "fp16": _fp16,
          "fp16x256": _fp16_scaled(256.0), "fp16d256": _fp16_scaled(1.0 / 256.0),
          "bf16x2": _split2(_bf16), "tf32x2": _split2(_tf32),
          "fp32": lambda x: np.asarray(x, np.float32).astype(np.float64)}

# operand -> storage precision in the tcgen05 kernel, and the form of its V_new
KERNEL_PREC = {
    "Arow": "tf32", "Acol": "tf32",       # q~, k~ and Kbar of the diagonal A blocks (rounded)
    "Aoff": "fp16",                       # q~, k~ and K^(b) of the off-diagonal A blocks (all <= 1)
    "T": "tf32t", "TV": "bf16", "Y": "tf32t",
    "Aqk": "fp16x256", "Khat": "fp16x256", "Vn": "fp16d256",   # the last MMA: fp16, scales 2^8 / 2^-8
    "KG": "bf16", "S": "bf16x2", "QG": "bf16",
}
KERNEL_FORM = "split"


def _block_inverse(A, sub=16):
    """(I + A)^-1 for strictly lower-triangular A: invert the 16x16 diagonal
    blocks by forward substitution, then merge blocks pairwise (16 -> 32 -> 64)."""
    C = A.shape[0]
    T = np.zeros_like(A)
    for b0 in range(0, C, sub):
        blk = A[b0:b0 + sub, b0:b0 + sub]
        n = blk.shape[0]
        Ti = np.eye(n)
        for i in range(1, n):
            # row i of (I+L)^-1: t_i = e_i - sum_{k<i} L[i,k] t_k
            Ti[i, :i] = -blk[i, :i] @ Ti[:i, :i]
        T[b0:b0 + sub, b0:b0 + sub] = Ti
    w = sub
    while w < C:
        for b0 in range(0, C, 2 * w):
            lo = slice(b0, b0 + w)
            hi = slice(b0 + w, min(C, b0 + 2 * w))
            if hi.start >= C:
                continue
            # [[T11, 0], [T21, T22]]: T21 = -T22 A21 T11
            T[hi, lo] = -T[hi, hi] @ A[hi, lo] @ T[lo, lo]
        w *= 2
    return T


def chunked_kda(q, k, v, g, beta, S0=None, scale=None, gate=None, g_floor=-5.0,
                C=64, sub=16, prec=None, form="wy"):
    """One sequence, all heads.  q,k,g [T,H,dk]; v [T,H,dv]; beta [T,H];
    S0 [H,dk,dv].  Returns (o [T,H,dv], S_T [H,dk,dv]) in fp64."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    prec = prec or {}
    rb = lambda name, x: _ROUND[prec[name]](x) if name in prec else x
    o = np.zeros((T, H, dv))
    S_out = np.zeros((H, dk, dv))
    nb = C // sub
    for h in range(H):
        S = np.zeros((dk, dv)) if S0 is None else np.array(S0[h], dtype=np.float64)
        for c0 in range(0, T, C):
            L = min(C, T - c0)
            qc = np.zeros((C, dk)); kc = np.zeros((C, dk)); gc = np.zeros((C, dk))
            vc = np.zeros((C, dv)); bc = np.zeros(C)
            qc[:L] = q[c0:c0 + L, h]; kc[:L] = k[c0:c0 + L, h]
            gc[:L] = np.maximum(g[c0:c0 + L, h], g_floor)
            vc[:L] = v[c0:c0 + L, h]; bc[:L] = beta[c0:c0 + L, h]
            G = np.cumsum(gc, axis=0)
            r = np.zeros((nb + 1, dk))
            for b in range(1, nb + 1):
                r[b] = G[b * sub - 1]
            blk = np.arange(C) // sub
            Gt = np.exp(G - r[blk])
            Kbar = kc * np.exp(r[blk] - G)
            with np.errstate(over="ignore"):
                D = np.exp(r[:, None, :] - r[None, :, :])      # D[b, b'] (used for b >= b')
                Kb = [Kbar * D[b, blk] for b in range(nb + 1)]   # rows j in blocks > b unused
            Qt = rb("Arow", qc * Gt)
            Kt = rb("Arow", kc * Gt)
            A_qk = np.zeros((C, C)); A_kk = np.zeros((C, C))
            for b in range(nb):
                rows = slice(b * sub, (b + 1) * sub)
                # rows j of K^(b) past block b overflow; they only meet masked (j > i) entries
                with np.errstate(over="ignore", invalid="ignore"):
                    colraw = np.where(blk <= b, 1.0, 0.0)[:, None] * np.nan_to_num(Kb[b], posinf=0.0)
                colop = rb("Acol", colraw)
                A_qk[rows] = Qt[rows] @ colop.T
                A_kk[rows] = Kt[rows] @ colop.T
                if "Aoff" in prec:
                    # off-diagonal blocks (j in blocks < b) from their own operand precision
                    off = slice(0, b * sub)
                    qo, ko, co = (_ROUND[prec["Aoff"]](x) for x in (qc[rows] * Gt[rows], kc[rows] * Gt[rows], colraw[off]))
                    A_qk[rows, off] = qo @ co.T
                    A_kk[rows, off] = ko @ co.T
            ii, jj = np.meshgrid(np.arange(C), np.arange(C), indexing="ij")
            A_qk = np.where(jj <= ii, A_qk, 0.0)
            A_kk = np.where(jj < ii, A_kk, 0.0) * bc[:, None]
            Tb = rb("T", _block_inverse(A_kk, sub) * bc[None, :])   # T' = T Diag(beta)
            Dq = D[blk, 0]                                   # exp(r_{b(i)}) = Gamma / Gt
            Sb = rb("S", S)
            if form == "z":
                Z = rb("Z", vc - rb("KG", kc * Gt * Dq) @ Sb)
                Vn = rb("Vn", Tb @ Z)
            elif form == "split":
                T_raw = _block_inverse(A_kk, sub) * bc[None, :]
                Y = rb("Y", rb("KG", kc * Gt * Dq) @ Sb)
                Vn = rb("Vn", rb("TV", T_raw) @ vc - Tb @ Y)
            else:
                W = rb("W", Tb @ rb("KG", kc * Gt * Dq))
                U = Tb @ vc
                Vn = rb("Vn", U - W @ Sb)
            O = scale * (rb("QG", qc * Gt * Dq) @ Sb + rb("Aqk", A_qk) @ Vn)
            S = D[nb, 0][:, None] * S + rb("Khat", Kb[nb]).T @ Vn
            o[c0:c0 + L, h] = O[:L]
        S_out[h] = S
    if gate is not None:
        z = np.asarray(gate, dtype=np.float64)
        o = o / (1.0 + np.exp(-z))
    return o, S_out
