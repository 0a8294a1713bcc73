"""CPU fp64 oracle for the Kimi Delta Attention (KDA) forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``gated_delta_rule_136_b200``) shares no code with it and never calls it.

Two independent formulations live here:

* :func:`kda_fwd_ref` -- the token-by-token recurrence in plain C (fp64,
  OpenMP over independent (sequence, head) units), ``kda_oracle.c``.  It is the
  oracle every GPU result is compared with.
* :func:`transition_product_ref` -- for short sequences (T <= 8), the state and
  every output written as explicit products of the dk x dk transition matrices
  ``A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)`` ("Diagonal-Plus-Low-Rank"
  transition, page "Kimi K3 深度拆解", 突破一), in NumPy.  It shares nothing
  with the C loop and pins it.

Inputs are taken at the exact values the GPU receives (bf16 tensors are
upcast exactly) and all arithmetic is fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libkda_oracle.so")

_lib = None


def build(force: bool = False, extra_flags=None, out_path: str | None = None) -> str:
    """Compile ``kda_oracle.c`` into a shared library with gcc and OpenMP.

    ``extra_flags``/``out_path`` let a test build a variant into a scratch
    path; the default build goes to ``oracle/_build/libkda_oracle.so``.
    """
    out = out_path or _LIB_PATH
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (not force and out_path is None and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", out, "-lm"]
    if extra_flags:
        cmd[1:1] = list(extra_flags)
    subprocess.run(cmd, check=True)
    return out


def _load(path: str | None = None):
    lib = ctypes.CDLL(path or build())
    f = lib.kda_oracle_fwd
    dp = ctypes.POINTER(ctypes.c_double)
    f.argtypes = [ctypes.c_int32, ctypes.POINTER(ctypes.c_int64), ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int32, dp, dp, dp, dp, dp, dp, dp,
                  ctypes.c_double, ctypes.c_double, dp, dp, ctypes.c_int32]
    f.restype = ctypes.c_int
    lib.kda_oracle_max_threads.restype = ctypes.c_int32
    return lib


def _get_lib():
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def max_threads() -> int:
    """Host threads the oracle uses by default."""
    return int(_get_lib().kda_oracle_max_threads())


def _f64(x):
    """Exact fp64 copy of a numpy array or torch tensor (bf16 upcasts exactly)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor, any device / dtype
        import torch
        x = x.detach().to("cpu")
        if x.dtype != torch.float64:
            x = x.to(torch.float64)
        return np.ascontiguousarray(x.numpy())
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def kda_fwd_ref(q, k, v, g, beta, cu_seqlens=None, S0=None, scale=None,
                gate=None, g_floor=-5.0, nthreads=0, lib=None):
    """Token-by-token KDA forward in fp64 (the oracle).

    Shapes: q,k,g [T,H,dk] (or [B,T,H,dk] with ``cu_seqlens`` None);
    v, gate [T,H,dv]; beta [T,H]; S0 [N,H,dk,dv] or None (zeros).
    ``scale`` defaults to 1/sqrt(dk).  Returns ``(o, S_T)`` as float64 numpy
    arrays, ``o`` in the layout of ``v`` and ``S_T`` [N,H,dk,dv].
    """
    q, k, v, g, beta = (_f64(t) for t in (q, k, v, g, beta))
    gate, S0 = _f64(gate), _f64(S0)
    batched = q.ndim == 4
    if batched:
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens is for packed [T,H,d] inputs")
        B, T = q.shape[:2]
        cu = np.arange(0, (B + 1) * T, T, dtype=np.int64)
        shape_o = v.shape
        q, k, g = (t.reshape(B * T, *t.shape[2:]) for t in (q, k, g))
        v = v.reshape(B * T, *v.shape[2:])
        beta = beta.reshape(B * T, -1)
        if gate is not None:
            gate = gate.reshape(B * T, *gate.shape[2:])
    else:
        T = q.shape[0]
        cu = (np.array([0, T], dtype=np.int64) if cu_seqlens is None
              else np.ascontiguousarray(np.asarray(
                  cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                  dtype=np.int64)))
        shape_o = v.shape
    Ttot, H, dk = q.shape
    dv = v.shape[-1]
    N = len(cu) - 1
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    o = np.zeros((Ttot, H, dv), dtype=np.float64)
    S_T = np.zeros((N, H, dk, dv), dtype=np.float64)
    if S0 is not None:
        S0 = np.ascontiguousarray(S0.reshape(N, H, dk, dv))
    lib = lib or _get_lib()
    rc = lib.kda_oracle_fwd(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, dk, dv,
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gate), _ptr(S0),
        float(scale), float(g_floor), _ptr(o), _ptr(S_T), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_fwd failed with code {rc}")
    return o.reshape(shape_o), S_T


def kda_decode_ref(q, k, v, g, beta, S, gate=None, scale=None, g_floor=-5.0,
                   nthreads=0, lib=None):
    """One decode step per (sequence, head): the recurrence applied to a
    single token.  q,k,g [B,H,dk]; v, gate [B,H,dv]; beta [B,H];
    S [B,H,dk,dv].  Returns ``(o [B,H,dv], S_new [B,H,dk,dv])``."""
    q = _f64(q)
    B = q.shape[0]
    cu = np.arange(B + 1, dtype=np.int64)
    return kda_fwd_ref(q, k, v, g, beta, cu_seqlens=cu, S0=S, scale=scale,
                       gate=gate, g_floor=g_floor, nthreads=nthreads, lib=lib)


def transition_product_ref(q, k, v, g, beta, S0=None, scale=None, gate=None,
                           g_floor=-5.0):
    """Second, independent oracle for one short sequence (T <= 8), one head.

    Forms the transition matrices A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)
    explicitly (diagonal plus rank one) and evaluates

        S_t = (A_t ... A_1) S0 + sum_{s<=t} (A_t ... A_{s+1}) beta_s k_s v_s^T
        o_t = scale * S_t^T q_t  (times sigmoid(gate_t) when given)

    as matrix products.  q,k,g [T,dk]; v [T,dv]; beta [T]; S0 [dk,dv].
    Returns ``(o [T,dv], S_T [dk,dv])``.
    """
    q, k, v, g, beta = (_f64(t) for t in (q, k, v, g, beta))
    gate, S0 = _f64(gate), _f64(S0)
    T, dk = q.shape
    dv = v.shape[1]
    if T > 8:
        raise ValueError("transition_product_ref is meant for T <= 8")
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    if S0 is None:
        S0 = np.zeros((dk, dv))
    eye = np.eye(dk)
    A = [(eye - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(np.maximum(g[t], g_floor)))
         for t in range(T)]
    writes = [beta[t] * np.outer(k[t], v[t]) for t in range(T)]
    o = np.zeros((T, dv))
    S_t = None
    for t in range(T):
        prod = eye.copy()
        for r in range(t, -1, -1):      # A_t A_{t-1} ... A_0
            prod = prod @ A[r]
        S_t = prod @ S0
        for s in range(t + 1):
            tail = eye.copy()
            for r in range(t, s, -1):   # A_t ... A_{s+1}
                tail = tail @ A[r]
            S_t = S_t + tail @ writes[s]
        o[t] = scale * (S_t.T @ q[t])
        if gate is not None:
            o[t] = o[t] / (1.0 + np.exp(-gate[t]))
    return o, S_t


def kda_bwd_ref(q, k, v, g, beta, do, cu_seqlens=None, S0=None, gate=None, dS_T=None,
                scale=None, g_floor=-5.0):
    """Gradients of the KDA forward, in fp64, by reverse-mode differentiation
    (PyTorch autograd) of the token-by-token recurrence written out below.

    The forward is the one :func:`kda_fwd_ref` computes, per head:
        alpha_t = exp(max(g_t, g_floor)),  S' = Diag(alpha_t) S,
        S = S' + beta_t k_t (v_t - S'^T k_t)^T,  o_t = scale S^T q_t [* sigmoid(gate_t)].
    The gradient is that of L = sum(o * do) + sum(S_T * dS_T): the vector-
    Jacobian product with the output gradient ``do`` [T,H,dv] and, optionally,
    the final-state gradient ``dS_T`` [N,H,dk,dv].  Where g equals the floor the
    derivative of max(g, floor) is taken as 1 (the clamp passes it through).
    Returns a dict of float64 numpy arrays: dq, dk, dv, dg, dbeta, and dgate
    and dS0 when ``gate`` / ``S0`` are given.  Meant for short sequences: the
    recurrence is unrolled in the autograd graph.
    """
    import torch

    def leaf(x):
        return None if x is None else torch.from_numpy(_f64(x)).requires_grad_(True)

    q, k, v, g, beta, gate, S0 = (leaf(x) for x in (q, k, v, g, beta, gate, S0))
    do = torch.from_numpy(_f64(do))
    dS_T = None if dS_T is None else torch.from_numpy(_f64(dS_T))
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = ([0, T] if cu_seqlens is None else
          [int(x) for x in np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens)])
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    alpha = torch.exp(torch.clamp(g, min=g_floor))
    loss = torch.zeros((), dtype=torch.float64)
    for n in range(len(cu) - 1):
        S = S0[n] if S0 is not None else torch.zeros(H, dk, dv, dtype=torch.float64)
        for t in range(cu[n], cu[n + 1]):
            S = alpha[t][:, :, None] * S
            u = torch.einsum("hkv,hk->hv", S, k[t])
            S = S + beta[t][:, None, None] * k[t][:, :, None] * (v[t] - u)[:, None, :]
            o = scale * torch.einsum("hkv,hk->hv", S, q[t])
            if gate is not None:
                o = o * torch.sigmoid(gate[t])
            loss = loss + (o * do[t]).sum()
        if dS_T is not None:
            loss = loss + (S * dS_T[n]).sum()
    loss.backward()
    out = {"dq": q.grad, "dk": k.grad, "dv": v.grad, "dg": g.grad, "dbeta": beta.grad}
    if gate is not None:
        out["dgate"] = gate.grad
    if S0 is not None:
        out["dS0"] = S0.grad
    return {name: (np.zeros(x.shape) if x is None else x.numpy()) for name, x in
            ((nm, out[nm]) for nm in out)}


def rel_err(x, ref) -> float:
    """max|x - ref| / RMS(ref): the parity metric used throughout."""
    x = _f64(x)
    ref = _f64(ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    d = float(np.max(np.abs(x - ref)))
    return d / rms if rms > 0 else d
