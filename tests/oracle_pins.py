"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics,
each checkable without trusting the oracle's own loop.

Every check takes the compiled oracle library (``lib``) so the same checks
can be run against deliberately broken copies of it (tests/test_oracle_mutants.py).
Each raises AssertionError on failure.

What pins what:
  closed_form_single_token   o_1 = scale*beta*(k.q)*v, S_1 = beta k v^T from S0 = 0
                             (read-out uses the state after the token's own write)
  frozen_state_beta_zero     beta = 0: S_t = Diag(exp(sum g)) S0, o_t = scale*S_t^T q_t
                             (decay acts per key row; no write)
  linear_attention_onehot    alpha = 1, mutually orthogonal keys: exact causal linear
                             attention with beta-weighted values
  linear_attention_limit     beta = eps -> 0: S_T / eps -> sum_t k_t v_t^T
  gated_deltanet_reduction   a scalar gate (same g on every channel) gives gated
                             DeltaNet, written as explicit matrices
  delta_rule_exact_recall    beta = 1, |k| = 1: S_t^T k_t = v_t for any decay
  three_step_picture         one-hot key e_i, beta = 0.7: row i -> (1-b)*a_i*row_i + b*v,
                             other rows only decay (page "Kimi-K3 为什么这么强？", §① ②)
  transition_product         T <= 8 against the explicit DPLR product
                             (page "Kimi K3 深度拆解", 突破一)
  stability_bound            |S_t|_F <= |S_{t-1}|_F + beta |v_t| for beta in [0,2]
  floor_clamp                values below the floor act as the floor (fupanwang.com
                             digest, KDA section, Fig. 3a)
  packing_invariance         packed sequences == separate runs; empty sequence keeps S0
  gate_special_values        sigmoid gate: z = 0 halves o, large z leaves it unchanged
"""
from __future__ import annotations

import numpy as np

import oracle

RTOL = 1e-11


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_inputs(rng, T, H, dk, dv, g_lo=-3.0):
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    g = rng.uniform(g_lo, 0.0, (T, H, dk))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    return q, k, v, g, beta


def _close(a, b, tol=RTOL, what=""):
    a = np.asarray(a)
    b = np.asarray(b)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if b.size else 0.0
    assert err <= tol * scale, f"{what}: max|diff| {err:.3e} > {tol:.1e} * {scale:.3e}"


def closed_form_single_token(lib):
    rng = _rng(1)
    for dk, dv in ((8, 8), (16, 12)):
        q, k, v, g, beta = _rand_inputs(rng, 1, 2, dk, dv)
        z = rng.standard_normal((1, 2, dv))
        for scale in (1.0, 0.37):
            o, S = oracle.kda_fwd_ref(q, k, v, g, beta, scale=scale, gate=z, lib=lib)
            for h in range(2):
                b = beta[0, h]
                exp_S = b * np.outer(k[0, h], v[0, h])
                exp_o = scale * b * float(k[0, h] @ q[0, h]) * v[0, h] / (1 + np.exp(-z[0, h]))
                _close(S[0, h], exp_S, what="S_1")
                _close(o[0, h], exp_o, what="o_1")


def frozen_state_beta_zero(lib):
    rng = _rng(2)
    T, H, dk, dv = 7, 2, 6, 5
    q, k, v, g, _ = _rand_inputs(rng, T, H, dk, dv)
    beta = np.zeros((T, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    o, S = oracle.kda_fwd_ref(q, k, v, g, beta, S0=S0, scale=1.0, lib=lib)
    for h in range(H):
        cum = np.zeros(dk)
        for t in range(T):
            cum += g[t, h]
            St = np.exp(cum)[:, None] * S0[0, h]
            _close(o[t, h], St.T @ q[t, h], what=f"o_t beta=0 t={t}")
        _close(S[0, h], St, what="S_T beta=0")
    # with alpha = 1 as well, the state is exactly frozen
    o, S = oracle.kda_fwd_ref(q, k, v, np.zeros_like(g), beta, S0=S0, scale=0.5, lib=lib)
    _close(S, S0, what="frozen S")
    for t in range(T):
        for h in range(H):
            _close(o[t, h], 0.5 * S0[0, h].T @ q[t, h], what="frozen o")


def linear_attention_onehot(lib):
    rng = _rng(3)
    T, H, dk, dv = 6, 2, 8, 5
    perm = rng.permutation(dk)[:T]
    k = np.zeros((T, H, dk))
    for t in range(T):
        k[t, :, perm[t]] = 1.0
    q = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    beta = rng.uniform(0.1, 1.0, (T, H))
    g = np.zeros((T, H, dk))
    o, S = oracle.kda_fwd_ref(q, k, v, g, beta, scale=1.0, lib=lib)
    for h in range(H):
        acc = np.zeros((dk, dv))
        for t in range(T):
            acc = acc + beta[t, h] * np.outer(k[t, h], v[t, h])
            # causal linear attention read-out: sum_{s<=t} beta_s (k_s . q_t) v_s
            lin = sum(beta[s, h] * float(k[s, h] @ q[t, h]) * v[s, h] for s in range(t + 1))
            _close(o[t, h], lin, what="linear attention o")
        _close(S[0, h], acc, what="linear attention S")


def linear_attention_limit(lib):
    rng = _rng(4)
    T, H, dk, dv = 16, 1, 8, 8
    q, k, v, _, _ = _rand_inputs(rng, T, H, dk, dv)
    g = np.zeros((T, H, dk))
    target = sum(np.outer(k[t, 0], v[t, 0]) for t in range(T))
    errs = []
    for eps in (1e-3, 1e-5):
        beta = np.full((T, H), eps)
        _, S = oracle.kda_fwd_ref(q, k, v, g, beta, lib=lib)
        errs.append(float(np.max(np.abs(S[0, 0] / eps - target))))
    # first-order error: shrinks in proportion to eps and stays O(eps * T^2)
    assert errs[1] <= 1e-5 * T * T * 10, errs
    assert errs[1] < errs[0] * 0.05, errs


def gated_deltanet_reduction(lib):
    rng = _rng(5)
    T, H, dk, dv = 20, 2, 8, 6
    q, k, v, _, beta = _rand_inputs(rng, T, H, dk, dv)
    a_log = rng.uniform(-1.0, 0.0, (T, H))
    g = np.repeat(a_log[:, :, None], dk, axis=2)
    S0 = rng.standard_normal((1, H, dk, dv)) * 0.1
    o, S = oracle.kda_fwd_ref(q, k, v, g, beta, S0=S0, scale=1.0, lib=lib)
    I = np.eye(dk)
    for h in range(H):
        M = S0[0, h].copy()
        for t in range(T):
            a = np.exp(a_log[t, h])
            M = a * (I - beta[t, h] * np.outer(k[t, h], k[t, h])) @ M \
                + beta[t, h] * np.outer(k[t, h], v[t, h])
            _close(o[t, h], M.T @ q[t, h], what="GDN o")
        _close(S[0, h], M, what="GDN S")


def delta_rule_exact_recall(lib):
    rng = _rng(6)
    T, H, dk, dv = 24, 2, 16, 16
    _, k, v, g, _ = _rand_inputs(rng, T, H, dk, dv, g_lo=-4.0)
    beta = np.ones((T, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    # q = k and scale = 1, so o_t = S_t^T k_t must reproduce v_t exactly
    o, _ = oracle.kda_fwd_ref(k, k, v, g, beta, S0=S0, scale=1.0, lib=lib)
    _close(o, v, tol=1e-12, what="exact recall")


def three_step_picture(lib):
    rng = _rng(7)
    dk, dv, H = 6, 4, 1
    S0 = rng.standard_normal((1, H, dk, dv))
    for i in range(dk):
        k = np.zeros((1, H, dk))
        k[0, 0, i] = 1.0
        q = rng.standard_normal((1, H, dk))
        v = rng.standard_normal((1, H, dv))
        g = rng.uniform(-2.0, 0.0, (1, H, dk))
        beta = np.full((1, H), 0.7)
        _, S = oracle.kda_fwd_ref(q, k, v, g, beta, S0=S0, lib=lib)
        alpha = np.exp(g[0, 0])
        exp_S = alpha[:, None] * S0[0, 0]                 # step 1: every row forgets
        exp_S[i] = (1 - 0.7) * exp_S[i] + 0.7 * v[0, 0]    # steps 2-3: weaken, write
        _close(S[0, 0], exp_S, what=f"three-step row {i}")


def transition_product(lib):
    rng = _rng(8)
    for T, dk, dv in ((1, 4, 3), (5, 6, 6), (8, 8, 5)):
        H = 2
        q, k, v, g, beta = _rand_inputs(rng, T, H, dk, dv, g_lo=-7.0)  # some below floor
        beta = beta * 1.8
        z = rng.standard_normal((T, H, dv))
        S0 = rng.standard_normal((1, H, dk, dv))
        o, S = oracle.kda_fwd_ref(q, k, v, g, beta, S0=S0, gate=z, lib=lib)
        for h in range(H):
            o2, S2 = oracle.transition_product_ref(q[:, h], k[:, h], v[:, h], g[:, h],
                                                   beta[:, h], S0=S0[0, h], gate=z[:, h])
            _close(o[:, h], o2, tol=1e-12, what="transition product o")
            _close(S[0, h], S2, tol=1e-12, what="transition product S")


def stability_bound(lib):
    rng = _rng(9)
    B, H, dk, dv, T = 3, 2, 8, 8, 30
    S = rng.standard_normal((B, H, dk, dv))
    for _ in range(T):
        q, k, v, g, _ = _rand_inputs(rng, B, H, dk, dv, g_lo=-1.0)
        beta = rng.uniform(0.0, 2.0, (B, H))
        _, S_new = oracle.kda_decode_ref(q, k, v, g, beta, S, lib=lib)
        for b in range(B):
            for h in range(H):
                lhs = np.linalg.norm(S_new[b, h])
                rhs = np.linalg.norm(S[b, h]) + beta[b, h] * np.linalg.norm(v[b, h])
                assert lhs <= rhs * (1 + 1e-12), (lhs, rhs)
        S = S_new


def floor_clamp(lib):
    rng = _rng(10)
    T, H, dk, dv = 9, 2, 6, 6
    q, k, v, g, beta = _rand_inputs(rng, T, H, dk, dv, g_lo=-9.0)
    S0 = rng.standard_normal((1, H, dk, dv))
    o1, S1 = oracle.kda_fwd_ref(q, k, v, g, beta, S0=S0, g_floor=-5.0, lib=lib)
    o2, S2 = oracle.kda_fwd_ref(q, k, v, np.maximum(g, -5.0), beta, S0=S0,
                                g_floor=-1e30, lib=lib)
    _close(o1, o2, what="floor o")
    _close(S1, S2, what="floor S")
    assert (g < -5.0).any()
    o3, _ = oracle.kda_fwd_ref(q, k, v, g, beta, S0=S0, g_floor=-1e30, lib=lib)
    assert np.max(np.abs(o3 - o1)) > 1e-6, "floor must matter for g below it"


def packing_invariance(lib):
    rng = _rng(11)
    lens = [5, 0, 9, 1]
    T, H, dk, dv = sum(lens), 2, 6, 4
    q, k, v, g, beta = _rand_inputs(rng, T, H, dk, dv)
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    o, S = oracle.kda_fwd_ref(q, k, v, g, beta, cu_seqlens=cu, S0=S0, lib=lib)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        if b == a:
            _close(S[n], S0[n], what="empty sequence keeps S0")
            continue
        o_n, S_n = oracle.kda_fwd_ref(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b],
                                      S0=S0[n:n + 1], lib=lib)
        _close(o[a:b], o_n, what="packed o")
        _close(S[n], S_n[0], what="packed S")


def gate_special_values(lib):
    rng = _rng(12)
    T, H, dk, dv = 6, 2, 5, 7
    q, k, v, g, beta = _rand_inputs(rng, T, H, dk, dv)
    o0, _ = oracle.kda_fwd_ref(q, k, v, g, beta, lib=lib)
    o_half, _ = oracle.kda_fwd_ref(q, k, v, g, beta, gate=np.zeros((T, H, dv)), lib=lib)
    o_one, _ = oracle.kda_fwd_ref(q, k, v, g, beta, gate=np.full((T, H, dv), 80.0), lib=lib)
    _close(o_half, 0.5 * o0, what="gate z=0")
    _close(o_one, o0, what="gate z=+80")
    assert np.max(np.abs(o0)) > 1e-3


ALL_PINS = [
    closed_form_single_token,
    frozen_state_beta_zero,
    linear_attention_onehot,
    linear_attention_limit,
    gated_deltanet_reduction,
    delta_rule_exact_recall,
    three_step_picture,
    transition_product,
    stability_bound,
    floor_clamp,
    packing_invariance,
    gate_special_values,
]
