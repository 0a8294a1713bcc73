"""Pins of the oracle backward (``kda_bwd_ref``, autograd through the token
recurrence) against central finite differences of the forward oracle
(``kda_fwd_ref``, the C loop), which shares no code with it.

L = sum(o * do) + sum(S_T * dS_T); every entry of every input is perturbed by
+-h and dL/dx = (L(x+h) - L(x-h)) / 2h, exact to O(h^2) in fp64.  A case with
part of g below the floor checks that the clamp passes no gradient there."""
import numpy as np
import pytest

import oracle


def _case(seed, lengths, H=2, dk=4, dv=3, gate=True, s0=True, below_floor=False):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    k = rng.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    x = {"q": rng.standard_normal((T, H, dk)), "k": k, "v": rng.standard_normal((T, H, dv)),
         "g": -rng.uniform(0.1, 1.0, (T, H, dk)), "beta": rng.uniform(0.1, 0.9, (T, H))}
    if below_floor:
        x["g"][::2, :, ::2] = -6.0                           # clamped to the floor (-5)
    x["gate"] = rng.standard_normal((T, H, dv)) if gate else None
    x["S0"] = 0.3 * rng.standard_normal((len(lengths), H, dk, dv)) if s0 else None
    do = rng.standard_normal((T, H, dv))
    dS_T = rng.standard_normal((len(lengths), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return x, do, dS_T, cu


def _loss(x, do, dS_T, cu):
    o, S_T = oracle.kda_fwd_ref(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=cu,
                                S0=x["S0"], gate=x["gate"], nthreads=1)
    return float(np.sum(o * do) + np.sum(S_T * dS_T))


@pytest.mark.parametrize("lengths,gate,s0,below", [([5], True, True, False), ([3, 4], False, True, False),
                                                   ([6], True, False, True)])
def test_backward_matches_finite_differences(lengths, gate, s0, below):
    x, do, dS_T, cu = _case(11 + len(lengths), lengths, gate=gate, s0=s0, below_floor=below)
    grads = oracle.kda_bwd_ref(x["q"], x["k"], x["v"], x["g"], x["beta"], do, cu_seqlens=cu,
                               S0=x["S0"], gate=x["gate"], dS_T=dS_T)
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta")]
    if gate:
        names.append(("gate", "dgate"))
    if s0:
        names.append(("S0", "dS0"))
    h = 1e-6
    for xn, gn in names:
        fd = np.zeros_like(x[xn])
        it = np.nditer(x[xn], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            keep = x[xn][idx]
            x[xn][idx] = keep + h
            lp = _loss(x, do, dS_T, cu)
            x[xn][idx] = keep - h
            lm = _loss(x, do, dS_T, cu)
            x[xn][idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(grads[gn] - fd)) / max(1.0, np.max(np.abs(fd)))
        assert err < 1e-6, (gn, err)
    if below:
        assert np.all(grads["dg"][::2, :, ::2] == 0.0)
