"""The chunked backward's factorisation (``chunk_bwd_mirror``, fp64) against the
oracle's autograd gradients (``kda_bwd_ref``): three stages, 16-token block
references and the chunk-end-state form of the gradient of the chunk's total
decay all reproduce the token recurrence's gradients to rounding."""
import numpy as np
import pytest
import torch

import oracle
from chunk_bwd_mirror import head_backward
from gated_delta_rule_136_b200 import inputs


def _run(lengths, H, dk, dv, seed, gate, s0, dS_T_on, g_mode="softplus"):
    inp = inputs.prefill_inputs(lengths, H=H, dk=dk, dv=dv, dtype=torch.float32, seed=seed,
                                s0_std=0.05 if s0 else None, gate=gate, g_mode=g_mode)
    rng = np.random.default_rng(seed + 100)
    T = sum(lengths)
    do = rng.standard_normal((T, H, dv))
    dS_T = 0.1 * rng.standard_normal((len(lengths), H, dk, dv)) if dS_T_on else None
    f = lambda t: None if t is None else t.double().numpy()
    x = {n: f(inp[n]) for n in ("q", "k", "v", "g", "beta", "gate", "S0")}
    cu = np.array(inp["cu_seqlens_host"], dtype=np.int64)
    ref = oracle.kda_bwd_ref(x["q"], x["k"], x["v"], x["g"], x["beta"], do, cu_seqlens=cu,
                             S0=x["S0"], gate=x["gate"], dS_T=dS_T, scale=inp["scale"])
    o_ref, _ = oracle.kda_fwd_ref(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=cu,
                                  S0=x["S0"], gate=x["gate"], scale=inp["scale"])
    got = {n: np.zeros_like(ref[n]) for n in ref}
    o = np.zeros_like(o_ref)
    for n in range(len(lengths)):
        sl = slice(cu[n], cu[n + 1])
        for h in range(H):
            r = head_backward(x["q"][sl, h], x["k"][sl, h], x["v"][sl, h], x["g"][sl, h],
                              x["beta"][sl, h], do[sl, h], None if x["gate"] is None else x["gate"][sl, h],
                              None if x["S0"] is None else x["S0"][n, h],
                              None if dS_T is None else dS_T[n, h], inp["scale"], -5.0)
            o[sl, h] = r["o"]
            for name in ("dq", "dk", "dv", "dg", "dgate"):
                if name in got:
                    got[name][sl, h] = r[name]
            got["dbeta"][sl, h] = r["dbeta"]
            if "dS0" in got:
                got["dS0"][n, h] = r["dS0"]
    return got, ref, o, o_ref


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b * b)), 1e-300))


@pytest.mark.parametrize("lengths,gate,s0,dst", [([150], True, True, True), ([64, 1, 70], False, True, False),
                                                 ([129, 0, 17], True, False, True)])
def test_chunk_bwd_mirror_matches_oracle_gradients(lengths, gate, s0, dst):
    got, ref, o, o_ref = _run(lengths, H=2, dk=16, dv=8, seed=5 + len(lengths), gate=gate, s0=s0, dS_T_on=dst)
    assert _rel(o, o_ref) < 1e-10
    for name in ref:
        assert _rel(got[name], ref[name]) < 1e-9, name


def test_chunk_bwd_mirror_floor_stress():
    """g spread down to the floor: block factors up to e^{16 |floor|}, clamped entries pass no gradient."""
    got, ref, o, o_ref = _run([100], H=1, dk=16, dv=8, seed=3, gate=True, s0=True, dS_T_on=True,
                              g_mode="floor_stress")
    assert _rel(o, o_ref) < 1e-10
    for name in ref:
        assert _rel(got[name], ref[name]) < 1e-9, name


def test_chunk_bwd_mirror_kernel_head_size():
    """dk = dv = 128, the chunked kernels' head size: three chunks, the last one ragged."""
    got, ref, o, o_ref = _run([150], H=1, dk=128, dv=128, seed=17, gate=True, s0=True, dS_T_on=True)
    assert _rel(o, o_ref) < 1e-10
    for name in ref:
        assert _rel(got[name], ref[name]) < 1e-9, name
