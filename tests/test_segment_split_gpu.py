"""Long-sequence segment split (context parallelism inside one GPU): each
segment's own state and transition product are computed independently,
joined by a prefix scan, and every segment is rerun from its true incoming
state (fupanwang.com Kimi K3 report digest, section 基础设施).  The split is
a tiling choice: results must match the oracle and the unsplit run.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import chunk_fwd, device_status, inputs
from parity import TOL_BF16, rel_max, rel_max_beyond_bf16

pytestmark = pytest.mark.gpu


def _cpu(x):
    return None if x is None else x.detach().to("cpu")


def _run(inp, segments=None):
    old = os.environ.get("KDA_SEGMENTS")
    try:
        if segments is None:
            os.environ.pop("KDA_SEGMENTS", None)
        else:
            os.environ["KDA_SEGMENTS"] = str(segments)
        return chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                         cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"],
                         gate=inp["gate"])
    finally:
        if old is None:
            os.environ.pop("KDA_SEGMENTS", None)
        else:
            os.environ["KDA_SEGMENTS"] = old


def _oracle(inp, heads=None):
    q, k, v, g, beta, gate = (_cpu(inp[n]) for n in ("q", "k", "v", "g", "beta", "gate"))
    S0 = _cpu(inp["S0"])
    if heads is not None:
        sel = lambda t: None if t is None else t[:, heads].contiguous()
        q, k, v, g, beta, gate = (sel(t) for t in (q, k, v, g, beta, gate))
        S0 = None if S0 is None else S0[:, heads].contiguous()
    return oracle.kda_fwd_ref(q, k, v, g, beta, cu_seqlens=np.array(inp["cu_seqlens_host"]),
                              S0=S0, gate=gate)


@pytest.mark.parametrize("g_mode", ["softplus", "floor_stress"])
def test_forced_split_matches_oracle_and_unsplit(g_mode):
    inp = inputs.prefill_inputs([1000], H=2, dk=128, dv=128, device="cuda", seed=41, s0_std=0.05,
                                g_mode=g_mode, gate=True)
    o_s, S_s = _run(inp, segments=4)
    o_u, S_u = _run(inp, segments=1)
    o_ref, S_ref = _oracle(inp)
    assert rel_max_beyond_bf16(o_s, o_ref) <= TOL_BF16 and rel_max(S_s, S_ref) <= TOL_BF16
    assert rel_max_beyond_bf16(o_s, o_u) <= TOL_BF16 and rel_max(S_s, S_u) <= TOL_BF16
    assert device_status() == 0


def test_slow_decay_split_carries_state():
    """With slow decay the transition products are far from zero, so a wrong
    M or scan would show."""
    inp = inputs.prefill_inputs([1500], H=2, dk=128, dv=128, device="cuda", seed=43, s0_std=0.05)
    inp["g"].mul_(0.02)
    o_s, S_s = _run(inp, segments=5)
    o_ref, S_ref = _oracle(inp)
    assert rel_max_beyond_bf16(o_s, o_ref) <= TOL_BF16 and rel_max(S_s, S_ref) <= TOL_BF16


def test_varlen_only_long_sequences_split():
    inp = inputs.prefill_inputs([700, 60, 1300, 0, 129], H=3, dk=128, dv=128, device="cuda",
                                seed=47, s0_std=0.05, gate=True)
    o_s, S_s = _run(inp, segments=3)
    o_ref, S_ref = _oracle(inp)
    assert rel_max_beyond_bf16(o_s, o_ref) <= TOL_BF16 and rel_max(S_s, S_ref) <= TOL_BF16
    assert torch.equal(S_s[3], inp["S0"][3])


def test_split_with_different_segment_counts():
    """Sequences cut into different numbers of segments (2 for 300 tokens, 3
    for 1300 under a forced 3), the smaller count first: each (sequence,
    head) takes its own P segments of the split buffers."""
    inp = inputs.prefill_inputs([300, 1300], H=3, dk=128, dv=128, device="cuda", seed=49, s0_std=0.05)
    o_s, S_s = _run(inp, segments=3)
    o_ref, S_ref = _oracle(inp)
    assert rel_max_beyond_bf16(o_s, o_ref) <= TOL_BF16 and rel_max(S_s, S_ref) <= TOL_BF16
    assert device_status() == 0


def test_long_sequence_default_policy_floor_stress():
    """1 sequence x 32 heads x 65536 tokens, decay near the floor: fewer units
    than SMs, so the default policy splits; two heads checked in full."""
    inp = inputs.prefill_inputs([65536], H=32, dk=128, dv=128, device="cuda", seed=3,
                                g_mode="floor_stress")
    o, S = _run(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    heads = [0, 31]
    o_ref, S_ref = _oracle(inp, heads=heads)
    assert rel_max_beyond_bf16(o[:, heads], o_ref) <= TOL_BF16
    assert rel_max(S[:, heads], S_ref) <= TOL_BF16
    assert device_status() == 0
