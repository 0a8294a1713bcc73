"""Speculative-decode verify and commit: the outputs of D draft tokens from a
state, and the in-place commit of an accepted prefix.  Pinned by the oracle
(the D tokens of each sequence as a prefill from the state) and by D single
decode steps."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import decode_step, device_status, inputs, spec_commit, spec_verify
from parity import TOL_BF16, TOL_FP32, rel_max, rel_max_beyond_bf16

pytestmark = pytest.mark.gpu


def _draft(B, D, H, d, dtype, seed, gate=True):
    inp = inputs.prefill_inputs([D] * B, H=H, dk=d, dv=d, dtype=dtype, device="cuda", seed=seed,
                                s0_std=0.05, gate=gate)
    shp = lambda t: None if t is None else t.view(B, D, *t.shape[1:])
    draft = {n: shp(inp[n]) for n in ("q", "k", "v", "g", "beta", "gate")}
    return inp, draft, inp["S0"].clone()


def _cpu(x):
    return None if x is None else x.detach().to("cpu")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("D", [1, 4, 5, 8])
def test_verify_and_commit_match_oracle(dtype, d, D):
    B, H = 3, 2
    inp, x, S = _draft(B, D, H, d, dtype, seed=31 + D)
    S_before = S.clone()
    o = spec_verify(x["q"], x["k"], x["v"], x["g"], x["beta"], S, gate=x["gate"])
    assert torch.equal(S, S_before)                           # verify reads the state only
    cu = np.array(inp["cu_seqlens_host"], dtype=np.int64)
    o_ref, _ = oracle.kda_fwd_ref(*(_cpu(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                  cu_seqlens=cu, S0=_cpu(S_before), gate=_cpu(inp["gate"]))
    o_flat = o.view(B * D, H, d)
    if dtype == torch.float32:
        assert rel_max(o_flat, o_ref) <= TOL_FP32
    else:
        assert rel_max_beyond_bf16(o_flat, o_ref) <= TOL_BF16
    # commit different accepted prefixes per sequence (0 .. D)
    acc = [0, D // 2, D][:B]
    spec_commit(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                torch.tensor(acc, dtype=torch.int32, device="cuda"))
    for b, a in enumerate(acc):
        if a == 0:
            assert torch.equal(S[b], S_before[b])
            continue
        rows = slice(int(cu[b]), int(cu[b]) + a)
        _, S_ref = oracle.kda_fwd_ref(*(_cpu(inp[n])[rows] for n in ("q", "k", "v", "g", "beta")),
                                      S0=_cpu(S_before[b:b + 1]))
        assert rel_max(S[b], S_ref[0]) <= (TOL_FP32 if dtype == torch.float32 else TOL_BF16)
    assert device_status() == 0


def test_commit_all_equals_decode_steps():
    """Committing all D tokens gives the state of D decode steps, and verify
    gives their outputs (same per-token arithmetic; fp32 I/O)."""
    B, D, H, d = 4, 6, 3, 128
    _, x, S = _draft(B, D, H, d, torch.float32, seed=41)
    S_dec = S.clone()
    o_dec = torch.stack([decode_step(x["q"][:, t].contiguous(), x["k"][:, t].contiguous(),
                                     x["v"][:, t].contiguous(), x["g"][:, t].contiguous(),
                                     x["beta"][:, t].contiguous(), S_dec,
                                     gate=x["gate"][:, t].contiguous()) for t in range(D)], dim=1)
    o = spec_verify(x["q"], x["k"], x["v"], x["g"], x["beta"], S, gate=x["gate"])
    spec_commit(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                torch.full((B,), D, dtype=torch.int32, device="cuda"))
    assert torch.allclose(o, o_dec, rtol=1e-5, atol=1e-6)
    assert torch.allclose(S, S_dec, rtol=1e-5, atol=1e-6)
    # counts outside [0, D] are clamped
    S2 = S.clone()
    spec_commit(x["q"], x["k"], x["v"], x["g"], x["beta"], S2,
                torch.tensor([-3, 0, 0, 0], dtype=torch.int32, device="cuda"))
    assert torch.equal(S2, S)
    assert device_status() == 0


@pytest.mark.parametrize("D,dk,dv,dtype", [(19, 128, 64, torch.float32), (64, 64, 128, torch.bfloat16)])
def test_long_draft_without_gate(D, dk, dv, dtype):
    """Drafts longer than one staged group of tokens (ragged last group), no
    output gate, dk != dv; the full commit gives the oracle's final state."""
    B, H = 2, 3
    inp = inputs.prefill_inputs([D] * B, H=H, dk=dk, dv=dv, dtype=dtype, device="cuda", seed=53 + D,
                                s0_std=0.05, gate=False)
    x = {n: inp[n].view(B, D, *inp[n].shape[1:]) for n in ("q", "k", "v", "g", "beta")}
    S = inp["S0"].clone()
    o = spec_verify(x["q"], x["k"], x["v"], x["g"], x["beta"], S)
    cu = np.array(inp["cu_seqlens_host"], dtype=np.int64)
    o_ref, S_ref = oracle.kda_fwd_ref(*(_cpu(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                      cu_seqlens=cu, S0=_cpu(inp["S0"]))
    spec_commit(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                torch.full((B,), D, dtype=torch.int32, device="cuda"))
    if dtype == torch.float32:
        assert rel_max(o.view(B * D, H, dv), o_ref) <= TOL_FP32
        assert rel_max(S, S_ref) <= TOL_FP32
    else:
        assert rel_max_beyond_bf16(o.view(B * D, H, dv), o_ref) <= TOL_BF16
        assert rel_max(S, S_ref) <= TOL_BF16
    assert device_status() == 0


def test_full_size_sampled():
    """The bench's launch: 512 sequences x 64 heads, 4 draft tokens verified,
    3 committed; sampled (sequence, head) pairs against the oracle."""
    B, D, H, d = 512, 4, 64, 128
    inp, x, S = _draft(B, D, H, d, torch.bfloat16, seed=59)
    S_before = S.clone()
    o = spec_verify(x["q"], x["k"], x["v"], x["g"], x["beta"], S, gate=x["gate"])
    spec_commit(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                torch.full((B,), 3, dtype=torch.int32, device="cuda"))
    assert device_status() == 0
    for b, h in ((0, 0), (137, 21), (511, 63), (300, 5)):
        sl = slice(b * D, (b + 1) * D)
        cut = lambda t, n=None: _cpu(t[sl, h:h + 1]) if n is None else _cpu(t[sl][:n, h:h + 1])
        o_ref, _ = oracle.kda_fwd_ref(*(cut(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                      S0=_cpu(S_before[b:b + 1, h:h + 1]), gate=cut(inp["gate"]))
        assert rel_max_beyond_bf16(o[b, :, h:h + 1], o_ref) <= TOL_BF16
        _, S_ref = oracle.kda_fwd_ref(*(cut(inp[n], 3) for n in ("q", "k", "v", "g", "beta")),
                                      S0=_cpu(S_before[b:b + 1, h:h + 1]))
        assert rel_max(S[b:b + 1, h:h + 1], S_ref) <= TOL_BF16
