"""Context-parallel prefill (KCP) kernels on one GPU: the piece summaries
(kda_segment_summary), the fold of gathered summaries (kda_state_combine) and
the whole KCP data flow with the ranks emulated one after another on the same
GPU (their kernels never wait on one another), each against the oracle
(Kimi K3 report digest, section 基础设施: segment states plus the incoming
state times the transition product, joined by a prefix scan)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import (chunk_fwd, device_status, inputs, kcp_chunk_fwd,
                                       segment_summary, split_pieces, state_combine)
from parity import TOL_BF16, TOL_FP32, rel_max, rel_max_beyond_bf16

pytestmark = pytest.mark.gpu


def _cpu(x):
    return None if x is None else x.detach().to("cpu")


def _pieces_of(inp, pieces):
    cu = inp["cu_seqlens_host"]
    idx = torch.cat([torch.arange(cu[n] + a, cu[n] + b) for n, (a, b) in enumerate(pieces)]).cuda()
    loc = {n: (None if inp[n] is None else inp[n].index_select(0, idx).contiguous())
           for n in ("q", "k", "v", "g", "beta", "gate")}
    loc["cu_seqlens_host"] = [0] + np.cumsum([b - a for a, b in pieces]).tolist()
    loc["cu_seqlens"] = torch.tensor(loc["cu_seqlens_host"], dtype=torch.int32, device="cuda")
    return loc


@pytest.mark.parametrize("with_s0", [True, False])
def test_summary_matches_oracle(with_s0):
    """S_loc and M of ragged pieces, an empty one included."""
    inp = inputs.prefill_inputs([300, 0, 130, 64], H=2, dk=128, dv=128, device="cuda", seed=61,
                                s0_std=0.05)
    S0 = inp["S0"] if with_s0 else None
    summ = segment_summary(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                           inp["cu_seqlens_host"], S0=S0)
    cu = np.array(inp["cu_seqlens_host"])
    q, k, v, g, beta = (_cpu(inp[n]) for n in ("q", "k", "v", "g", "beta"))
    _, S_loc = oracle.kda_fwd_ref(q, k, v, g, beta, cu_seqlens=cu, S0=_cpu(S0))
    eye = np.broadcast_to(np.eye(128), (4, 2, 128, 128)).copy()
    _, M = oracle.kda_fwd_ref(q, k, torch.zeros_like(v), g, beta, cu_seqlens=cu, S0=eye)
    assert rel_max(summ[0], S_loc) <= TOL_BF16
    assert rel_max(summ[1], M) <= TOL_BF16
    assert torch.equal(summ[1, 1].cpu(), torch.eye(128).expand(2, 128, 128))   # empty piece: M = I
    assert device_status() == 0


@pytest.mark.parametrize("P", [1, 2, 5])
def test_combine_matches_fold(P):
    gen = torch.Generator().manual_seed(70 + P)
    N, H = 3, 2
    S_loc = torch.randn(P, N, H, 128, 128, generator=gen, dtype=torch.float64) * 0.05
    M = 0.9 * torch.eye(128, dtype=torch.float64) + 0.01 * torch.randn(P, N, H, 128, 128, generator=gen,
                                                                        dtype=torch.float64)
    summ = torch.stack([S_loc, M], dim=1)                       # [P, 2, N, H, D, D]
    got = state_combine(summ.float().cuda())
    ref = summ.float().double()[0, 0].clone()                   # the fp32 inputs, folded in fp64
    for p in range(1, P):
        ref = summ.float().double()[p, 1] @ ref + summ.float().double()[p, 0]
    assert rel_max(got, ref) <= TOL_FP32
    assert device_status() == 0


@pytest.mark.parametrize("lengths,H,world", [([300, 130, 64], 2, 3), ([4096], 4, 4)])
def test_emulated_ranks_match_whole_sequence(lengths, H, world):
    """Every rank's summary, the all-gathered stack, each rank's fold and its
    rerun, one rank after another on this GPU; outputs and the last rank's
    final state against the oracle over the whole sequences."""
    inp = inputs.prefill_inputs(lengths, H=H, dk=128, dv=128, device="cuda", seed=83, s0_std=0.05,
                                gate=True)
    per_rank = split_pieces(lengths, world)
    locs = [_pieces_of(inp, per_rank[r]) for r in range(world)]
    summ = []
    for r, loc in enumerate(locs):
        if r < world - 1:
            summ.append(segment_summary(loc["q"], loc["k"], loc["v"], loc["g"], loc["beta"],
                                        loc["cu_seqlens"], loc["cu_seqlens_host"],
                                        S0=inp["S0"] if r == 0 else None, with_M=r > 0))
        else:
            summ.append(torch.zeros_like(summ[0]))
    gathered = torch.stack(summ)
    outs = []
    for r, loc in enumerate(locs):
        S_in = inp["S0"] if r == 0 else state_combine(gathered[:r].contiguous())
        outs.append(chunk_fwd(loc["q"], loc["k"], loc["v"], loc["g"], loc["beta"], S0=S_in,
                              cu_seqlens=loc["cu_seqlens"], cu_seqlens_host=loc["cu_seqlens_host"],
                              gate=loc["gate"]))
    o_ref, S_ref = oracle.kda_fwd_ref(*(_cpu(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                      cu_seqlens=np.array(inp["cu_seqlens_host"]), S0=_cpu(inp["S0"]),
                                      gate=_cpu(inp["gate"]))
    cu = inp["cu_seqlens_host"]
    for n in range(len(lengths)):
        parts = []
        for r in range(world):
            lens = [b - a for a, b in per_rank[r]]
            s = int(sum(lens[:n]))
            parts.append(outs[r][0][s:s + lens[n]])
        assert rel_max_beyond_bf16(torch.cat(parts), o_ref[cu[n]:cu[n + 1]]) <= TOL_BF16
    assert rel_max(outs[-1][1], S_ref) <= TOL_BF16
    assert device_status() == 0


def test_single_rank_is_plain_prefill():
    """Without a process group KCP is the plain prefill."""
    inp = inputs.prefill_inputs([200, 77], H=2, dk=128, dv=128, device="cuda", seed=91, s0_std=0.05)
    args = [inp[n] for n in ("q", "k", "v", "g", "beta")]
    o1, S1 = kcp_chunk_fwd(*args, inp["cu_seqlens"], inp["cu_seqlens_host"], S0=inp["S0"])
    o2, S2 = chunk_fwd(*args, S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
                       cu_seqlens_host=inp["cu_seqlens_host"])
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def _summary_with_segments(inp, S0, segments):
    import os
    old = os.environ.get("KDA_SEGMENTS")
    try:
        if segments is None:
            os.environ.pop("KDA_SEGMENTS", None)
        else:
            os.environ["KDA_SEGMENTS"] = str(segments)
        return segment_summary(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["cu_seqlens"],
                               inp["cu_seqlens_host"], S0=S0)
    finally:
        if old is None:
            os.environ.pop("KDA_SEGMENTS", None)
        else:
            os.environ["KDA_SEGMENTS"] = old


@pytest.mark.parametrize("lengths,segments", [([1000, 300], 3), ([300, 1000], 3), ([8192], None)])
def test_split_summary_matches_oracle_and_unsplit(lengths, segments):
    """Pieces cut into sub-segments (forced, or chosen because the chains are
    fewer than the SMs) and folded by the scan: S_loc and M as the oracle's
    and as the one-chain summary's."""
    inp = inputs.prefill_inputs(lengths, H=2, dk=128, dv=128, device="cuda", seed=67, s0_std=0.05,
                                g_mode="floor_stress")
    split = _summary_with_segments(inp, inp["S0"], segments)
    whole = _summary_with_segments(inp, inp["S0"], 1)
    cu = np.array(inp["cu_seqlens_host"])
    q, k, v, g, beta = (_cpu(inp[n]) for n in ("q", "k", "v", "g", "beta"))
    _, S_loc = oracle.kda_fwd_ref(q, k, v, g, beta, cu_seqlens=cu, S0=_cpu(inp["S0"]))
    eye = np.broadcast_to(np.eye(128), (len(lengths), 2, 128, 128)).copy()
    _, M = oracle.kda_fwd_ref(q, k, torch.zeros_like(v), g, beta, cu_seqlens=cu, S0=eye)
    for got in (split, whole):
        assert rel_max(got[0], S_loc) <= TOL_BF16
        assert rel_max(got[1], M) <= TOL_BF16
    assert rel_max(split[0], whole[0].cpu()) <= TOL_BF16 and rel_max(split[1], whole[1].cpu()) <= TOL_BF16
    assert device_status() == 0
