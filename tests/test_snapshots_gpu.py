"""State snapshots (the prefix-cache hook): the state after every `interval`
tokens of each sequence.  Each snapshot is pinned by the oracle run on that
prefix (its final state), and at full size by the final state of the same
call where a sequence ends on a snapshot position."""
import os

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import chunk_fwd, chunk_fwd_snapshots, device_status, inputs
from parity import TOL_BF16, TOL_FP32, rel_max

pytestmark = pytest.mark.gpu


def _cpu(x):
    return None if x is None else x.detach().to("cpu")


def _oracle_prefix_state(inp, n, length):
    """Oracle final state of sequence n after its first `length` tokens."""
    cu = list(inp["cu_seqlens_host"])
    rows = slice(cu[n], cu[n] + length)
    q, k, v, g, beta = (_cpu(inp[name])[rows] for name in ("q", "k", "v", "g", "beta"))
    S0 = None if inp["S0"] is None else _cpu(inp["S0"])[n:n + 1]
    _, S = oracle.kda_fwd_ref(q, k, v, g, beta, S0=S0, scale=inp["scale"])
    return S[0]


def _check_all(inp, snaps, base, interval, tol):
    cu = list(inp["cu_seqlens_host"])
    count = 0
    for n in range(len(cu) - 1):
        L = cu[n + 1] - cu[n]
        assert int(base[n + 1] - base[n]) == L // interval
        for m in range(1, L // interval + 1):
            ref = _oracle_prefix_state(inp, n, m * interval)
            err = rel_max(snaps[int(base[n]) + m - 1], ref)
            assert err <= tol, (n, m, err)
            count += 1
    return count


@pytest.mark.parametrize("interval", [64, 192])
def test_snapshots_tensor_core_path(interval):
    lengths = [700, 64, 1300, 0, 129, 383]
    inp = inputs.prefill_inputs(lengths, H=2, dk=128, dv=128, device="cuda", seed=21, s0_std=0.02,
                                gate=True)
    o, S, snaps, base = chunk_fwd_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                            interval, S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
                                            cu_seqlens_host=inp["cu_seqlens_host"], gate=inp["gate"])
    assert _check_all(inp, snaps, base, interval, TOL_BF16) > 0
    # outputs and final states are those of the plain call
    o2, S2 = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                       cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"],
                       gate=inp["gate"])
    assert torch.equal(o, o2) and torch.equal(S, S2)
    assert device_status() == 0


def test_snapshots_cuda_core_path_fp32():
    lengths = [300, 128, 17]
    inp = inputs.prefill_inputs(lengths, H=2, dk=64, dv=64, dtype=torch.float32, device="cuda",
                                seed=22, s0_std=0.02)
    _, _, snaps, base = chunk_fwd_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], 64,
                                            S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
                                            cu_seqlens_host=inp["cu_seqlens_host"])
    assert _check_all(inp, snaps, base, 64, TOL_FP32) == 300 // 64 + 2
    assert device_status() == 0


def test_snapshots_with_the_segment_split():
    """A forced split of one long sequence: pass 2 runs the segments from
    their true incoming states, so its snapshots are the true states."""
    inp = inputs.prefill_inputs([1000], H=2, dk=128, dv=128, device="cuda", seed=23, s0_std=0.05)
    old = os.environ.get("KDA_SEGMENTS")
    os.environ["KDA_SEGMENTS"] = "4"
    try:
        _, S, snaps, base = chunk_fwd_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                                128, S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
                                                cu_seqlens_host=inp["cu_seqlens_host"])
    finally:
        if old is None:
            os.environ.pop("KDA_SEGMENTS", None)
        else:
            os.environ["KDA_SEGMENTS"] = old
    assert _check_all(inp, snaps, base, 128, TOL_BF16) == 1000 // 128
    assert device_status() == 0


def test_snapshots_full_size_config1():
    """8 x 4096 tokens x 32 heads, interval 512: the last snapshot of every
    sequence is its final state (bitwise: the same registers are stored), and
    the first snapshot of sequence 0 matches the oracle for two heads."""
    inp = inputs.prefill_inputs([4096] * 8, H=32, dk=128, dv=128, device="cuda", seed=0)
    _, S, snaps, base = chunk_fwd_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], 512,
                                            cu_seqlens=inp["cu_seqlens"],
                                            cu_seqlens_host=inp["cu_seqlens_host"])
    assert snaps.shape == (64, 32, 128, 128)
    for n in range(8):
        assert torch.equal(snaps[int(base[n + 1]) - 1], S[n])
    for h in (0, 31):
        prefix = [_cpu(inp[name][:512, h:h + 1]) for name in ("q", "k", "v", "g", "beta")]
        _, ref = oracle.kda_fwd_ref(*prefix, scale=inp["scale"])
        assert rel_max(snaps[0, h], ref[0, 0]) <= TOL_BF16
    assert device_status() == 0
