"""Prefill from and to host memory (kda_chunk_fwd_host): the same results as
the device-buffer prefill and the oracle, whatever the grouping of sequences
into pipeline stages, with page-locked or pageable host buffers."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import chunk_fwd, chunk_fwd_host, device_status, inputs
from parity import TOL_BF16, TOL_FP32, rel_max, rel_max_beyond_bf16

pytestmark = pytest.mark.gpu

LENGTHS = [300, 0, 70, 64, 129, 1, 500, 33, 250, 90, 12]      # 11 sequences: 8 pipeline groups


def _host(inp, names, pin):
    out = {}
    for n in names:
        t = None if inp[n] is None else inp[n].to("cpu")
        out[n] = t.pin_memory() if (pin and t is not None) else t
    return out


@pytest.mark.parametrize("pin", [True, False])
def test_host_prefill_matches_device_and_oracle(pin):
    inp = inputs.prefill_inputs(LENGTHS, H=2, dk=128, dv=128, device="cuda", seed=71, s0_std=0.05, gate=True)
    h = _host(inp, ("q", "k", "v", "g", "beta", "gate", "S0"), pin)
    o, S_T = chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], inp["cu_seqlens_host"], S0=h["S0"],
                            gate=h["gate"])
    assert device_status() == 0
    o_d, S_d = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                         cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"], gate=inp["gate"])
    o_ref, S_ref = oracle.kda_fwd_ref(h["q"], h["k"], h["v"], h["g"], h["beta"],
                                      cu_seqlens=np.array(inp["cu_seqlens_host"]), S0=h["S0"], gate=h["gate"])
    assert rel_max_beyond_bf16(o, o_ref) <= TOL_BF16 and rel_max(S_T, S_ref) <= TOL_BF16
    assert rel_max_beyond_bf16(o, o_d.cpu().double()) <= TOL_BF16 and rel_max(S_T, S_d) <= TOL_BF16


def test_host_prefill_fp32_single_sequence_and_repeat():
    """One sequence (one group), fp32 I/O; two calls back to back agree exactly."""
    inp = inputs.prefill_inputs([777], H=3, dk=64, dv=128, dtype=torch.float32, device="cuda", seed=73,
                                s0_std=0.05)
    h = _host(inp, ("q", "k", "v", "g", "beta", "S0"), True)
    o1, S1 = chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], inp["cu_seqlens_host"], S0=h["S0"])
    o2, S2 = chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], inp["cu_seqlens_host"], S0=h["S0"])
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    o_ref, S_ref = oracle.kda_fwd_ref(h["q"], h["k"], h["v"], h["g"], h["beta"], S0=h["S0"])
    assert rel_max(o1, o_ref) <= TOL_FP32 and rel_max(S1, S_ref) <= TOL_FP32
    assert device_status() == 0


def test_host_prefill_bench_shape_sampled():
    """The bench's e2e launch: 8 x 4096 tokens x 32 heads, bf16, S_T returned;
    two heads checked against the oracle."""
    inp = inputs.prefill_inputs([4096] * 8, H=32, device="cuda", seed=0)
    h = _host(inp, ("q", "k", "v", "g", "beta"), True)
    o, S_T = chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], inp["cu_seqlens_host"])
    assert device_status() == 0
    for n, hh in ((0, 0), (7, 31)):
        rows = slice(4096 * n, 4096 * (n + 1))
        o_ref, S_ref = oracle.kda_fwd_ref(*(h[x][rows, hh:hh + 1] for x in ("q", "k", "v", "g", "beta")))
        assert rel_max_beyond_bf16(o[rows, hh:hh + 1], o_ref) <= TOL_BF16
        assert rel_max(S_T[n:n + 1, hh:hh + 1], S_ref) <= TOL_BF16
