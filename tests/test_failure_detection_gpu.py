"""Failure detection without a GPU fault: every device-side wait in the
kernels is bounded; when one gives up it records a timeout in the device
error word and its kernel returns, leaving the context usable.  Here a
diagnostic entry point makes a wait run out on a barrier that nothing
completes (the same wait primitive the prefill uses) and the host reads the
status back."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import chunk_fwd, device_status, inputs, selftest_bounded_wait
from gated_delta_rule_136_b200.kda import STATUS_NAMES
from parity import TOL_BF16, rel_max, rel_max_beyond_bf16

pytestmark = pytest.mark.gpu

TIMEOUT = [k for k, v in STATUS_NAMES.items() if v == "KDA_ERR_TIMEOUT"][0]


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    assert device_status() == 0
    assert selftest_bounded_wait(256) == 0        # launched
    assert device_status() == TIMEOUT             # the wait gave up and said so
    assert device_status() == 0                   # reading cleared it
    # the context still runs the prefill correctly
    inp = inputs.prefill_inputs([150, 64], H=2, dk=128, dv=128, device="cuda", seed=13, s0_std=0.02)
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"])
    cpu = lambda t: t.detach().to("cpu")
    o_ref, S_ref = oracle.kda_fwd_ref(*(cpu(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                      cu_seqlens=np.array(inp["cu_seqlens_host"]), S0=cpu(inp["S0"]))
    assert rel_max_beyond_bf16(o, o_ref) <= TOL_BF16 and rel_max(S, S_ref) <= TOL_BF16
    assert device_status() == 0
