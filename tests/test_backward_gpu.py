"""Backward of the prefill (kda_chunk_bwd) against the oracle's fp64 gradients
(autograd through the token recurrence, itself pinned by finite differences):
dq, dk, dv, dg, dbeta, dgate and dS0 for L = sum(o * dout) + sum(S_T * dS_T).
Ragged sequences cover partial chunks and sub-blocks and an empty sequence;
fp32 I/O runs the CUDA-core forward for the checkpoints and the per-token
backward, bf16 I/O the tensor-core forward and (dk = dv = 128) the chunked
backward."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import chunk_bwd, device_status, inputs
from parity import TOL_BF16, TOL_FP32, rel_max, rel_max_beyond_bf16

pytestmark = pytest.mark.gpu


def _cpu(x):
    return None if x is None else x.detach().to("cpu")


def _run(lengths, H, dtype, seed, gate=True, s0=True, ds_t=True, heads=None, dk=128, dv=128, g_mode="softplus"):
    inp = inputs.prefill_inputs(lengths, H=H, dk=dk, dv=dv, dtype=dtype, device="cuda", seed=seed,
                                s0_std=0.05 if s0 else None, gate=gate, g_mode=g_mode)
    gen = torch.Generator(device="cuda").manual_seed(seed + 1)
    dout = torch.randn(inp["v"].shape, generator=gen, device="cuda").to(dtype)
    N = len(lengths)
    dS_T = (0.1 * torch.randn((N, H, dk, dv), generator=gen, device="cuda")) if ds_t else None
    got = chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout,
                    cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"], S0=inp["S0"],
                    gate=inp["gate"], dS_T=dS_T)
    assert device_status() == 0
    sel = (lambda t: t) if heads is None else (lambda t: None if t is None else t[:, heads].contiguous())
    ref = oracle.kda_bwd_ref(*(sel(_cpu(inp[n])) for n in ("q", "k", "v", "g", "beta")), sel(_cpu(dout)),
                             cu_seqlens=np.array(inp["cu_seqlens_host"]), S0=sel(_cpu(inp["S0"])),
                             gate=sel(_cpu(inp["gate"])), dS_T=sel(_cpu(dS_T)))
    return {n: sel(t) for n, t in got.items()}, ref


def _check(got, ref, dtype):
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dgate"):
        if name not in ref:
            continue
        if dtype == torch.float32:
            assert rel_max(got[name], ref[name]) <= TOL_FP32, name
        else:
            assert rel_max_beyond_bf16(got[name], ref[name]) <= TOL_BF16, name
    if "dS0" in ref:
        assert rel_max(got["dS0"], ref["dS0"]) <= (TOL_FP32 if dtype == torch.float32 else TOL_BF16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_matches_oracle(dtype):
    got, ref = _run([150, 0, 70, 64], H=2, dtype=dtype, seed=101)
    _check(got, ref, dtype)


@pytest.mark.parametrize("dk,dv,dtype", [(64, 64, torch.float32), (128, 64, torch.bfloat16),
                                         (64, 128, torch.float32)])
def test_backward_other_head_sizes(dk, dv, dtype):
    got, ref = _run([150, 70], H=2, dtype=dtype, seed=109, dk=dk, dv=dv)
    _check(got, ref, dtype)


def test_backward_without_gate_s0_or_final_gradient():
    got, ref = _run([97, 128], H=2, dtype=torch.float32, seed=103, gate=False, s0=False, ds_t=False)
    _check(got, ref, torch.float32)
    assert "dgate" not in got


def test_backward_full_length_sampled_head():
    """The bf16 workload's sequence length (4096) and head count; one head is
    checked against the oracle over the whole sequence."""
    got, ref = _run([4096], H=32, dtype=torch.bfloat16, seed=107, heads=[5])
    _check(got, ref, torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_floor_stress(dtype):
    """g spread down to and below the floor: the 16-token block factors of the
    chunked form reach e^{16 |floor|}, and clamped entries must pass no gradient."""
    got, ref = _run([200, 64, 33], H=2, dtype=dtype, seed=113, g_mode="floor_stress")
    _check(got, ref, dtype)


def test_backward_many_sequences():
    """Twelve sequences of lengths around the chunk and block sizes (empty, 1,
    one chunk exactly, one token past it, ...): the chunk tables, the chain
    over each sequence's chunks and the gradients at every sequence boundary."""
    lengths = [0, 1, 15, 16, 63, 64, 65, 127, 128, 129, 200, 7]
    got, ref = _run(lengths, H=2, dtype=torch.bfloat16, seed=127)
    _check(got, ref, torch.bfloat16)


def test_backward_bench_shape_sampled_units():
    """The bench's backward workload as launched (8 x 4096 tokens x 32 heads,
    bf16, no gate, S0 = 0, the bench's input recipe); two (sequence, head)
    units -- the first and the last of the launch -- against the oracle."""
    B, T, H = 8, 4096, 32
    inp = inputs.prefill_inputs([T] * B, H=H, device="cuda", seed=0)
    gen = torch.Generator(device="cuda").manual_seed(200)
    dout = torch.randn(inp["v"].shape, generator=gen, device="cuda").to(torch.bfloat16)
    got = chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, cu_seqlens=inp["cu_seqlens"],
                    cu_seqlens_host=inp["cu_seqlens_host"], want_dS0=False)
    assert device_status() == 0
    for n, h in ((0, 0), (B - 1, H - 1)):
        sl = slice(n * T, (n + 1) * T)
        part = lambda t: _cpu(t[sl, h:h + 1]).contiguous()
        ref = oracle.kda_bwd_ref(*(part(inp[x]) for x in ("q", "k", "v", "g", "beta")), part(dout),
                                 cu_seqlens=np.array([0, T]))
        mine = {name: got[name][sl, h:h + 1] for name in ref}
        _check(mine, ref, torch.bfloat16)
