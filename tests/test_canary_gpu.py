"""Canary-padded outputs: every output buffer sits inside a larger allocation
whose bytes before and after it hold a known pattern; after each call the
pattern must be intact, so no kernel writes outside the buffers it was given.
Covers the tensor-core prefill (ragged, gated, with S0; the long-sequence
segment split), the CUDA-core prefill (fp32), decode and speculative
verify/commit."""
import pytest
import torch

from gated_delta_rule_136_b200 import (chunk_fwd, chunk_fwd_snapshots, decode_step, device_status,
                                       inputs, spec_commit, spec_verify)

pytestmark = pytest.mark.gpu

PAD = 1 << 16          # bytes of canary on each side (16-byte multiple keeps alignment)
PATTERN = 0xA5


def padded(shape, dtype):
    """A tensor of `shape` inside a byte buffer with PAD canary bytes on each side."""
    n = torch.Size(shape).numel() * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((PAD + n + PAD,), PATTERN, dtype=torch.uint8, device="cuda")
    view = raw[PAD:PAD + n].view(dtype).view(shape)
    return raw, view


def intact(raw):
    torch.cuda.synchronize()
    return bool((raw[:PAD] == PATTERN).all()) and bool((raw[-PAD:] == PATTERN).all())


@pytest.mark.parametrize("case", ["ragged_gate_s0", "split", "fp32"])
def test_prefill_writes_stay_in_bounds(case):
    if case == "ragged_gate_s0":
        lengths, H, dtype, kw = [1, 17, 64, 0, 100, 257, 15], 3, torch.bfloat16, dict(s0_std=0.02, gate=True)
    elif case == "split":
        lengths, H, dtype, kw = [4096], 8, torch.bfloat16, dict(s0_std=0.02)     # few units: segment split
    else:
        lengths, H, dtype, kw = [70, 130], 2, torch.float32, dict(s0_std=0.02, gate=True)
    inp = inputs.prefill_inputs(lengths, H=H, dk=128, dv=128, dtype=dtype, device="cuda", seed=61, **kw)
    T, N = inp["q"].shape[0], len(lengths)
    ro, o = padded((T, H, 128), dtype)
    rs, S = padded((N, H, 128, 128), torch.float32)
    chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
              cu_seqlens_host=inp["cu_seqlens_host"], gate=inp["gate"], out=o, final_state_out=S)
    assert intact(ro) and intact(rs)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    assert device_status() == 0


def test_prefill_after_snapshot_call_stays_in_bounds():
    """A forward with snapshots every 64 tokens, then the plain forward on the
    same inputs with its outputs inside canaries."""
    inp = inputs.prefill_inputs([1024, 300], H=4, dk=128, dv=128, device="cuda", seed=67, s0_std=0.02)
    chunk_fwd_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], 64, S0=inp["S0"],
                        cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"])
    assert device_status() == 0
    T = inp["q"].shape[0]
    ro, o2 = padded((T, 4, 128), torch.bfloat16)
    rs, S2 = padded((2, 4, 128, 128), torch.float32)
    chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
              cu_seqlens_host=inp["cu_seqlens_host"], out=o2, final_state_out=S2)
    assert intact(ro) and intact(rs)
    assert device_status() == 0


def test_decode_and_speculative_writes_stay_in_bounds():
    d = inputs.decode_inputs(batch=16, H=4, dk=128, dv=128, steps=1, device="cuda", seed=71)
    rS, S = padded((16, 4, 128, 128), torch.float32)
    S.copy_(d["S"])
    ro, o = padded((16, 4, 128), torch.bfloat16)
    decode_step(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0], S, gate=d["gate"][0], out=o)
    assert intact(rS) and intact(ro)
    D = 4
    sd = inputs.prefill_inputs([D] * 16, H=4, dk=128, dv=128, device="cuda", seed=73, s0_std=0.02, gate=True)
    xs = {n: sd[n].view(16, D, *sd[n].shape[1:]) for n in ("q", "k", "v", "g", "beta", "gate")}
    rSs, Ss = padded((16, 4, 128, 128), torch.float32)
    Ss.copy_(sd["S0"])
    rov, ov = padded((16, D, 4, 128), torch.bfloat16)
    spec_verify(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], Ss, gate=xs["gate"], out=ov)
    acc = torch.tensor([0, 1, 2, 3, 4] * 3 + [2], dtype=torch.int32, device="cuda")
    spec_commit(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], Ss, acc)
    assert intact(rSs) and intact(rov)
    assert device_status() == 0
