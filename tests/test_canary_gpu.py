"""Canary-padded outputs: every output buffer sits inside a larger allocation
whose bytes before and after it hold a known pattern; after each call the
pattern must be intact, so no kernel writes outside the buffers it was given.
Covers the tensor-core prefill (ragged, gated, with S0; the long-sequence
segment split), the CUDA-core prefill (fp32), decode, speculative
verify/commit and the backward (chunked and per-token)."""
import ctypes

import pytest
import torch

from gated_delta_rule_136_b200 import (chunk_bwd, chunk_fwd, chunk_fwd_snapshots, decode_step, device_status,
                                       inputs, kda, spec_commit, spec_verify)

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


@pytest.mark.parametrize("dk,dtype", [(128, torch.bfloat16), (128, torch.float32), (64, torch.float32)])
def test_backward_writes_stay_in_bounds(dk, dtype):
    """kda_chunk_bwd through the C ABI with every gradient inside canaries (dk = dv = 128:
    the chunked kernels; 64: the per-token kernel); the gradients equal the wrapper's."""
    lengths, H = [150, 0, 70, 64], 2
    inp = inputs.prefill_inputs(lengths, H=H, dk=dk, dv=dk, dtype=dtype, device="cuda", seed=71,
                                s0_std=0.05, gate=True)
    gen = torch.Generator(device="cuda").manual_seed(72)
    dout = torch.randn(inp["v"].shape, generator=gen, device="cuda").to(dtype)
    N, T = len(lengths), inp["q"].shape[0]
    dS_T = 0.1 * torch.randn((N, H, dk, dk), generator=gen, device="cuda")
    ref = chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, cu_seqlens=inp["cu_seqlens"],
                    cu_seqlens_host=inp["cu_seqlens_host"], S0=inp["S0"], gate=inp["gate"], dS_T=dS_T)
    shapes = {"dq": (T, H, dk), "dk": (T, H, dk), "dv": (T, H, dk), "dg": (T, H, dk), "dbeta": (T, H),
              "dgate": (T, H, dk)}
    raws, outs = {}, {}
    for name, shape in shapes.items():
        raws[name], outs[name] = padded(shape, dtype)
    raws["dS0"], outs["dS0"] = padded((N, H, dk, dk), torch.float32)
    lib = kda.load_library()
    desc = kda.FwdDesc(T, N, H, dk, dk, kda.KDA_BF16 if dtype == torch.bfloat16 else kda.KDA_FP32,
                       float(inp["scale"]), -5.0, 0, 0)
    cu_h = (ctypes.c_int32 * (N + 1))(*inp["cu_seqlens_host"])
    ws_bytes = lib.kda_chunk_bwd_workspace_size(ctypes.byref(desc), cu_h)
    ws = torch.empty(int(ws_bytes), dtype=torch.uint8, device="cuda")
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib.kda_chunk_bwd(ctypes.byref(desc), vp(inp["q"]), vp(inp["k"]), vp(inp["v"]), vp(inp["g"]),
                           vp(inp["beta"]), vp(inp["S0"]),
                           ctypes.cast(vp(inp["cu_seqlens"]), ctypes.POINTER(ctypes.c_int32)), cu_h,
                           vp(inp["gate"]), vp(dout), vp(dS_T), vp(outs["dq"]), vp(outs["dk"]), vp(outs["dv"]),
                           vp(outs["dg"]), vp(outs["dbeta"]), vp(outs["dgate"]), vp(outs["dS0"]), vp(ws),
                           ctypes.c_size_t(ws.numel()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    for name in outs:
        assert intact(raws[name]), name
        assert torch.equal(outs[name], ref[name]), name
    assert device_status() == 0
