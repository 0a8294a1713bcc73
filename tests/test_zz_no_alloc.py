"""kda_chunk_fwd_noalloc, called through the C ABI, against the fp64 oracle
and against kda_chunk_fwd.

This entry point serves callers that cannot give the library any device
memory (a plugin interface that passes only inputs and outputs, a runtime
that plans all device memory in advance and forbids allocating once it
runs): its scratch is a fixed array compiled into the library.  The test
makes two calls in a row with different shapes, so the second one runs on
scratch the first one left behind, and compares each result with the oracle
and with the workspace-taking entry point within the parity tolerances; a
third call goes through the Python wrapper with caller-provided outputs.  It is meant to
pass on its own in a fresh process (where its first call also performs the
per-device set-up) and after every other test.  This file is named so that
pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import chunk_fwd, device_status, inputs, kda
from parity import TOL_BF16, rel_max, rel_max_beyond_bf16


def _oracle(inp):
    cpu = lambda t: None if t is None else t.detach().cpu()
    return oracle.kda_fwd_ref(*(cpu(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                              cu_seqlens=np.array(inp["cu_seqlens_host"], dtype=np.int64),
                              S0=cpu(inp["S0"]), scale=inp["scale"], gate=cpu(inp["gate"]))


def _call_noalloc(lib, inp, o, S_T):
    q = inp["q"]
    T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    N = len(inp["lengths"])
    desc = kda.FwdDesc(T, N, H, dk, dv, kda.KDA_BF16, float(inp["scale"]), -5.0, 0, 0)
    f = lib.kda_chunk_fwd_noalloc
    vp = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(kda.FwdDesc), vp, vp, vp, vp, vp, vp,
                  ctypes.POINTER(ctypes.c_int32), vp, vp, vp, vp]
    f.restype = ctypes.c_int
    ptr = lambda t: None if t is None else vp(t.data_ptr())
    cu = ctypes.cast(vp(inp["cu_seqlens"].data_ptr()), ctypes.POINTER(ctypes.c_int32))
    stream = vp(torch.cuda.current_stream().cuda_stream)
    return f(ctypes.byref(desc), ptr(inp["q"]), ptr(inp["k"]), ptr(inp["v"]), ptr(inp["g"]),
             ptr(inp["beta"]), ptr(inp["S0"]), cu, ptr(inp["gate"]), ptr(o), ptr(S_T), stream)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    lib = kda.load_library()
    cases = [
        dict(lengths=[300, 17, 64, 1, 129], H=4, seed=31, gate=True),
        dict(lengths=[40, 500, 3], H=2, seed=37, gate=False),   # fewer sequences: stale scratch
    ]
    for c in cases:
        inp = inputs.prefill_inputs(c["lengths"], H=c["H"], dk=128, dv=128, device="cuda",
                                    seed=c["seed"], s0_std=0.02, gate=c["gate"])
        T, H = inp["q"].shape[:2]
        N = len(c["lengths"])
        o = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
        S_T = torch.empty((N, H, 128, 128), dtype=torch.float32, device="cuda")
        assert _call_noalloc(lib, inp, o, S_T) == 0
        o_ws, S_ws = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                               S0=inp["S0"], cu_seqlens=inp["cu_seqlens"],
                               cu_seqlens_host=inp["cu_seqlens_host"], gate=inp["gate"])
        torch.cuda.synchronize()
        o_ref, S_ref = _oracle(inp)
        assert rel_max_beyond_bf16(o, o_ref) <= TOL_BF16
        assert rel_max(S_T, S_ref) <= TOL_BF16
        assert rel_max_beyond_bf16(o, o_ws) <= TOL_BF16
        assert rel_max(S_T, S_ws) <= TOL_BF16
    assert device_status() == 0


@pytest.mark.gpu
def test_noalloc_python_wrapper_with_caller_outputs():
    """kda.chunk_fwd_noalloc with out= and final_state_out=: the results land in
    the caller's tensors and match the oracle."""
    inp = inputs.prefill_inputs([200, 64, 7, 333], H=3, dk=128, dv=128, device="cuda", seed=41,
                                s0_std=0.02, gate=True)
    T, H = inp["q"].shape[:2]
    o = torch.full((T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S_T = torch.full((4, H, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
    o2, S2 = kda.chunk_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                   inp["cu_seqlens"], S0=inp["S0"], gate=inp["gate"],
                                   out=o, final_state_out=S_T)
    assert o2 is o and S2 is S_T
    torch.cuda.synchronize()
    o_ref, S_ref = _oracle(inp)
    assert rel_max_beyond_bf16(o, o_ref) <= TOL_BF16
    assert rel_max(S_T, S_ref) <= TOL_BF16
    assert device_status() == 0


def test_noalloc_rejects_too_many_sequences():
    """Host-side check only (runs without a GPU): nothing is launched."""
    lib = kda.load_library()
    N = kda.NOALLOC_MAX_SEQS + 1
    desc = kda.FwdDesc(N, N, 1, 128, 128, kda.KDA_BF16, 0.088, -5.0, 0, 0)
    f = lib.kda_chunk_fwd_noalloc
    vp = ctypes.c_void_p
    f.argtypes = [ctypes.POINTER(kda.FwdDesc), vp, vp, vp, vp, vp, vp,
                  ctypes.POINTER(ctypes.c_int32), vp, vp, vp, vp]
    f.restype = ctypes.c_int
    # rejected on the host before any pointer is touched or anything launched
    fake = vp(0x10000000)
    st = f(ctypes.byref(desc), fake, fake, fake, fake, fake, None,
           ctypes.cast(fake, ctypes.POINTER(ctypes.c_int32)), None, fake, None, None)
    assert st == 3   # KDA_ERR_WORKSPACE
