"""The debug variant of the library (-DKDA_DEBUG, loaded with
KDA_DEBUG_LIBRARY=1): its results match the oracle, and a unit whose token
range lies outside the launch (device cu_seqlens that disagree with the
host copy the call was validated with) is refused on the device --
KDA_ERR_DEVICE_BOUNDS in the error word, nothing touched -- by both prefill
kernels and both backward paths (chunked and per-token).  Run in a child
process, since a process loads one library."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
    import numpy as np, torch
    import oracle
    from gated_delta_rule_136_b200 import chunk_bwd, chunk_fwd, device_status, inputs, kda
    from parity import TOL_BF16, TOL_FP32, rel_max, rel_max_beyond_bf16
    assert kda.library_path().endswith("libkda_b200_debug.so")
    cpu = lambda t: None if t is None else t.detach().cpu()
    # 1. results of the debug build against the oracle (tensor-core and CUDA-core kernels)
    for dtype, tol in ((torch.bfloat16, TOL_BF16), (torch.float32, TOL_FP32)):
        inp = inputs.prefill_inputs([1, 17, 64, 0, 100, 257], H=2, dtype=dtype, device="cuda", seed=83,
                                    s0_std=0.02, gate=True)
        o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                         cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"], gate=inp["gate"])
        o_ref, S_ref = oracle.kda_fwd_ref(*(cpu(inp[n]) for n in ("q", "k", "v", "g", "beta")),
                                          cu_seqlens=np.array(inp["cu_seqlens_host"]), S0=cpu(inp["S0"]),
                                          scale=inp["scale"], gate=cpu(inp["gate"]))
        eo = rel_max_beyond_bf16(o, o_ref) if dtype == torch.bfloat16 else rel_max(o, o_ref)
        assert eo <= tol and rel_max(S, S_ref) <= tol, (dtype, eo)
        assert device_status() == 0
    # 2. device cu_seqlens past the tokens the call was validated for: refused on the device
    for dtype, H in ((torch.bfloat16, 80), (torch.float32, 2)):
        inp = inputs.prefill_inputs([300, 200], H=H, dtype=dtype, device="cuda", seed=89)
        bad = torch.tensor([0, 300, 564], dtype=torch.int32, device="cuda")   # 564 > 500 tokens
        chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu_seqlens=bad,
                  cu_seqlens_host=[0, 300, 500])
        st = device_status()
        assert st == 6, st          # KDA_ERR_DEVICE_BOUNDS
        assert device_status() == 0  # (the word is cleared by reading it)
    # 3. the backward of the debug build against the oracle (bf16: the chunked kernels)
    inp = inputs.prefill_inputs([150, 70], H=2, device="cuda", seed=91, s0_std=0.05, gate=True)
    gen = torch.Generator(device="cuda").manual_seed(92)
    dout = torch.randn(inp["v"].shape, generator=gen, device="cuda").to(torch.bfloat16)
    got = chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, cu_seqlens=inp["cu_seqlens"],
                    cu_seqlens_host=inp["cu_seqlens_host"], S0=inp["S0"], gate=inp["gate"])
    ref = oracle.kda_bwd_ref(*(cpu(inp[n]) for n in ("q", "k", "v", "g", "beta")), cpu(dout),
                             cu_seqlens=np.array(inp["cu_seqlens_host"]), S0=cpu(inp["S0"]), gate=cpu(inp["gate"]))
    for name, r in ref.items():
        e = rel_max_beyond_bf16(got[name], r) if name != "dS0" else rel_max(got[name], r)
        assert e <= TOL_BF16, (name, e)
    assert device_status() == 0
    # 4. the backward with device cu_seqlens past the validated tokens: refused on the device
    for dtype in (torch.bfloat16, torch.float32):      # the chunked and the per-token kernels
        inp = inputs.prefill_inputs([300, 200], H=2, dtype=dtype, device="cuda", seed=97)
        dout = torch.randn(inp["v"].shape, generator=gen, device="cuda").to(dtype)
        bad = torch.tensor([0, 300, 564], dtype=torch.int32, device="cuda")
        chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], dout, cu_seqlens=bad,
                  cu_seqlens_host=[0, 300, 500])
        st = device_status()
        assert st == 6, (dtype, st)
        assert device_status() == 0
    print("debug build ok")
""")


def test_debug_library_checks_units_on_the_device():
    env = dict(os.environ, KDA_DEBUG_LIBRARY="1")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout
