"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs, plus invariants that hold at any size.

Tolerances: bf16 I/O -- S_T max|d|/RMS <= 2e-2; o the same bound beyond its
own bf16 storage half-ulp (see tests/parity.py).  fp32 I/O -- 1e-4 plain.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_136_b200 import chunk_fwd, decode_step, device_status, inputs
from parity import TOL_BF16, TOL_FP32, bf16_half_ulp, rel_max, rel_max_beyond_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cpu(x):
    return None if x is None else x.detach().to("cpu")


def _oracle_prefill(inp, heads=None, seqs=None, g_floor=-5.0):
    """Oracle on a subset of heads / sequences (units are independent).  The
    heads are selected on the device, so only their slices reach the host."""
    def pick(name):
        t = inp[name]
        if t is None:
            return None
        if heads is not None:   # dim 1 is the head for every input, S0 included
            t = t.index_select(1, torch.tensor(heads, device=t.device))
        return _cpu(t)
    q, k, v, g, beta, gate, S0 = (pick(n) for n in ("q", "k", "v", "g", "beta", "gate", "S0"))
    cu = list(inp["cu_seqlens_host"])
    if seqs is not None:
        rows = torch.cat([torch.arange(cu[n], cu[n + 1]) for n in seqs])
        newcu = [0]
        for n in seqs:
            newcu.append(newcu[-1] + cu[n + 1] - cu[n])
        q, k, v, g, beta = (t[rows] for t in (q, k, v, g, beta))
        gate = None if gate is None else gate[rows]
        S0 = None if S0 is None else S0[list(seqs)]
        cu = newcu
    return oracle.kda_fwd_ref(q, k, v, g, beta, cu_seqlens=np.array(cu, dtype=np.int64), S0=S0,
                              scale=inp["scale"], gate=gate, g_floor=g_floor)


def _all_finite(t, rows_per_slab=1 << 16):
    """Finite check without materialising a full-size temporary."""
    flat = t.reshape(t.shape[0], -1) if t.dim() > 1 else t.reshape(-1, 1)
    return all(bool(torch.isfinite(flat[i:i + rows_per_slab]).all())
               for i in range(0, flat.shape[0], rows_per_slab))


def _assert_close(o, S, o_ref, S_ref, dtype, what=""):
    assert torch.isfinite(o.float()).all(), f"{what}: non-finite o"
    if S is not None:
        assert torch.isfinite(S).all(), f"{what}: non-finite S_T"
    if dtype == torch.float32:
        eo, es = rel_max(o, o_ref), (rel_max(S, S_ref) if S is not None else 0.0)
        assert eo <= TOL_FP32 and es <= TOL_FP32, f"{what}: o {eo:.2e} S {es:.2e}"
    else:
        eo, es = rel_max_beyond_bf16(o, o_ref), (rel_max(S, S_ref) if S is not None else 0.0)
        assert eo <= TOL_BF16 and es <= TOL_BF16, f"{what}: o {eo:.2e} S {es:.2e}"
    return eo, es


def test_config0_fp32_chunk16():
    """fp32, B=1, H=2, T=256, dk=dv=64, chunk 16, S0 = 0: bound 1e-4."""
    inp = inputs.prefill_inputs([256], H=2, dk=64, dv=64, dtype=torch.float32, device=DEV, seed=0)
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"],
                     chunk=16)
    o_ref, S_ref = _oracle_prefill(inp)
    _assert_close(o, S, o_ref, S_ref, torch.float32, "config 0")


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("chunk", [0, 16])
def test_varlen_ragged_gate_s0(dk, dv, dtype, chunk):
    lengths = [1, 17, 64, 0, 100, 257, 15]
    inp = inputs.prefill_inputs(lengths, H=3, dk=dk, dv=dv, dtype=dtype, device=DEV, seed=3,
                                s0_std=0.02, gate=True)
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"],
                     gate=inp["gate"], chunk=chunk)
    o_ref, S_ref = _oracle_prefill(inp)
    _assert_close(o, S, o_ref, S_ref, dtype, f"varlen {dk}x{dv} {dtype} chunk {chunk}")
    # the empty sequence keeps its initial state exactly
    assert torch.equal(S[3], inp["S0"][3])


def test_floor_stress_bf16():
    """Decay drawn near the floor (g ~ -5 U(0.8,1)) with some values below it."""
    inp = inputs.prefill_inputs([300, 77], H=2, dk=128, dv=128, device=DEV, seed=5,
                                g_mode="floor_stress", s0_std=0.02)
    inp["g"][:, 0, :7] = -9.0   # below the floor: acts as the floor
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"])
    o_ref, S_ref = _oracle_prefill(inp)
    _assert_close(o, S, o_ref, S_ref, torch.bfloat16, "floor stress")


@pytest.mark.parametrize("g_floor", [-4.7, -5.45, -0.3])
def test_floor_not_a_bf16_value(g_floor):
    """A floor that bf16 cannot represent: the tensor-core prefill clamps with
    the nearest bf16 below it and adds the exact remainder for every clamped
    token, so the result must still match max(g, floor) in the oracle.  At
    -0.3 every token is clamped; at -5.45 (the lowest floor) a third are."""
    assert float(torch.tensor(g_floor, dtype=torch.bfloat16)) != float(np.float32(g_floor))
    inp = inputs.prefill_inputs([300, 77], H=2, dk=128, dv=128, device=DEV, seed=7,
                                g_mode="floor_stress", s0_std=0.02, gate=True)
    inp["g"][::3] = -6.0
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"],
                     gate=inp["gate"], g_floor=g_floor)
    o_ref, S_ref = _oracle_prefill(inp, g_floor=g_floor)
    _assert_close(o, S, o_ref, S_ref, torch.bfloat16, f"floor {g_floor}")
    assert device_status() == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_decode_against_oracle(dtype, dk, dv):
    d = inputs.decode_inputs(batch=16, H=4, dk=dk, dv=dv, steps=3, dtype=dtype, device=DEV, seed=7)
    S = d["S"].clone()
    S_ref = _cpu(d["S"]).double().numpy()
    for t in range(3):
        o = decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S, gate=d["gate"][t])
        o_ref, S_ref = oracle.kda_decode_ref(_cpu(d["q"][t]), _cpu(d["k"][t]), _cpu(d["v"][t]),
                                             _cpu(d["g"][t]), _cpu(d["beta"][t]), S_ref,
                                             gate=_cpu(d["gate"][t]))
        _assert_close(o, S, o_ref, S_ref, dtype, f"decode step {t}")


def test_decode_steps_equal_prefill_fp32():
    """T decode steps from S0 give the prefill of the same T tokens."""
    B, H, T, d = 4, 2, 40, 128
    inp = inputs.prefill_inputs([T] * B, H=H, dk=d, dv=d, dtype=torch.float32, device=DEV,
                                seed=11, s0_std=0.05, gate=True)
    o_p, S_p = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                         cu_seqlens=inp["cu_seqlens"], gate=inp["gate"])
    S = inp["S0"].clone()
    resh = lambda x: x.view(B, T, *x.shape[1:])
    q, k, v, g, beta, z = (resh(inp[n]) for n in ("q", "k", "v", "g", "beta", "gate"))
    outs = []
    for t in range(T):
        outs.append(decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                                g[:, t].contiguous(), beta[:, t].contiguous(), S,
                                gate=z[:, t].contiguous()))
    o_d = torch.stack(outs, 1).reshape(B * T, H, d)
    assert rel_max(o_d, o_p) <= TOL_FP32 and rel_max(S, S_p) <= TOL_FP32


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_split_invariance(dtype):
    """prefill(T1) then prefill(T2) from its final state == prefill(T1 + T2):
    the state is the whole checkpoint (the segment decomposition of context
    parallelism, fupanwang.com digest, section 基础设施)."""
    T1, T2 = 130, 190
    inp = inputs.prefill_inputs([T1 + T2], H=2, dk=128, dv=128, dtype=dtype, device=DEV, seed=13,
                                s0_std=0.02)
    full_o, full_S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"])
    sl = lambda a, b: [inp[n][a:b].contiguous() for n in ("q", "k", "v", "g", "beta")]
    o1, S1 = chunk_fwd(*sl(0, T1), S0=inp["S0"])
    o2, S2 = chunk_fwd(*sl(T1, T1 + T2), S0=S1)
    o_split = torch.cat([o1, o2])
    if dtype == torch.float32:
        assert rel_max(o_split, full_o) <= TOL_FP32 and rel_max(S2, full_S) <= TOL_FP32
    else:   # different chunk boundaries round differently: the bf16 bar applies
        assert rel_max_beyond_bf16(o_split, full_o) <= TOL_BF16
        assert rel_max(S2, full_S) <= TOL_BF16


def test_packing_is_bitwise_invariant():
    """Packed varlen results equal separate runs exactly (units are independent)."""
    lengths = [33, 200, 5]
    inp = inputs.prefill_inputs(lengths, H=2, dk=128, dv=128, device=DEV, seed=17, s0_std=0.02,
                                gate=True)
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                     cu_seqlens=inp["cu_seqlens"], gate=inp["gate"])
    cu = inp["cu_seqlens_host"]
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        on, Sn = chunk_fwd(*[inp[x][a:b].contiguous() for x in ("q", "k", "v", "g", "beta")],
                           S0=inp["S0"][n:n + 1].contiguous(), gate=inp["gate"][a:b].contiguous())
        assert torch.equal(on, o[a:b]) and torch.equal(Sn[0], S[n])


def test_linearity_in_v_and_S0_fp32():
    T, H, d = 150, 2, 64
    a = inputs.prefill_inputs([T], H=H, dk=d, dv=d, dtype=torch.float32, device=DEV, seed=19,
                              s0_std=0.1)
    b = inputs.prefill_inputs([T], H=H, dk=d, dv=d, dtype=torch.float32, device=DEV, seed=23,
                              s0_std=0.1)
    base = [a[n] for n in ("q", "k")]
    run = lambda v, S0: chunk_fwd(base[0], base[1], v, a["g"], a["beta"], S0=S0)
    o1, S1 = run(a["v"], a["S0"])
    o2, S2 = run(b["v"], b["S0"])
    o3, S3 = run(a["v"] + b["v"], a["S0"] + b["S0"])
    assert rel_max(o3, o1 + o2) <= TOL_FP32 and rel_max(S3, S1 + S2) <= TOL_FP32


def _unit_errors(o, S, o_ref, S_ref, cu, heads):
    """Parity of a full-size output, and its per-(sequence, head) breakdown.

    The stated metric is taken over the whole compared output: o (bf16) --
    max over all compared elements of |d| beyond half a bf16 ulp, divided by
    the RMS of all compared reference values; S_T (fp32) likewise, plain.
    The per-unit figures (each unit's max over that unit's own RMS) are
    returned for the report.  ``o``/``S`` hold the CUDA results for ``heads``
    (in that order), ``o_ref``/``S_ref`` the oracle's."""
    o = o.detach().to("cpu", torch.float64).numpy()
    S = S.detach().to("cpu", torch.float64).numpy()
    units = {}
    dmax_o = dmax_s = 0.0
    ss_o = ss_s = 0.0
    cnt_o = cnt_s = 0
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        for j, h in enumerate(heads):
            r, x = o_ref[a:b, j], o[a:b, j]
            rs, xs = S_ref[n, j], S[n, j]
            do = float(np.max(np.maximum(np.abs(x - r) - bf16_half_ulp(r), 0.0))) if r.size else 0.0
            ds = float(np.max(np.abs(xs - rs)))
            so, sst = float(np.sum(r * r)), float(np.sum(rs * rs))
            dmax_o, dmax_s = max(dmax_o, do), max(dmax_s, ds)
            ss_o, ss_s, cnt_o, cnt_s = ss_o + so, ss_s + sst, cnt_o + r.size, cnt_s + rs.size
            units[(n, h)] = (do / np.sqrt(so / r.size) if r.size and so > 0 else do,
                             ds / np.sqrt(sst / rs.size) if sst > 0 else ds)
    whole = (dmax_o / np.sqrt(ss_o / cnt_o), dmax_s / np.sqrt(ss_s / cnt_s))
    return whole, units


def _check_units(res, what):
    (eo, es), units = res
    worst_o = max(units.items(), key=lambda kv: kv[1][0])
    worst_s = max(units.items(), key=lambda kv: kv[1][1])
    print(f"{what}: {len(units)} units; whole output o {eo:.3e}, S_T {es:.3e}; per unit: "
          f"worst o {worst_o[1][0]:.3e} at {worst_o[0]}, worst S_T {worst_s[1][1]:.3e} at {worst_s[0]}")
    assert eo <= TOL_BF16 and es <= TOL_BF16, f"{what}: o {eo:.3e}, S_T {es:.3e}"


def test_config1_full_size_all_units():
    """B=8, H=32, T=4096, dk=dv=128, bf16 in the bench's launch: all 256
    (sequence, head) units against the oracle, each unit's error on its own."""
    inp = inputs.prefill_inputs([4096] * 8, H=32, dk=128, dv=128, device=DEV, seed=0)
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"])
    assert device_status() == 0
    o_ref, S_ref = _oracle_prefill(inp)
    _check_units(_unit_errors(o, S, o_ref, S_ref, list(inp["cu_seqlens_host"]), list(range(32))),
                 "config 1")


def test_config2_varlen_full_size_all_sequences_four_heads():
    """64 packed sequences with lengths uniform in [512, 32768], H=64,
    dk=dv=128, bf16, S0 ~ N(0, 0.02): all 64 sequences on 4 seeded heads
    against the oracle, each (sequence, head) error on its own; every output
    checked finite."""
    lengths = inputs.varlen_lengths(64, 512, 32768, seed=0)
    inp = inputs.prefill_inputs(lengths, H=64, dk=128, dv=128, device=DEV, seed=0, s0_std=0.02)
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S0=inp["S0"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"])
    assert _all_finite(o) and _all_finite(S)
    assert device_status() == 0
    heads = sorted(int(h) for h in np.random.default_rng(2).choice(64, size=4, replace=False))
    o_ref, S_ref = _oracle_prefill(inp, heads=heads)
    hsel = torch.tensor(heads, device=o.device)
    _check_units(_unit_errors(o.index_select(1, hsel), S.index_select(1, hsel), o_ref, S_ref,
                              list(inp["cu_seqlens_host"]), heads), "config 2")


def test_config3_long_context_full_size_four_heads():
    """B=1, H=32, T=2^20, dk=dv=128, bf16, decay near the floor
    (g ~ -5 U(0.8, 1)): 4 seeded heads checked in full (1M tokens each);
    every output checked finite."""
    inp = inputs.prefill_inputs([1 << 20], H=32, dk=128, dv=128, device=DEV, seed=0,
                                g_mode="floor_stress")
    o, S = chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                     cu_seqlens=inp["cu_seqlens"], cu_seqlens_host=inp["cu_seqlens_host"])
    assert _all_finite(o) and _all_finite(S)
    assert device_status() == 0
    heads = sorted(int(h) for h in np.random.default_rng(3).choice(32, size=4, replace=False))
    o_ref, S_ref = _oracle_prefill(inp, heads=heads)
    hsel = torch.tensor(heads, device=o.device)
    _check_units(_unit_errors(o.index_select(1, hsel), S.index_select(1, hsel), o_ref, S_ref,
                              list(inp["cu_seqlens_host"]), heads), "config 3")


def test_config4_decode_full_batch_all_units():
    """512 sequences x 64 heads, 128x128 fp32 state per head, bf16 inputs,
    sigmoid gate: three consecutive steps, every unit against the oracle."""
    d = inputs.decode_inputs(batch=512, H=64, dk=128, dv=128, steps=3, device=DEV, seed=0)
    S = d["S"].clone()
    S_ref = _cpu(d["S"]).double().numpy()
    for t in range(3):
        o = decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S, gate=d["gate"][t])
        o_ref, S_ref = oracle.kda_decode_ref(*(_cpu(d[n][t]) for n in ("q", "k", "v", "g", "beta")),
                                             S_ref, gate=_cpu(d["gate"][t]))
        _assert_close(o, S, o_ref, S_ref, torch.bfloat16, f"config 4 step {t}")
