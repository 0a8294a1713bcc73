"""Seeded synthetic inputs for the KDA forward workloads.

This module only draws random tensors (torch RNG on CPU or GPU) with the
distributions of the workloads; it holds none of the method's arithmetic and
is the one module shared by the tests, the bench and the oracle checks.

Every tensor has its own generator, seeded ``seed + index`` with the index in
the fixed order q, k, v, g, beta, S0, z (gate logits), lengths, so a tensor's
values do not depend on which other tensors were drawn.

Distributions (per (token, head) rows):
  q, k  ~ N(0,1), then L2-normalised over dk;   v ~ N(0,1)
  beta  = sigmoid(N(0,1))
  g     = max(-5, -softplus(N(0,1)))  ("softplus" mode)
        = -5 * U(0.8, 1)              ("floor_stress" mode: decay near the floor)
  S0    ~ N(0, s0_std)                (fp32, optional)
  z     ~ N(0,1)                      (gate logits, optional)
Large tensors are drawn in fixed-size slabs so device memory stays bounded.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F

_IDX = {"q": 0, "k": 1, "v": 2, "g": 3, "beta": 4, "S0": 5, "z": 6, "lengths": 7}
_SLAB_ELEMS = 1 << 26   # fp32 elements per drawing slab (256 MiB)


def _gen(device, seed: int, name: str) -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) * 1000 + _IDX[name])
    return gen


def _fill_rows(out: torch.Tensor, gen: torch.Generator, kind: str) -> torch.Tensor:
    """Fill ``out`` ([rows, ..., d], any float dtype) slab by slab."""
    d = out.shape[-1]
    flat = out.view(-1, d)
    rows_per_slab = max(1, _SLAB_ELEMS // d)
    for r0 in range(0, flat.shape[0], rows_per_slab):
        r1 = min(flat.shape[0], r0 + rows_per_slab)
        x = torch.empty((r1 - r0, d), device=out.device, dtype=torch.float32)
        if kind == "uniform_floor":
            x.uniform_(0.8, 1.0, generator=gen)
            x.mul_(-5.0)
        else:
            x.normal_(0.0, 1.0, generator=gen)
        if kind == "unit":
            x = F.normalize(x, p=2.0, dim=-1)
        elif kind == "softplus_decay":
            x = torch.clamp(-F.softplus(x), min=-5.0)
        elif kind == "sigmoid":
            x = torch.sigmoid(x)
        flat[r0:r1].copy_(x)
    return out


def prefill_inputs(lengths, H: int, dk: int = 128, dv: int = 128,
                   dtype=torch.bfloat16, device="cpu", seed: int = 0,
                   g_mode: str = "softplus", s0_std: float | None = None,
                   gate: bool = False) -> dict:
    """Packed variable-length prefill inputs.

    ``lengths``: list of per-sequence token counts.  Returns a dict with
    q,k,g [T,H,dk], v [T,H,dv], beta [T,H] (``dtype``), ``cu_seqlens`` int32
    [N+1] on ``device``, ``cu_seqlens_host`` (python list), S0 fp32
    [N,H,dk,dv] or None, gate [T,H,dv] or None, and ``scale`` = 1/sqrt(dk).
    """
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    N = len(lengths)
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    dev = torch.device(device)
    mk = lambda d: torch.empty((T, H, d), device=dev, dtype=dtype)
    out = {
        "q": _fill_rows(mk(dk), _gen(dev, seed, "q"), "unit"),
        "k": _fill_rows(mk(dk), _gen(dev, seed, "k"), "unit"),
        "v": _fill_rows(mk(dv), _gen(dev, seed, "v"), "normal"),
        "g": _fill_rows(mk(dk), _gen(dev, seed, "g"),
                        "uniform_floor" if g_mode == "floor_stress" else "softplus_decay"),
        "beta": _fill_rows(torch.empty((T, H), device=dev, dtype=dtype),
                           _gen(dev, seed, "beta"), "sigmoid"),
    }
    if s0_std is not None:
        S0 = torch.empty((N, H, dk, dv), device=dev, dtype=torch.float32)
        _fill_rows(S0, _gen(dev, seed, "S0"), "normal")
        out["S0"] = S0.mul_(s0_std)
    else:
        out["S0"] = None
    out["gate"] = (_fill_rows(mk(dv), _gen(dev, seed, "z"), "normal") if gate else None)
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=dev)
    out["cu_seqlens_host"] = cu
    out["scale"] = 1.0 / math.sqrt(dk)
    out["lengths"] = lengths
    return out


def varlen_lengths(num_seqs: int, lo: int, hi: int, seed: int = 0):
    """Integer lengths drawn uniformly in [lo, hi] (CPU generator)."""
    gen = _gen("cpu", seed, "lengths")
    return [int(x) for x in torch.randint(lo, hi + 1, (num_seqs,), generator=gen)]


def decode_inputs(batch: int, H: int, dk: int = 128, dv: int = 128, steps: int = 1,
                  dtype=torch.bfloat16, device="cpu", seed: int = 0,
                  s_std: float = 0.02, gate: bool = True) -> dict:
    """Inputs for ``steps`` consecutive decode steps.

    q,k,g [steps,batch,H,dk], v [steps,batch,H,dv], beta [steps,batch,H]
    (``dtype``), gate logits z [steps,batch,H,dv] or None, and the initial
    state S [batch,H,dk,dv] fp32 ~ N(0, s_std).
    """
    dev = torch.device(device)
    mk = lambda d: torch.empty((steps, batch, H, d), device=dev, dtype=dtype)
    S = torch.empty((batch, H, dk, dv), device=dev, dtype=torch.float32)
    _fill_rows(S, _gen(dev, seed, "S0"), "normal").mul_(s_std)
    return {
        "q": _fill_rows(mk(dk), _gen(dev, seed, "q"), "unit"),
        "k": _fill_rows(mk(dk), _gen(dev, seed, "k"), "unit"),
        "v": _fill_rows(mk(dv), _gen(dev, seed, "v"), "normal"),
        "g": _fill_rows(mk(dk), _gen(dev, seed, "g"), "softplus_decay"),
        "beta": _fill_rows(torch.empty((steps, batch, H), device=dev, dtype=dtype),
                           _gen(dev, seed, "beta"), "sigmoid"),
        "gate": _fill_rows(mk(dv), _gen(dev, seed, "z"), "normal") if gate else None,
        "S": S,
        "scale": 1.0 / math.sqrt(dk),
    }
