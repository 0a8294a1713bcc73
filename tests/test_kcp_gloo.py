"""Context-parallel prefill (KCP) across ranks: the collective logic of
``kcp_chunk_fwd`` on CPU ranks over gloo, world sizes 2 and 3.

The compute steps are the oracle's (fp64): a piece's summary is its final
state from zero (from S0 on rank 0) and, run from the identity with v = 0,
its transition product.  Stitched by the all-gather and the fold, every
rank's outputs and the last rank's final state must equal the oracle run on
the whole sequences (Kimi K3 report digest, section 基础设施: segment states
plus the incoming state times the transition product).  Pieces of unequal
length and empty pieces are included."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_136_b200 import inputs
from gated_delta_rule_136_b200.kcp import kcp_chunk_fwd, split_pieces

LENGTHS = [300, 130, 64]        # with 3 ranks the 64-token sequence leaves two empty pieces
H, D = 2, 16
SEED = 7


class OracleOps:
    """The three compute steps of KCP, from the oracle (CPU, fp64)."""

    summary_dtype = torch.float64

    def summary(self, q, k, v, g, beta, cu_seqlens, cu_host, S0, with_M, scale, g_floor):
        N, Hh, dk, dv = len(cu_host) - 1, q.shape[1], q.shape[2], v.shape[2]
        cu = np.asarray(cu_host, dtype=np.int64)
        out = np.zeros((2, N, Hh, dk, dv))
        _, out[0] = oracle.kda_fwd_ref(q, k, v, g, beta, cu_seqlens=cu, S0=S0, scale=scale,
                                       g_floor=g_floor)
        if with_M:
            eye = np.broadcast_to(np.eye(dk), (N, Hh, dk, dk)).copy()
            zero_v = torch.zeros(q.shape[0], Hh, dk, dtype=torch.float64)
            _, out[1] = oracle.kda_fwd_ref(q, k, zero_v, g, beta, cu_seqlens=cu, S0=eye, scale=scale,
                                           g_floor=g_floor)
        return torch.from_numpy(out)

    def combine(self, summaries):
        S = summaries[0, 0].clone()
        for p in range(1, summaries.shape[0]):
            S = summaries[p, 1] @ S + summaries[p, 0]
        return S

    def prefill(self, q, k, v, g, beta, cu_seqlens, cu_host, S0, gate, scale, g_floor):
        o, S_T = oracle.kda_fwd_ref(q, k, v, g, beta, cu_seqlens=np.asarray(cu_host, dtype=np.int64),
                                    S0=S0, scale=scale, gate=gate, g_floor=g_floor)
        return torch.from_numpy(o), torch.from_numpy(S_T)


def _full_inputs():
    return inputs.prefill_inputs(LENGTHS, H=H, dk=D, dv=D, dtype=torch.float32, device="cpu",
                                 seed=SEED, s0_std=0.05, gate=True)


def _local(full, pieces):
    """This rank's pieces, packed: row slices of every sequence."""
    cu = full["cu_seqlens_host"]
    rows = [torch.arange(cu[n] + a, cu[n] + b) for n, (a, b) in enumerate(pieces)]
    idx = torch.cat(rows)
    loc = {name: full[name][idx] for name in ("q", "k", "v", "g", "beta", "gate")}
    lens = [b - a for a, b in pieces]
    loc["cu_seqlens_host"] = [0] + list(np.cumsum(lens).tolist())
    return loc


def _rank_main(rank, world, port, outdir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        full = _full_inputs()
        pieces = split_pieces(LENGTHS, world)[rank]
        loc = _local(full, pieces)
        cu_dev = torch.tensor(loc["cu_seqlens_host"], dtype=torch.int32)
        o, S_end = kcp_chunk_fwd(loc["q"], loc["k"], loc["v"], loc["g"], loc["beta"], cu_dev,
                                 loc["cu_seqlens_host"], S0=full["S0"], gate=loc["gate"],
                                 ops=OracleOps())
        torch.save({"o": o, "S_end": S_end, "pieces": pieces}, os.path.join(outdir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_kcp_matches_whole_sequence_oracle(world, tmp_path):
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    full = _full_inputs()
    o_ref, S_ref = oracle.kda_fwd_ref(full["q"], full["k"], full["v"], full["g"], full["beta"],
                                      cu_seqlens=np.asarray(full["cu_seqlens_host"]), S0=full["S0"],
                                      gate=full["gate"])
    res = [torch.load(os.path.join(tmp_path, f"rank{r}.pt")) for r in range(world)]
    cu = full["cu_seqlens_host"]
    for n in range(len(LENGTHS)):
        parts = []
        for r in range(world):
            lens = [b - a for a, b in res[r]["pieces"]]
            start = int(np.sum(lens[:n]))
            parts.append(res[r]["o"][start:start + lens[n]].numpy())
        o_n = np.concatenate(parts)
        ref_n = o_ref[cu[n]:cu[n + 1]]
        assert o_n.shape == ref_n.shape
        assert np.max(np.abs(o_n - ref_n)) <= 1e-10 * max(1.0, np.max(np.abs(ref_n)))
    S_last = res[-1]["S_end"].numpy()
    assert np.max(np.abs(S_last - S_ref)) <= 1e-10 * max(1.0, np.max(np.abs(S_ref)))


def test_split_pieces_cover_each_sequence():
    for world in (1, 2, 3, 8):
        per_rank = split_pieces([0, 1, 63, 64, 65, 1000, 4097], world)
        for n, L in enumerate([0, 1, 63, 64, 65, 1000, 4097]):
            spans = [per_rank[r][n] for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == L
            for (a0, b0), (a1, b1) in zip(spans, spans[1:]):
                assert b0 == a1 and a0 <= b0
            for a, b in spans[:-1]:
                assert a % 64 == 0 and b % 64 == 0 or b == L
