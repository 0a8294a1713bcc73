#!/usr/bin/env python
"""Benchmark of the KDA forward on B200.

Default workload (one "step"): KDA chunked prefill, bf16 I/O, fp32 state,
B=8 sequences x T=4096 tokens, H=32 heads, dk=dv=128, S0 = 0, final state
returned -- the configuration the headline metric is quoted on.  The decode
hot path is measured in the same run (512 sequences x 64 heads, 128x128 fp32
state per head, bf16 inputs with a sigmoid output gate, 1000 consecutive
steps) and reported in the ``decode`` object of the same JSON line, and so
are the two other prefill workloads (64 varlen sequences x 64 heads; one
2^20-token sequence x 32 heads with decay near the floor), each with its own
roofline object under ``other_workloads`` (``--no-extra`` skips them).

Prints ONE JSON line on rank 0.  ``--impl reference`` times the fp64 CPU
oracle (the only reference implementation there is) on a bounded sample of
the same workload.

Multi-GPU: one process per GPU (torchrun); every rank runs the full
single-GPU workload on its own GPU (independent units, no data-path
collective: weak scaling); value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s + TFLOP/s (% BF16 peak); decode steps/s + state HBM GB/s"

# workload (prefill)
B, T, H, DK, DV = 8, 4096, 32, 128, 128
CHUNK_ALG = 64
# workload (decode)
DEC_B, DEC_H, DEC_STEPS = 512, 64, 1000
EXTRA_WORKLOADS = ("varlen", "long", "snapshots", "spec", "backward", "kcp")
DEFAULT_EXTRAS = ("varlen", "long")   # the other two prefill workloads, timed in every run


def flops_per_token_head(dk=DK, dv=DV, C=CHUNK_ALG):
    """Algorithmic FLOPs per token and head of the chunked forward: the
    state products (W S, (Q e^G) S, K^T Vn: 6 dk dv), the intra-chunk
    products (A_qk, A_kk, W, U, A_qk Vn: C (3 dk + 2 dv), causal halves) and
    the triangular inverse (C^2 / 3)."""
    return 6 * dk * dv + C * (3 * dk + 2 * dv) + C * C / 3.0


def bytes_per_token_head(dk=DK, dv=DV, esz=2):
    """Minimum HBM bytes per token and head: read q, k, g, v, beta; write o."""
    return esz * (3 * dk + dv + 1) + esz * dv


# DRAM traffic per unit from the ncu captures under profiles/ (bytes), valid only
# for the kernel source they were taken from (sha1 prefix); otherwise null.
PROFILED_TRAFFIC = {
    "csrc/kda_chunk_tc.cuh": {"sha1": "372ef2e0393a", "bytes_per_token_head": (269.303296e6 + 52.576000e6) / 262144,
                              "profile": "profiles/chunk_tc_kernel_prefill_4x4096x16.md"},
    "csrc/kda_decode.cuh": {"sha1": "8e75484b34f3", "bytes_per_head_step": (273.707520e6 + 212.401408e6) / 4096,
                            "profile": "profiles/decode_kernel_64x64.md"},
    # speculative verify (4 draft tokens) + commit (3) at batch 128 x 64 heads: per head and round
    "csrc/kda_spec.cuh": {"sha1": "5f78f5eaf7b5",
                          "bytes_per_head_round": (579.116800e6 + 4.305920e6 + 555.884544e6 + 477.843968e6) / 8192,
                          "profile": "profiles/spec_kernel_verify_commit_128x64.md"},
    # chunked backward's gradient kernel (chain_grad) at 1 x 4096 x 32 (bf16): per token-head
    "csrc/kda_bwd_chunk.cuh": {"sha1": "572415ff7970", "bytes_per_token_head": (638.781952e6 + 183.433984e6) / 131072,
                               "profile": "profiles/bwd_chunk_kernels_1x4096x32.md"},
}


def profiled_traffic(src: str, key: str, units: float):
    """Traffic per launch scaled from the capture, or None if the kernel changed."""
    import hashlib
    rec = PROFILED_TRAFFIC[src]
    path = os.path.join(ROOT, "gated_delta_rule_136_b200", src)
    try:
        digest = hashlib.sha1(open(path, "rb").read()).hexdigest()[:12]
    except OSError:
        return None
    return rec[key] * units if digest == rec["sha1"] else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """Samples nvidia-smi clocks / throttle reasons in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.windows = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for ts, line in self.lines:
            if not any(a - 0.25 <= ts <= b + 0.25 for a, b in self.windows):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]),
                             "util": float(parts[4]) if parts[4] not in ("", "[N/A]") else 100.0,
                             "reasons": parts[5:10]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r["util"] >= 50] or rows
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(1, 5)
                          if r["reasons"][i].lower() == "active"})
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in loaded), "reasons": reasons,
                "samples": len(loaded)}


def gpu_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


def run_oracle_sample(seconds_target: float, seed: int = 0):
    """Times the fp64 oracle on a bounded slice of the prefill workload: whole
    4096-token sequences with all heads, as many sequences as fit the time
    target.  Returns (token_heads, secs, threads, description)."""
    import oracle
    from gated_delta_rule_136_b200 import inputs
    threads = oracle.max_threads()
    seqs = max(1, math.ceil(threads / H))
    inp = inputs.prefill_inputs([T] * seqs, H=H, dk=DK, dv=DV, device="cpu", seed=seed)
    args = [inp[n] for n in ("q", "k", "v", "g", "beta")]
    t0 = time.perf_counter()
    oracle.kda_fwd_ref(*args, cu_seqlens=inp["cu_seqlens_host"], nthreads=threads)
    dt = time.perf_counter() - t0
    reps = max(1, min(B, int(seconds_target / max(dt, 1e-3))))
    if reps > 1:
        seqs = min(B, seqs * reps)
        inp = inputs.prefill_inputs([T] * seqs, H=H, dk=DK, dv=DV, device="cpu", seed=seed)
        args = [inp[n] for n in ("q", "k", "v", "g", "beta")]
        t0 = time.perf_counter()
        oracle.kda_fwd_ref(*args, cu_seqlens=inp["cu_seqlens_host"], nthreads=threads)
        dt = time.perf_counter() - t0
    th = seqs * T * H
    desc = (f"{seqs} of {B} sequences x {H} heads x {T} tokens (dk=dv={DK}, bf16-valued "
            f"inputs, fp64 math) of the prefill workload")
    return th, dt, threads, desc


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from gated_delta_rule_136_b200 import inputs
    threads = oracle.max_threads()
    heads, seqs = H, max(1, math.ceil(threads / H))   # at least one unit per host thread
    inp = inputs.prefill_inputs([T] * seqs, H=heads, dk=DK, dv=DV, device="cpu", seed=0)
    a = [inp[n] for n in ("q", "k", "v", "g", "beta")]
    for _ in range(args.warmup):
        oracle.kda_fwd_ref(*a, cu_seqlens=inp["cu_seqlens_host"], nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.kda_fwd_ref(*a, cu_seqlens=inp["cu_seqlens_host"], nthreads=threads)
    dt = time.perf_counter() - t0
    tok_per_s = (seqs * T * heads / H) * args.steps / dt
    sample = (f"each step: {seqs} of {B} sequences x {heads} heads x {T} tokens of the prefill "
              f"workload (fp64 oracle, bf16-valued inputs)")
    line = {"metric": METRIC, "value": tok_per_s, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": f"KDA prefill B={B} T={T} H={H} dk=dv={DK}", "global_batch": B,
                       "seq_len": T, "parallelism": "cpu"},
            "cpu_baseline": {"value": tok_per_s, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": tok_per_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    global B, T, H, DEC_B, DEC_STEPS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    # smaller workloads for profiling runs only (a reported bench line uses the defaults)
    ap.add_argument("--batch", type=int, default=B)
    ap.add_argument("--seqlen", type=int, default=T)
    ap.add_argument("--heads", type=int, default=H)
    ap.add_argument("--decode-batch", type=int, default=DEC_B)
    ap.add_argument("--decode-steps", type=int, default=DEC_STEPS)
    ap.add_argument("--extra", default="",
                    help="comma-separated extra workloads to time: " + ", ".join(EXTRA_WORKLOADS)
                         + " (varlen and long are timed by default)")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the headline prefill and the decode (not varlen / long)")
    ap.add_argument("--all-workloads", action="store_true",
                    help="also time the varlen (64 x [512, 32768] x 64 heads) and the "
                         "1M-token x 32-head floor-stress prefill, the headline prefill "
                         "with state snapshots every 512 tokens, speculative-decode "
                         "verify/commit rounds, the backward of the headline prefill and, "
                         "with more than one rank, the context-parallel prefill")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    extras = {x for x in args.extra.split(",") if x}
    if args.all_workloads:
        extras = set(EXTRA_WORKLOADS)
    elif not args.no_extra:
        extras |= set(DEFAULT_EXTRAS)
    if extras - set(EXTRA_WORKLOADS):
        ap.error(f"--extra: unknown workload(s) {sorted(extras - set(EXTRA_WORKLOADS))}; "
                 f"choose from {', '.join(EXTRA_WORKLOADS)}")
    B, T, H = args.batch, args.seqlen, args.heads
    DEC_B, DEC_STEPS = args.decode_batch, args.decode_steps
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    import torch.distributed as dist
    from gated_delta_rule_136_b200 import chunk_fwd, decode_step, device_status, inputs
    from gated_delta_rule_136_b200 import kda as kbind

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    peaks = load_peaks()
    kbind.load_library()
    sampler = ClockSampler(gpu_uuid(torch, dev)) if rank == 0 else None
    if sampler:
        sampler.start()

    # ---------------- prefill (headline) ----------------
    inp = inputs.prefill_inputs([T] * B, H=H, dk=DK, dv=DV, device=dev, seed=rank)
    q, k, v, g, beta = (inp[n] for n in ("q", "k", "v", "g", "beta"))
    cu, cu_host = inp["cu_seqlens"], inp["cu_seqlens_host"]
    o = torch.empty_like(v)
    S_T = torch.empty((B, H, DK, DV), device=dev, dtype=torch.float32)
    ws = torch.empty(max(256, kbind.workspace_size(B * T, B, H, DK, DV, cu_seqlens_host=cu_host,
                                                   chunk=args.chunk)), dtype=torch.uint8, device=dev)

    def prefill_step():
        chunk_fwd(q, k, v, g, beta, cu_seqlens=cu, cu_seqlens_host=cu_host, out=o,
                  final_state_out=S_T, workspace=ws, chunk=args.chunk)

    for _ in range(args.warmup):
        prefill_step()
    barrier()
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t_wall0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        prefill_step()
        ev[i][1].record(stream)
    end.record(stream)
    barrier()
    t_wall1 = time.time()
    if sampler:
        sampler.mark(t_wall0, t_wall1)
    elapsed_ms = max_over_ranks(start.elapsed_time(end))
    per_call_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    status = device_status(dev)
    if status != 0:
        raise RuntimeError(f"device error word after prefill: {status}")

    th = B * T * H
    tok_per_step = B * T
    value = world * tok_per_step * args.steps / (elapsed_ms / 1e3)
    alg_bytes = th * bytes_per_token_head() + B * H * DK * DV * 4   # + S_T write
    alg_flops = th * flops_per_token_head()
    achieved_gbs = alg_bytes / (per_call_ms / 1e3) / 1e9
    tflops = alg_flops / (per_call_ms / 1e3) / 1e12

    # ---------------- e2e through host buffers ----------------
    # kda_chunk_fwd_host: inputs from and outputs to page-locked host memory,
    # the copies pipelined with the prefill inside the library; the binding
    # synchronises the stream (the result read) before it returns
    e2e = None
    if not args.no_e2e:
        from gated_delta_rule_136_b200 import chunk_fwd_host
        host = {n: inp[n].to("cpu").pin_memory() for n in ("q", "k", "v", "g", "beta")}
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        S_host = torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_host.numel() * o_host.element_size() + S_host.numel() * S_host.element_size()

        def e2e_step():
            chunk_fwd_host(host["q"], host["k"], host["v"], host["g"], host["beta"], cu_host,
                           out=o_host, final_state_out=S_host, device=dev)

        e2e_steps = max(3, min(args.steps, 10))
        for _ in range(args.warmup):
            e2e_step()
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tw0 = time.time()
        s0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        s1.record(stream)
        barrier()
        if sampler:
            sampler.mark(tw0, time.time())
        e2e_ms = max_over_ranks(s0.elapsed_time(s1))
        e2e = {"value": world * tok_per_step * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "api": "kda_chunk_fwd_host (host buffers; copies pipelined with the prefill)"}
        del host, o_host, S_host

    del inp, q, k, v, g, beta, o
    torch.cuda.empty_cache()

    # ---------------- decode ----------------
    decode = None
    if not args.no_decode:
        d = inputs.decode_inputs(batch=DEC_B, H=DEC_H, dk=DK, dv=DV, steps=DEC_STEPS, device=dev,
                                 seed=rank)
        S = d["S"]
        od = torch.empty((DEC_STEPS, DEC_B, DEC_H, DV), dtype=torch.bfloat16, device=dev)
        for t in range(args.warmup):
            decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S,
                        gate=d["gate"][t], out=od[t])
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tw0 = time.time()
        s0.record(stream)
        for t in range(DEC_STEPS):
            decode_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S,
                        gate=d["gate"][t], out=od[t])
        s1.record(stream)
        barrier()
        if sampler:
            sampler.mark(tw0, time.time())
        dec_ms = max_over_ranks(s0.elapsed_time(s1))
        if device_status(dev) != 0:
            raise RuntimeError("device error word after decode")
        units = DEC_B * DEC_H
        dec_bytes = units * (2 * DK * DV * 4 + 2 * (3 * DK + DV + 1) + 2 * DV + 2 * DV)
        per_step_s = dec_ms / 1e3 / DEC_STEPS
        dec_gbs = dec_bytes / per_step_s / 1e9
        decode = {"workload": f"KDA decode_step batch={DEC_B} H={DEC_H} dk=dv={DK} fp32 state, "
                              f"bf16 q/k/v/g/beta, sigmoid gate, {DEC_STEPS} consecutive steps",
                  "steps_per_s": world / per_step_s, "ms_per_step": per_step_s * 1e3,
                  "state_hbm_gbs": dec_gbs,
                  "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"],
                               "traffic": profiled_traffic("csrc/kda_decode.cuh",
                                                           "bytes_per_head_step", units)},
                  "bytes_per_step": dec_bytes, "gpu_launches": DEC_STEPS}
        del d, S, od
        torch.cuda.empty_cache()

    others = None
    if extras:
        others = {}
        cases = {
            "varlen 64 sequences, lengths U[512, 32768], H=64, S0 ~ N(0, 0.02)":
                dict(lengths=inputs.varlen_lengths(64, 512, 32768, seed=0), H=64, s0_std=0.02,
                     g_mode="softplus"),
            "1 sequence x 2^20 tokens, H=32, g ~ -5 U(0.8, 1)":
                dict(lengths=[1 << 20], H=32, s0_std=None, g_mode="floor_stress"),
        }
        keys = dict(zip(cases, ("varlen", "long")))
        cases = {name: c for name, c in cases.items() if keys[name] in extras}
        for name, c in cases.items():
            w = inputs.prefill_inputs(c["lengths"], H=c["H"], dk=DK, dv=DV, device=dev, seed=rank,
                                      s0_std=c["s0_std"], g_mode=c["g_mode"])
            ow = torch.empty_like(w["v"])
            Sw = torch.empty((len(c["lengths"]), c["H"], DK, DV), device=dev, dtype=torch.float32)
            wsz = kbind.workspace_size(w["q"].shape[0], len(c["lengths"]), c["H"], DK, DV,
                                       cu_seqlens_host=w["cu_seqlens_host"])
            wsw = torch.empty(max(256, wsz), dtype=torch.uint8, device=dev)
            run = lambda: chunk_fwd(w["q"], w["k"], w["v"], w["g"], w["beta"], S0=w["S0"],
                                    cu_seqlens=w["cu_seqlens"], cu_seqlens_host=w["cu_seqlens_host"],
                                    out=ow, final_state_out=Sw, workspace=wsw)
            for _ in range(2):
                run()
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 3
            tw0 = time.time()
            a.record(stream)
            for _ in range(reps):
                run()
            b.record(stream)
            barrier()
            if sampler:
                sampler.mark(tw0, time.time())
            ms = max_over_ranks(a.elapsed_time(b)) / reps
            ttok = int(w["q"].shape[0])
            byts = ttok * c["H"] * bytes_per_token_head() + len(c["lengths"]) * c["H"] * DK * DV * 4 * (
                2 if c["s0_std"] is not None else 1)
            gbs = byts / (ms / 1e3) / 1e9
            others[name] = {"tokens": ttok, "ms": ms, "tokens_per_s": world * ttok / (ms / 1e3),
                            "alg_gbs": gbs, "roofline_frac": gbs / peaks["hbm_gbs"],
                            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                                         "traffic": None, "alg_bytes_per_launch": byts,
                                         "kernel": "kda_chunk_fwd (plan or segment split + chunk kernel)",
                                         "peak_source": peaks["source"]}}
            del w, ow, Sw, wsw
            torch.cuda.empty_cache()

        if "snapshots" in extras:
            # the headline prefill with state snapshots every 512 tokens (prefix-cache hook)
            from gated_delta_rule_136_b200 import chunk_fwd_snapshots
            w = inputs.prefill_inputs([T] * B, H=H, dk=DK, dv=DV, device=dev, seed=rank)
            interval = 512
            run = lambda: chunk_fwd_snapshots(w["q"], w["k"], w["v"], w["g"], w["beta"], interval,
                                              cu_seqlens=w["cu_seqlens"],
                                              cu_seqlens_host=w["cu_seqlens_host"])
            for _ in range(2):
                run()
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            tw0 = time.time()
            a.record(stream)
            for _ in range(reps):
                run()
            b.record(stream)
            barrier()
            if sampler:
                sampler.mark(tw0, time.time())
            if device_status(dev) != 0:
                raise RuntimeError("device error word after the snapshot prefill")
            ms = max_over_ranks(a.elapsed_time(b)) / reps
            nsnap = B * (T // interval)
            byts = B * T * H * bytes_per_token_head() + B * H * DK * DV * 4 + nsnap * H * DK * DV * 4
            others[f"prefill B={B} T={T} H={H} with state snapshots every {interval} tokens"] = {
                "tokens": B * T, "ms": ms, "tokens_per_s": world * B * T / (ms / 1e3),
                "snapshot_bytes": nsnap * H * DK * DV * 4, "alg_gbs": byts / (ms / 1e3) / 1e9,
                "roofline_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                "note": "timed through the Python binding, which allocates the snapshot buffer and "
                        "uploads the slot table on every call"}
            del w
            torch.cuda.empty_cache()

        if "spec" in extras:
            # speculative decode: verify D = 4 draft tokens, commit 3, per round (decode batch)
            from gated_delta_rule_136_b200 import spec_commit, spec_verify
            Dd = 4
            sd = inputs.prefill_inputs([Dd] * DEC_B, H=DEC_H, dk=DK, dv=DV, device=dev, seed=rank,
                                       s0_std=0.02, gate=True)
            xs = {n: sd[n].view(DEC_B, Dd, *sd[n].shape[1:]) for n in ("q", "k", "v", "g", "beta", "gate")}
            Ssp = sd["S0"]
            osp = torch.empty_like(xs["v"])
            accd = torch.full((DEC_B,), 3, dtype=torch.int32, device=dev)

            def spec_round():
                spec_verify(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], Ssp, gate=xs["gate"], out=osp)
                spec_commit(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], Ssp, accd)

            for _ in range(args.warmup):
                spec_round()
            barrier()
            rounds = 50
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            tw0 = time.time()
            a.record(stream)
            for _ in range(rounds):
                spec_round()
            b.record(stream)
            barrier()
            if sampler:
                sampler.mark(tw0, time.time())
            if device_status(dev) != 0:
                raise RuntimeError("device error word after speculative decode")
            ms = max_over_ranks(a.elapsed_time(b)) / rounds

            def time_one(fn):   # one call type alone, on the same (cached-out) state
                a.record(stream)
                for _ in range(rounds):
                    fn()
                b.record(stream)
                barrier()
                return max_over_ranks(a.elapsed_time(b)) / rounds
            ms_v = time_one(lambda: spec_verify(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], Ssp,
                                                gate=xs["gate"], out=osp))
            ms_c = time_one(lambda: spec_commit(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], Ssp, accd))
            heads = DEC_B * DEC_H
            byts = heads * (3 * DK * DV * 4 + Dd * (2 * (3 * DK + DV + 1) + 2 * DV + 2 * DV)
                            + 3 * 2 * (3 * DK + DV + 1))
            byts_v = heads * (DK * DV * 4 + Dd * (2 * (3 * DK + DV + 1) + 2 * DV + 2 * DV))
            others[f"speculative decode batch={DEC_B} H={DEC_H}: verify {Dd} draft tokens, commit 3"] = {
                "rounds_per_s": world * 1e3 / ms, "ms_per_round": ms,
                "ms_verify": ms_v, "ms_commit": ms_c,
                "verify_roofline": {"bound": "hbm", "achieved": byts_v / (ms_v / 1e3) / 1e9,
                                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": byts_v / (ms_v / 1e3) / 1e9 / peaks["hbm_gbs"], "traffic": None},
                "verified_tokens_per_s": world * DEC_B * Dd / (ms / 1e3),
                "alg_gbs": byts / (ms / 1e3) / 1e9, "roofline_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                "alg_bytes_per_round": byts,
                "traffic": profiled_traffic("csrc/kda_spec.cuh", "bytes_per_head_round", heads),
                "note": "the state crosses HBM three times per round (verify read, commit read and "
                        "write) instead of twice per token"}
            del sd, xs, Ssp, osp, accd
            torch.cuda.empty_cache()

        if "backward" in extras:
            # backward of the headline prefill (training): gradients of sum(o * dout)
            from gated_delta_rule_136_b200 import chunk_bwd
            xb = inputs.prefill_inputs([T] * B, H=H, dk=DK, dv=DV, device=dev, seed=rank)
            gen = torch.Generator(device=dev).manual_seed(200 + rank)
            dout = torch.randn(xb["v"].shape, generator=gen, device=dev).to(torch.bfloat16)
            runb = lambda: chunk_bwd(xb["q"], xb["k"], xb["v"], xb["g"], xb["beta"], dout,
                                     cu_seqlens=xb["cu_seqlens"], cu_seqlens_host=xb["cu_seqlens_host"],
                                     want_dS0=False)
            for _ in range(2):
                runb()
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 3
            tw0 = time.time()
            a.record(stream)
            for _ in range(reps):
                runb()
            b.record(stream)
            barrier()
            if sampler:
                sampler.mark(tw0, time.time())
            if device_status(dev) != 0:
                raise RuntimeError("device error word after backward")
            ms = max_over_ranks(a.elapsed_time(b)) / reps
            # inputs q, k, g, v, dout and beta read once, dq, dk, dg, dv and dbeta written once
            byts = B * T * H * (5 * DK * 2 + 2 + 4 * DK * 2 + 2)
            others[f"backward B={B} T={T} H={H} (gradients of sum(o * dout), bf16)"] = {
                "tokens": B * T, "ms": ms, "tokens_per_s": world * B * T / (ms / 1e3),
                "alg_gbs": byts / (ms / 1e3) / 1e9, "roofline_frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                "alg_bytes": byts,
                "traffic_chain_grad_kernel": profiled_traffic("csrc/kda_bwd_chunk.cuh", "bytes_per_token_head",
                                                              B * T * H),
                "note": "forward with 64-token state snapshots, then the chunked backward: the gradient "
                        "chain's per-chunk constants (a CTA per chunk x head), the chain over chunks (a CTA "
                        "per sequence x head), every gradient of a chunk (a CTA per chunk x head); tf32 "
                        "mma.sync products, 3xTF32 where dg's terms cancel"}
            del xb, dout
            torch.cuda.empty_cache()

        if "kcp" in extras:
            # one rank's KCP summary: a 2^20 / 8-token piece, H=32, state from zero and
            # transition product (a middle rank of eight), on this GPU alone
            from gated_delta_rule_136_b200 import segment_summary
            Lp, Hp = (1 << 20) // 8, 32
            wp = inputs.prefill_inputs([Lp], H=Hp, dk=DK, dv=DV, device=dev, seed=300 + rank,
                                       g_mode="floor_stress")
            runs = lambda: segment_summary(wp["q"], wp["k"], wp["v"], wp["g"], wp["beta"], wp["cu_seqlens"],
                                           wp["cu_seqlens_host"], with_M=True)
            for _ in range(2):
                runs()
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 3
            tw0 = time.time()
            a.record(stream)
            for _ in range(reps):
                runs()
            b.record(stream)
            barrier()
            if sampler:
                sampler.mark(tw0, time.time())
            if device_status(dev) != 0:
                raise RuntimeError("device error word after the piece summary")
            ms = max_over_ranks(a.elapsed_time(b)) / reps
            others[f"KCP piece summary: {Lp} tokens x H={Hp} (S_loc and M), one rank"] = {
                "tokens": Lp, "ms": ms, "tokens_per_s": world * Lp / (ms / 1e3),
                "note": "two chains per (piece, head), cut into sub-segments folded by the scan kernel "
                        "when the chains are fewer than the SMs"}
            del wp
            torch.cuda.empty_cache()

        if world > 1 and "kcp" in extras:
            # context-parallel prefill (KCP): one 2^20-token sequence, H=32, cut into one
            # piece per rank; the piece summaries cross ranks in one NCCL all-gather
            from gated_delta_rule_136_b200 import kcp_chunk_fwd, split_pieces
            Lk, Hk = 1 << 20, 32
            a0, b0 = split_pieces([Lk], world)[rank][0]
            wk = inputs.prefill_inputs([b0 - a0], H=Hk, dk=DK, dv=DV, device=dev, seed=100 + rank,
                                       s0_std=None, g_mode="floor_stress")
            runk = lambda: kcp_chunk_fwd(wk["q"], wk["k"], wk["v"], wk["g"], wk["beta"], wk["cu_seqlens"],
                                         wk["cu_seqlens_host"])
            for _ in range(2):
                runk()
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 3
            tw0 = time.time()
            a.record(stream)
            for _ in range(reps):
                runk()
            b.record(stream)
            barrier()
            if sampler:
                sampler.mark(tw0, time.time())
            if device_status(dev) != 0:
                raise RuntimeError("device error word after context-parallel prefill")
            ms = max_over_ranks(a.elapsed_time(b)) / reps
            others[f"context-parallel prefill: 1 sequence x 2^20 tokens, H={Hk}, one piece per rank"] = {
                "tokens": Lk, "ranks": world, "ms": ms, "tokens_per_s": Lk / (ms / 1e3),
                "scaling": "strong",
                "note": "summary (state from zero and transition product per piece), NCCL all-gather "
                        "of the summaries, fold, rerun of each piece with outputs"}
            del wk
            torch.cuda.empty_cache()

    if sampler:
        sampler.stop()
        clocks = sampler.summary()
    else:
        clocks = None

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        th_s, secs, threads, desc = run_oracle_sample(args.cpu_seconds)
        cpu_baseline = {"value": th_s / H / secs, "unit": "tokens/s", "cores": threads,
                        "kind": "oracle", "sample": desc + f"; {secs:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"KDA prefill B={B} T={T} H={H} dk=dv={DK} bf16 I/O fp32 state, "
                                   f"S0=0, final state returned", "global_batch": B * world,
                       "seq_len": T, "heads": H, "dk": DK, "dv": DV,
                       "parallelism": f"dp{world} (independent units per rank)",
                       "l2": "inputs (1.36 GB per step) larger than L2; no flush"},
            "tflops": tflops, "pct_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                         "traffic": profiled_traffic("csrc/kda_chunk_tc.cuh", "bytes_per_token_head", th),
                         "kernel": "kda_chunk_fwd (plan + chunk kernel)",
                         "alg_bytes_per_launch": alg_bytes, "alg_flops_per_launch": alg_flops,
                         "peak_source": peaks["source"]},
            "e2e": e2e, "decode": decode, "cpu_baseline": cpu_baseline,
            "other_workloads": others,
            "gpu_launches": 2 * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
