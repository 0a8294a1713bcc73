"""Python binding of the KDA C ABI (``include/kda.h``).

Argument marshalling only: shape/dtype/device checks, output and workspace
allocation through PyTorch (device memory and streams are PyTorch's job), and
raw pointers plus the current CUDA stream handed to the library.  Every step
of the forward runs in the library's CUDA kernels; there is no CPU or PyTorch
fallback, and a missing library or GPU raises.
"""
from __future__ import annotations

import ctypes
import os
import itertools
import math
import threading

import torch

from . import build as _build

KDA_OK = 0
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_WORKSPACE", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_TIMEOUT",
                6: "KDA_ERR_DEVICE_BOUNDS"}
KDA_BF16, KDA_FP32 = 0, 1

# Every function include/kda.h declares.
EXPORTED_SYMBOLS = ("kda_chunk_fwd_workspace_size", "kda_chunk_fwd", "kda_decode_step",
                    "kda_get_device_status", "kda_status_string", "kda_version",
                    "kda_chunk_fwd_noalloc", "kda_selftest_bounded_wait",
                    "kda_chunk_fwd_snapshots", "kda_spec_verify", "kda_spec_commit",
                    "kda_segment_summary_workspace_size", "kda_segment_summary",
                    "kda_state_combine", "kda_chunk_bwd_workspace_size", "kda_chunk_bwd",
                    "kda_chunk_fwd_host_workspace_size", "kda_chunk_fwd_host")
NOALLOC_MAX_SEQS = 65536   # KDA_NOALLOC_MAX_SEQS in include/kda.h


class Snapshots(ctypes.Structure):
    """``kda_snapshots``."""
    _fields_ = [("interval", ctypes.c_int32), ("total", ctypes.c_int64),
                ("base", ctypes.c_void_p), ("states", ctypes.c_void_p)]


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {STATUS_NAMES.get(status, status)}")


class FwdDesc(ctypes.Structure):
    _fields_ = [("total_tokens", ctypes.c_int64), ("num_seqs", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("io_dtype", ctypes.c_int), ("scale", ctypes.c_float),
                ("g_floor", ctypes.c_float), ("chunk", ctypes.c_int32),
                ("max_seqlen", ctypes.c_int32)]


class DecodeDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("io_dtype", ctypes.c_int),
                ("scale", ctypes.c_float), ("g_floor", ctypes.c_float)]


class SpecDesc(ctypes.Structure):
    """``kda_spec_desc``."""
    _fields_ = [("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("draft", ctypes.c_int32),
                ("io_dtype", ctypes.c_int), ("scale", ctypes.c_float), ("g_floor", ctypes.c_float)]


class CombineDesc(ctypes.Structure):
    """``kda_combine_desc``."""
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("num_summaries", ctypes.c_int32)]


SPEC_MAX_DRAFT = 64   # KDA_SPEC_MAX_DRAFT in include/kda.h

_lib = None
_lock = threading.Lock()


def _debug_library() -> bool:
    return os.environ.get("KDA_DEBUG_LIBRARY", "") not in ("", "0")


def library_path() -> str:
    return _build.DEBUG_LIB_PATH if _debug_library() else _build.LIB_PATH


def load_library(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load (building first if missing or stale) the KDA shared library; with
    KDA_DEBUG_LIBRARY=1 in the environment, its debug variant (device-side
    argument checks)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        debug = _debug_library()
        path = _build.build(debug=debug) if build_if_missing else library_path()
        lib = ctypes.CDLL(path)
        vp, sz, i32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32)
        lib.kda_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(FwdDesc), i32p]
        lib.kda_chunk_fwd_workspace_size.restype = sz
        lib.kda_chunk_fwd.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, vp, vp, vp, vp, i32p,
                                      vp, vp, vp, vp, sz, vp]
        lib.kda_chunk_fwd.restype = ctypes.c_int
        lib.kda_decode_step.argtypes = [ctypes.POINTER(DecodeDesc), vp, vp, vp, vp, vp, vp, vp,
                                        vp, vp]
        lib.kda_decode_step.restype = ctypes.c_int
        lib.kda_get_device_status.argtypes = [vp]
        lib.kda_get_device_status.restype = ctypes.c_int
        lib.kda_status_string.argtypes = [ctypes.c_int]
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_version.restype = ctypes.c_int32
        lib.kda_chunk_fwd_snapshots.argtypes = [ctypes.POINTER(FwdDesc), ctypes.POINTER(Snapshots),
                                                vp, vp, vp, vp, vp, vp, i32p, i32p, vp, vp, vp, vp,
                                                sz, vp]
        lib.kda_chunk_fwd_snapshots.restype = ctypes.c_int
        lib.kda_spec_verify.argtypes = [ctypes.POINTER(SpecDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.kda_spec_verify.restype = ctypes.c_int
        lib.kda_spec_commit.argtypes = [ctypes.POINTER(SpecDesc), vp, vp, vp, vp, vp, vp, vp, vp]
        lib.kda_spec_commit.restype = ctypes.c_int
        lib.kda_segment_summary_workspace_size.argtypes = [ctypes.POINTER(FwdDesc), i32p, ctypes.c_int32]
        lib.kda_segment_summary_workspace_size.restype = sz
        lib.kda_segment_summary.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, vp, vp, vp, i32p,
                                            i32p, vp, vp, vp, sz, vp]
        lib.kda_segment_summary.restype = ctypes.c_int
        lib.kda_state_combine.argtypes = [ctypes.POINTER(CombineDesc), vp, vp, vp]
        lib.kda_state_combine.restype = ctypes.c_int
        lib.kda_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(FwdDesc), i32p]
        lib.kda_chunk_bwd_workspace_size.restype = sz
        lib.kda_chunk_bwd.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, vp, vp, vp, i32p, i32p, vp,
                                      vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.kda_chunk_bwd.restype = ctypes.c_int
        lib.kda_chunk_fwd_host_workspace_size.argtypes = [ctypes.POINTER(FwdDesc), i32p, ctypes.c_int32,
                                                          ctypes.c_int32, ctypes.c_int32]
        lib.kda_chunk_fwd_host_workspace_size.restype = sz
        lib.kda_chunk_fwd_host.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, vp, vp, vp, i32p, vp, vp,
                                           vp, vp, sz, vp]
        lib.kda_chunk_fwd_host.restype = ctypes.c_int
        lib.kda_selftest_bounded_wait.argtypes = [ctypes.c_int32, vp]
        lib.kda_selftest_bounded_wait.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_FP32
    raise TypeError(f"KDA I/O tensors must be bfloat16 or float32, got {t.dtype}")


def _check(t, name, shape, dtype, device):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _require_cuda():
    if not torch.cuda.is_available():
        raise RuntimeError("the KDA library needs a CUDA GPU (sm_100a); none is available")


def chunk_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, scale=None, gate=None,
              g_floor: float = -5.0, chunk: int = 0, cu_seqlens_host=None,
              output_final_state: bool = True, out=None, final_state_out=None,
              workspace=None):
    """KDA chunked prefill.  Returns ``(o, S_T)`` (``S_T`` None if not requested).

    q, k, g [T,H,dk] (or [B,T,H,dk] with ``cu_seqlens`` None); v, gate
    [T,H,dv]; beta [T,H]; all bf16 or all fp32 on one GPU.  S0 fp32
    [N,H,dk,dv] or None.  ``cu_seqlens`` int32 [N+1] on the GPU (None for a
    single sequence or a fixed-length batch); ``cu_seqlens_host`` an optional
    host copy (list or CPU tensor) used to validate and plan.
    """
    o, S_T, _, _ = _chunk_fwd(q, k, v, g, beta, S0, cu_seqlens, scale, gate, g_floor, chunk,
                              cu_seqlens_host, output_final_state, out, final_state_out, workspace, 0)
    return o, S_T


def chunk_fwd_snapshots(q, k, v, g, beta, interval: int, S0=None, cu_seqlens=None, scale=None,
                        gate=None, g_floor: float = -5.0, chunk: int = 0, cu_seqlens_host=None,
                        output_final_state: bool = True):
    """``kda_chunk_fwd_snapshots``: the prefill of :func:`chunk_fwd` plus the
    state after every ``interval`` tokens of each sequence (a multiple of 64).
    Returns ``(o, S_T, snaps, base)``: ``snaps`` fp32 [total, H, dk, dv] and
    ``base`` int64 [N+1] (CPU) with sequence n's snapshots at rows
    ``base[n] .. base[n+1]-1`` (after ``interval``, ``2 interval``, ... tokens).
    ``cu_seqlens_host`` is required (a single sequence or a fixed-length
    batch supplies its own)."""
    return _chunk_fwd(q, k, v, g, beta, S0, cu_seqlens, scale, gate, g_floor, chunk,
                      cu_seqlens_host, output_final_state, None, None, None, int(interval))


def _chunk_fwd(q, k, v, g, beta, S0, cu_seqlens, scale, gate, g_floor, chunk, cu_seqlens_host,
               output_final_state, out, final_state_out, workspace, snapshot_interval):
    _require_cuda()
    lib = load_library()
    batched = q.dim() == 4
    if batched:
        if cu_seqlens is not None:
            raise ValueError("cu_seqlens is for packed [T,H,d] inputs")
        B, Tb = q.shape[:2]
        q, k, g = (x.reshape(B * Tb, *x.shape[2:]) for x in (q, k, g))
        out_shape = v.shape
        v = v.reshape(B * Tb, *v.shape[2:])
        beta = beta.reshape(B * Tb, -1)
        if gate is not None:
            gate = gate.reshape(B * Tb, *gate.shape[2:])
        cu_host = [i * Tb for i in range(B + 1)]
        cu_seqlens = torch.tensor(cu_host, dtype=torch.int32, device=q.device)
        if cu_seqlens_host is None:
            cu_seqlens_host = cu_host
    else:
        out_shape = v.shape
        if cu_seqlens is None:
            cu_host = [0, q.shape[0]]
            cu_seqlens = torch.tensor(cu_host, dtype=torch.int32, device=q.device)
            if cu_seqlens_host is None:
                cu_seqlens_host = cu_host
    device = q.device
    T, H, dk = q.shape
    dv = v.shape[-1]
    dtype = q.dtype
    N = cu_seqlens.numel() - 1
    _check(q, "q", (T, H, dk), dtype, device)
    _check(k, "k", (T, H, dk), dtype, device)
    _check(g, "g", (T, H, dk), dtype, device)
    _check(v, "v", (T, H, dv), dtype, device)
    _check(beta, "beta", (T, H), dtype, device)
    if gate is not None:
        _check(gate, "gate", (T, H, dv), dtype, device)
    if S0 is not None:
        _check(S0, "S0", (N, H, dk, dv), torch.float32, device)
    _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, device)
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    host_arr = None
    vals = None
    if cu_seqlens_host is not None:
        vals = [int(x) for x in (cu_seqlens_host.tolist() if hasattr(cu_seqlens_host, "tolist")
                                 else cu_seqlens_host)]
        if len(vals) != N + 1:
            raise ValueError("cu_seqlens_host must have N+1 entries")
        host_arr = (ctypes.c_int32 * (N + 1))(*vals)
    desc = FwdDesc(T, N, H, dk, dv, _io_dtype(q), float(scale), float(g_floor), int(chunk), 0)
    ws_bytes = lib.kda_chunk_fwd_workspace_size(ctypes.byref(desc), host_arr)
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise KDAError(1, "kda_chunk_fwd_workspace_size")
    o = out if out is not None else torch.empty((T, H, dv), dtype=dtype, device=device)
    _check(o, "out", (T, H, dv), dtype, device)
    S_T = None
    if output_final_state:
        S_T = (final_state_out if final_state_out is not None
               else torch.empty((N, H, dk, dv), dtype=torch.float32, device=device))
        _check(S_T, "final_state_out", (N, H, dk, dv), torch.float32, device)
    if ws_bytes > 0 and (workspace is None or workspace.numel() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    cu_ptr = ctypes.cast(ctypes.c_void_p(cu_seqlens.data_ptr()), ctypes.POINTER(ctypes.c_int32))
    wsp = _ptr(workspace) if ws_bytes > 0 else None
    snaps = base_host = None
    with torch.cuda.device(device):
        if snapshot_interval:
            if cu_seqlens_host is None:
                raise ValueError("snapshots need cu_seqlens_host")
            counts = [(vals[n + 1] - vals[n]) // int(snapshot_interval) for n in range(N)]
            base_host = torch.tensor([0] + list(itertools.accumulate(counts)), dtype=torch.int64)
            total = int(base_host[-1])
            snaps = torch.empty((total, H, dk, dv), dtype=torch.float32, device=device)
            base_dev = base_host.to(device)
            sd = Snapshots(int(snapshot_interval), total, base_dev.data_ptr() if total else None,
                           snaps.data_ptr() if total else None)
            st = lib.kda_chunk_fwd_snapshots(ctypes.byref(desc), ctypes.byref(sd), _ptr(q), _ptr(k),
                                             _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), cu_ptr, host_arr,
                                             _ptr(gate), _ptr(o), _ptr(S_T), wsp, ws_bytes,
                                             _stream_handle(device))
            where = "kda_chunk_fwd_snapshots"
        else:
            st = lib.kda_chunk_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                   _ptr(S0), cu_ptr, host_arr, _ptr(gate), _ptr(o), _ptr(S_T), wsp,
                                   ws_bytes, _stream_handle(device))
            where = "kda_chunk_fwd"
    if st != KDA_OK:
        raise KDAError(st, where)
    return o.view(out_shape), S_T, snaps, base_host


def workspace_size(T, N, H, dk, dv, dtype=torch.bfloat16, chunk=0, g_floor=-5.0,
                   cu_seqlens_host=None) -> int:
    """Workspace bytes kda_chunk_fwd needs for this problem."""
    lib = load_library()
    desc = FwdDesc(T, N, H, dk, dv, KDA_BF16 if dtype == torch.bfloat16 else KDA_FP32,
                   1.0 / math.sqrt(dk), float(g_floor), int(chunk), 0)
    host_arr = None
    if cu_seqlens_host is not None:
        host_arr = (ctypes.c_int32 * (N + 1))(*[int(x) for x in cu_seqlens_host])
    return int(lib.kda_chunk_fwd_workspace_size(ctypes.byref(desc), host_arr))


def decode_step(q, k, v, g, beta, S, gate=None, scale=None, g_floor: float = -5.0, out=None):
    """One decode step; updates ``S`` in place and returns ``o``.

    q, k, g [B,H,dk]; v, gate [B,H,dv]; beta [B,H]; S fp32 [B,H,dk,dv].
    """
    _require_cuda()
    lib = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    device, dtype = q.device, q.dtype
    _check(q, "q", (B, H, dk), dtype, device)
    _check(k, "k", (B, H, dk), dtype, device)
    _check(g, "g", (B, H, dk), dtype, device)
    _check(v, "v", (B, H, dv), dtype, device)
    _check(beta, "beta", (B, H), dtype, device)
    _check(S, "S", (B, H, dk, dv), torch.float32, device)
    if gate is not None:
        _check(gate, "gate", (B, H, dv), dtype, device)
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    o = out if out is not None else torch.empty((B, H, dv), dtype=dtype, device=device)
    _check(o, "out", (B, H, dv), dtype, device)
    desc = DecodeDesc(B, H, dk, dv, _io_dtype(q), float(scale), float(g_floor))
    with torch.cuda.device(device):
        st = lib.kda_decode_step(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                 _ptr(beta), _ptr(S), _ptr(gate), _ptr(o), _stream_handle(device))
    if st != KDA_OK:
        raise KDAError(st, "kda_decode_step")
    return o


def _spec_desc(q, k, v, g, beta, S, gate, scale, g_floor):
    B, D, H, dk = q.shape
    dv = v.shape[-1]
    device, dtype = q.device, q.dtype
    _check(q, "q", (B, D, H, dk), dtype, device)
    _check(k, "k", (B, D, H, dk), dtype, device)
    _check(g, "g", (B, D, H, dk), dtype, device)
    _check(v, "v", (B, D, H, dv), dtype, device)
    _check(beta, "beta", (B, D, H), dtype, device)
    _check(S, "S", (B, H, dk, dv), torch.float32, device)
    if gate is not None:
        _check(gate, "gate", (B, D, H, dv), dtype, device)
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    return SpecDesc(B, H, dk, dv, D, _io_dtype(q), float(scale), float(g_floor))


def spec_verify(q, k, v, g, beta, S, gate=None, scale=None, g_floor: float = -5.0, out=None):
    """``kda_spec_verify``: outputs of D draft tokens per sequence, replayed from
    ``S`` without changing it.  q, k, g [B,D,H,dk]; v, gate [B,D,H,dv]; beta
    [B,D,H]; S fp32 [B,H,dk,dv].  Returns o [B,D,H,dv]."""
    _require_cuda()
    lib = load_library()
    desc = _spec_desc(q, k, v, g, beta, S, gate, scale, g_floor)
    o = out if out is not None else torch.empty(v.shape, dtype=q.dtype, device=q.device)
    _check(o, "out", tuple(v.shape), q.dtype, q.device)
    with torch.cuda.device(q.device):
        st = lib.kda_spec_verify(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(S), _ptr(gate), _ptr(o), _stream_handle(q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_spec_verify")
    return o


def spec_commit(q, k, v, g, beta, S, accepted, scale=None, g_floor: float = -5.0):
    """``kda_spec_commit``: applies the first ``accepted[b]`` of the D draft tokens
    of sequence b to ``S`` in place (``accepted`` int32 [B] on the GPU)."""
    _require_cuda()
    lib = load_library()
    desc = _spec_desc(q, k, v, g, beta, S, None, scale, g_floor)
    _check(accepted, "accepted", (q.shape[0],), torch.int32, q.device)
    with torch.cuda.device(q.device):
        st = lib.kda_spec_commit(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 _ptr(S), _ptr(accepted), _stream_handle(q.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_spec_commit")
    return S


def segment_summary(q, k, v, g, beta, cu_seqlens, cu_seqlens_host, S0=None, with_M: bool = True,
                    scale=None, g_floor: float = -5.0):
    """``kda_segment_summary``: the affine summary of each sequence piece,
    S_end = M S_start + S_loc.  q, k, g, v [T,H,128] bf16; beta [T,H];
    ``cu_seqlens`` int32 [N+1] on the GPU and its host copy.  Returns one fp32
    buffer [2,N,H,128,128]: [0] = S_loc (from S0 if given, else from zero),
    [1] = M (zeros when ``with_M`` is False).  The layout is what an
    all-gather of every rank's buffer hands to :func:`state_combine`."""
    _require_cuda()
    lib = load_library()
    device = q.device
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu_host = [int(x) for x in cu_seqlens_host]
    N = len(cu_host) - 1
    for name, t, shape in (("q", q, (T, H, dk)), ("k", k, (T, H, dk)), ("g", g, (T, H, dk)),
                           ("v", v, (T, H, dv)), ("beta", beta, (T, H))):
        _check(t, name, shape, q.dtype, device)
    _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, device)
    if S0 is not None:
        _check(S0, "S0", (N, H, dk, dv), torch.float32, device)
    desc = FwdDesc(total_tokens=T, num_seqs=N, num_heads=H, dk=dk, dv=dv, io_dtype=_io_dtype(q),
                   scale=float(dk ** -0.5 if scale is None else scale), g_floor=float(g_floor),
                   chunk=0, max_seqlen=0)
    cu_h = (ctypes.c_int32 * (N + 1))(*cu_host)
    ws_bytes = lib.kda_segment_summary_workspace_size(ctypes.byref(desc), cu_h, int(with_M))
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise KDAError(1, "kda_segment_summary_workspace_size")
    ws = torch.empty(max(int(ws_bytes), 256), dtype=torch.uint8, device=device)
    summ = torch.empty((2, N, H, dk, dv), dtype=torch.float32, device=device)
    if not with_M:
        summ[1].zero_()
    with torch.cuda.device(device):
        st = lib.kda_segment_summary(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                     _ptr(S0), ctypes.cast(_ptr(cu_seqlens), ctypes.POINTER(ctypes.c_int32)),
                                     cu_h, _ptr(summ[0]), _ptr(summ[1]) if with_M else None, _ptr(ws),
                                     ws.numel(), _stream_handle(device))
    if st != KDA_OK:
        raise KDAError(st, "kda_segment_summary")
    return summ


def state_combine(summaries, out=None):
    """``kda_state_combine``: folds P piece summaries [P,2,N,H,128,128] (fp32,
    in piece order) into the start state of piece P: S = S_loc(0), then
    S = M(p) S + S_loc(p).  Returns S_in fp32 [N,H,128,128]."""
    _require_cuda()
    lib = load_library()
    P, two, N, H, dk, dv = summaries.shape
    if two != 2:
        raise ValueError("summaries must be [P, 2, N, H, dk, dv]")
    _check(summaries, "summaries", tuple(summaries.shape), torch.float32, summaries.device)
    S_in = out if out is not None else torch.empty((N, H, dk, dv), dtype=torch.float32,
                                                   device=summaries.device)
    _check(S_in, "out", (N, H, dk, dv), torch.float32, summaries.device)
    desc = CombineDesc(num_seqs=N, num_heads=H, dk=dk, dv=dv, num_summaries=P)
    with torch.cuda.device(summaries.device):
        st = lib.kda_state_combine(ctypes.byref(desc), _ptr(summaries), _ptr(S_in),
                                   _stream_handle(summaries.device))
    if st != KDA_OK:
        raise KDAError(st, "kda_state_combine")
    return S_in


def chunk_fwd_host(q, k, v, g, beta, cu_seqlens_host, S0=None, gate=None, scale=None,
                   g_floor: float = -5.0, out=None, final_state_out=None, output_final_state=True,
                   device=None, workspace=None):
    """``kda_chunk_fwd_host``: the prefill of :func:`chunk_fwd` with inputs
    and outputs in host memory (CPU tensors, page-locked for the copies to
    overlap the compute), pipelined over groups of sequences.  Returns
    ``(o, S_T)`` as CPU tensors once the call's stream has been synchronised."""
    if not torch.cuda.is_available():
        raise RuntimeError("the KDA library needs a CUDA GPU (sm_100a); none is available")
    lib = load_library()
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    T, H, dk = q.shape
    dv = v.shape[-1]
    cu_host = [int(x) for x in cu_seqlens_host]
    N = len(cu_host) - 1
    cpu = torch.device("cpu")
    for name, t, shape in (("q", q, (T, H, dk)), ("k", k, (T, H, dk)), ("g", g, (T, H, dk)),
                           ("v", v, (T, H, dv)), ("beta", beta, (T, H))):
        if t.device != cpu or t.dtype != q.dtype or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor of shape {shape} and dtype {q.dtype}")
    if gate is not None and (gate.device != cpu or tuple(gate.shape) != (T, H, dv) or not gate.is_contiguous()):
        raise ValueError("gate must be a contiguous CPU tensor of v's shape")
    if S0 is not None and (S0.device != cpu or S0.dtype != torch.float32 or tuple(S0.shape) != (N, H, dk, dv)
                           or not S0.is_contiguous()):
        raise ValueError("S0 must be a contiguous fp32 CPU tensor [N,H,dk,dv]")
    o = out if out is not None else torch.empty((T, H, dv), dtype=q.dtype, pin_memory=True)
    S_T = None
    if output_final_state:
        S_T = (final_state_out if final_state_out is not None
               else torch.empty((N, H, dk, dv), dtype=torch.float32, pin_memory=True))
    desc = FwdDesc(total_tokens=T, num_seqs=N, num_heads=H, dk=dk, dv=dv, io_dtype=_io_dtype(q),
                   scale=float(dk ** -0.5 if scale is None else scale), g_floor=float(g_floor),
                   chunk=0, max_seqlen=0)
    cu_h = (ctypes.c_int32 * (N + 1))(*cu_host)
    ws_bytes = lib.kda_chunk_fwd_host_workspace_size(ctypes.byref(desc), cu_h, int(gate is not None),
                                                     int(S0 is not None), int(S_T is not None))
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise KDAError(1, "kda_chunk_fwd_host_workspace_size")
    ws = workspace
    if ws is None or ws.numel() < ws_bytes:
        ws = torch.empty(max(int(ws_bytes), 256), dtype=torch.uint8, device=device)
    with torch.cuda.device(device):
        stream = torch.cuda.current_stream(device)
        st = lib.kda_chunk_fwd_host(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                    _ptr(S0), cu_h, _ptr(gate), _ptr(o), _ptr(S_T), _ptr(ws), ws.numel(),
                                    ctypes.c_void_p(stream.cuda_stream))
        if st != KDA_OK:
            raise KDAError(st, "kda_chunk_fwd_host")
        stream.synchronize()
    return o, S_T


def chunk_bwd(q, k, v, g, beta, dout, cu_seqlens=None, cu_seqlens_host=None, S0=None, gate=None,
              dS_T=None, scale=None, g_floor: float = -5.0, want_dS0: bool = True):
    """``kda_chunk_bwd``: gradients of sum(o * dout) + sum(S_T * dS_T) through
    the prefill of :func:`chunk_fwd` (same inputs and layouts; dk, dv in {64, 128}).
    Returns a dict: dq, dk, dv, dg, dbeta (input dtype), dgate (if ``gate``)
    and dS0 (fp32 [N,H,dk,dv], if ``want_dS0``)."""
    _require_cuda()
    lib = load_library()
    device = q.device
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu_seqlens_host = [0, T]
        cu_seqlens = torch.tensor(cu_seqlens_host, dtype=torch.int32, device=device)
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu().tolist()
    cu_host = [int(x) for x in cu_seqlens_host]
    N = len(cu_host) - 1
    for name, t, shape in (("q", q, (T, H, dk)), ("k", k, (T, H, dk)), ("g", g, (T, H, dk)),
                           ("v", v, (T, H, dv)), ("beta", beta, (T, H)), ("dout", dout, (T, H, dv))):
        _check(t, name, shape, q.dtype, device)
    if gate is not None:
        _check(gate, "gate", (T, H, dv), q.dtype, device)
    _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, device)
    for name, t in (("S0", S0), ("dS_T", dS_T)):
        if t is not None:
            _check(t, name, (N, H, dk, dv), torch.float32, device)
    desc = FwdDesc(total_tokens=T, num_seqs=N, num_heads=H, dk=dk, dv=dv, io_dtype=_io_dtype(q),
                   scale=float(dk ** -0.5 if scale is None else scale), g_floor=float(g_floor),
                   chunk=0, max_seqlen=0)
    cu_h = (ctypes.c_int32 * (N + 1))(*cu_host)
    ws_bytes = lib.kda_chunk_bwd_workspace_size(ctypes.byref(desc), cu_h)
    if ws_bytes == ctypes.c_size_t(-1).value:
        raise KDAError(1, "kda_chunk_bwd_workspace_size")
    ws = torch.empty(max(int(ws_bytes), 256), dtype=torch.uint8, device=device)
    out = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "dg": torch.empty_like(g), "dbeta": torch.empty_like(beta)}
    if gate is not None:
        out["dgate"] = torch.empty_like(gate)
    if want_dS0:
        out["dS0"] = torch.empty((N, H, dk, dv), dtype=torch.float32, device=device)
    with torch.cuda.device(device):
        st = lib.kda_chunk_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                               _ptr(S0), ctypes.cast(_ptr(cu_seqlens), ctypes.POINTER(ctypes.c_int32)),
                               cu_h, _ptr(gate), _ptr(dout), _ptr(dS_T), _ptr(out["dq"]),
                               _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
                               _ptr(out.get("dgate")), _ptr(out.get("dS0")), _ptr(ws), ws.numel(),
                               _stream_handle(device))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_bwd")
    return out


def device_status(device=None) -> int:
    """Synchronise the current stream and read/clear the device error word."""
    _require_cuda()
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib.kda_get_device_status(_stream_handle(dev)))


def selftest_bounded_wait(max_polls: int = 1024, device=None) -> int:
    """``kda_selftest_bounded_wait``: one bounded device-side wait that runs out
    (nothing completes its barrier); returns the launch status.  The timeout it
    records is read, and cleared, by :func:`device_status`."""
    _require_cuda()
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib.kda_selftest_bounded_wait(int(max_polls), _stream_handle(dev)))


def _noalloc_fn(lib):
    f = lib.kda_chunk_fwd_noalloc
    if f.restype is not ctypes.c_int:
        vp = ctypes.c_void_p
        f.argtypes = [ctypes.POINTER(FwdDesc), vp, vp, vp, vp, vp, vp,
                      ctypes.POINTER(ctypes.c_int32), vp, vp, vp, vp]
        f.restype = ctypes.c_int
    return f


def chunk_fwd_noalloc(q, k, v, g, beta, cu_seqlens, S0=None, scale=None, gate=None,
                      g_floor: float = -5.0, out=None, final_state_out=None):
    """``kda_chunk_fwd_noalloc``: the chunked prefill for callers that cannot
    give the library device memory of its own (its per-call scratch is a fixed
    array inside the library, for up to ``NOALLOC_MAX_SEQS`` sequences).

    Packed inputs only: q, k, g [T,H,dk]; v, gate [T,H,dv]; beta [T,H];
    ``cu_seqlens`` int32 [N+1] on the GPU.  ``out`` / ``final_state_out`` may
    be passed to keep this call free of any allocation; when omitted they are
    allocated here with PyTorch.  Returns ``(o, S_T)``.
    """
    _require_cuda()
    lib = load_library()
    T, H, dk = q.shape
    dv = v.shape[-1]
    device, dtype = q.device, q.dtype
    N = cu_seqlens.numel() - 1
    for t, name, shape in ((q, "q", (T, H, dk)), (k, "k", (T, H, dk)), (g, "g", (T, H, dk)),
                           (v, "v", (T, H, dv)), (beta, "beta", (T, H))):
        _check(t, name, shape, dtype, device)
    if gate is not None:
        _check(gate, "gate", (T, H, dv), dtype, device)
    if S0 is not None:
        _check(S0, "S0", (N, H, dk, dv), torch.float32, device)
    _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, device)
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    o = out if out is not None else torch.empty((T, H, dv), dtype=dtype, device=device)
    S_T = (final_state_out if final_state_out is not None
           else torch.empty((N, H, dk, dv), dtype=torch.float32, device=device))
    desc = FwdDesc(T, N, H, dk, dv, _io_dtype(q), float(scale), float(g_floor), 0, 0)
    with torch.cuda.device(device):
        st = _noalloc_fn(lib)(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                              _ptr(S0), ctypes.cast(ctypes.c_void_p(cu_seqlens.data_ptr()),
                                                    ctypes.POINTER(ctypes.c_int32)),
                              _ptr(gate), _ptr(o), _ptr(S_T), _stream_handle(device))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_noalloc")
    return o, S_T
