"""The C-ABI library builds, loads and exports every symbol include/kda.h
declares; host-side validation rejects bad arguments before any launch.
CPU only: every call here fails validation by construction, so nothing is
ever launched (the fake pointers below are never dereferenced)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_136_b200 import kda

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    return kda.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    assert set(declared_functions()) == set(kda.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    for code, name in kda.STATUS_NAMES.items():
        assert lib.kda_status_string(code).decode() == name
    assert lib.kda_status_string(99).decode() == "KDA_UNKNOWN_STATUS"
    assert lib.kda_version() >= 100


def _desc(**kw):
    base = dict(total_tokens=64, num_seqs=1, num_heads=2, dk=128, dv=128, io_dtype=kda.KDA_BF16,
                scale=0.0883883, g_floor=-5.0, chunk=0, max_seqlen=0)
    base.update(kw)
    return kda.FwdDesc(**base)


SIZE_MAX = ctypes.c_size_t(-1).value


@pytest.mark.parametrize("bad", [dict(num_seqs=0), dict(num_heads=0), dict(total_tokens=-1),
                                 dict(dk=0), dict(io_dtype=7), dict(g_floor=-6.0),
                                 dict(g_floor=0.5), dict(chunk=32), dict(scale=float("nan")),
                                 dict(dk=96), dict(dv=256), dict(max_seqlen=-1)])
def test_workspace_size_rejects_bad_desc(lib, bad):
    d = _desc(**bad)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(d), None) == SIZE_MAX


def test_workspace_size_valid_and_aligned(lib):
    d = _desc(num_seqs=3)
    n = lib.kda_chunk_fwd_workspace_size(ctypes.byref(d), None)
    assert n % 256 == 0 and n >= 12


def test_workspace_size_checks_host_seqlens(lib):
    d = _desc(num_seqs=2, total_tokens=10)
    good = (ctypes.c_int32 * 3)(0, 4, 10)
    assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(d), good) != SIZE_MAX
    for vals in ((1, 4, 10), (0, 6, 5), (0, 4, 9)):
        arr = (ctypes.c_int32 * 3)(*vals)
        assert lib.kda_chunk_fwd_workspace_size(ctypes.byref(d), arr) == SIZE_MAX


# Fake, never-dereferenced device addresses: every call below fails validation.
A = 0x10000000
MB = 1 << 20


def _fwd(lib, desc, q=A, k=A + 4 * MB, v=A + 8 * MB, g=A + 12 * MB, beta=A + 16 * MB, S0=None,
         cu=A + 20 * MB, cu_host=None, gate=None, o=A + 24 * MB, S_T=None, ws=A + 64 * MB,
         ws_bytes=1 << 20):
    cu_p = ctypes.cast(ctypes.c_void_p(cu), ctypes.POINTER(ctypes.c_int32)) if cu else None
    return lib.kda_chunk_fwd(ctypes.byref(desc), q, k, v, g, beta, S0, cu_p, cu_host, gate, o,
                             S_T, ws, ws_bytes, None)


def test_fwd_rejects_null_required_pointers(lib):
    d = _desc()
    for field in ("q", "k", "v", "g", "beta", "o", "cu"):
        assert _fwd(lib, d, **{field: None}) == 1, field


def test_fwd_rejects_overlapping_output(lib):
    d = _desc()
    assert _fwd(lib, d, o=A + 1024) == 1                      # o inside q
    assert _fwd(lib, d, S_T=A + 12 * MB + 64) == 1            # S_T inside g
    assert _fwd(lib, d, S0=A + 40 * MB, S_T=A + 40 * MB + 4096) == 1   # S_T overlaps S0
    assert _fwd(lib, d, ws=A + 8 * MB) == 1                   # workspace inside v


def test_fwd_rejects_workspace_problems(lib):
    d = _desc()
    assert _fwd(lib, d, ws=None) == 3
    assert _fwd(lib, d, ws_bytes=16) == 3
    assert _fwd(lib, d, ws=A + 64 * MB + 8) == 3              # not 256-byte aligned


def test_fwd_rejects_bad_host_seqlens(lib):
    d = _desc(num_seqs=2, total_tokens=10)
    assert _fwd(lib, d, cu_host=(ctypes.c_int32 * 3)(0, 7, 3)) == 1
    assert _fwd(lib, d, cu_host=(ctypes.c_int32 * 3)(0, 3, 11)) == 1


def test_fwd_unsupported_head_dim(lib):
    assert _fwd(lib, _desc(dk=96)) == 2
    assert _fwd(lib, _desc(dv=32)) == 2


def _dec(lib, desc, q=A, k=A + MB, v=A + 2 * MB, g=A + 3 * MB, beta=A + 4 * MB, S=A + 8 * MB,
         gate=None, o=A + 40 * MB):
    return lib.kda_decode_step(ctypes.byref(desc), q, k, v, g, beta, S, gate, o, None)


def test_decode_validation(lib):
    good = dict(batch=4, num_heads=2, dk=128, dv=128, io_dtype=kda.KDA_BF16, scale=0.09,
                g_floor=-5.0)
    for bad in (dict(batch=0), dict(num_heads=0), dict(g_floor=-7.0), dict(io_dtype=3)):
        assert _dec(lib, kda.DecodeDesc(**{**good, **bad})) == 1, bad
    assert _dec(lib, kda.DecodeDesc(**{**good, "dk": 80})) == 2
    d = kda.DecodeDesc(**good)
    for field in ("q", "k", "v", "g", "beta", "S", "o"):
        assert _dec(lib, d, **{field: None}) == 1, field
    assert _dec(lib, d, o=A + 8 * MB + 256) == 1      # o inside S
    assert _dec(lib, d, S=A + 8 * MB + 4) == 1        # S not 16-byte aligned
    assert _dec(lib, d, gate=A + 8 * MB) == 1         # gate inside S


@pytest.mark.parametrize("polls", [0, -1, 65537])
def test_selftest_rejects_bad_poll_counts(lib, polls):
    """Checked on the host before any launch, so this runs without a GPU."""
    assert lib.kda_selftest_bounded_wait(polls, None) == 1   # KDA_ERR_INVALID_ARG


def _snapfwd(lib, desc, snap, cu_host=None, o=A + 24 * MB):
    cu_p = ctypes.cast(ctypes.c_void_p(A + 20 * MB), ctypes.POINTER(ctypes.c_int32))
    return lib.kda_chunk_fwd_snapshots(ctypes.byref(desc), ctypes.byref(snap) if snap else None,
                                       A, A + 4 * MB, A + 8 * MB, A + 12 * MB, A + 16 * MB, None,
                                       cu_p, cu_host, None, o, None, A + 64 * MB, 1 << 20, None)


def test_snapshots_validation(lib):
    """Rejected on the host before any launch (fake pointers never touched)."""
    d = _desc(num_seqs=2, total_tokens=300)
    cu_host = (ctypes.c_int32 * 3)(0, 200, 300)           # 200 // 64 + 100 // 64 = 4 slots needed
    ok = dict(interval=64, total=4, base=A + 80 * MB, states=A + 96 * MB)
    assert _snapfwd(lib, d, None) == 1                                      # no descriptor
    for bad in (dict(interval=0), dict(interval=32), dict(interval=-64), dict(total=-1),
                dict(states=None), dict(base=None),
                dict(total=3),                                              # fewer slots than needed
                dict(states=A + 8 * MB),                                    # states inside v
                dict(base=A + 24 * MB),                                     # base inside o
                dict(states=A + 64 * MB)):                                  # states inside workspace
        snap = kda.Snapshots(**{**ok, **bad})
        assert _snapfwd(lib, d, snap, cu_host) == 1, bad


def _spec(**kw):
    base = dict(batch=2, num_heads=2, dk=128, dv=128, draft=4, io_dtype=kda.KDA_BF16, scale=0.09,
                g_floor=-5.0)
    base.update(kw)
    return kda.SpecDesc(**base)


def _verify(lib, desc, S=A + 40 * MB, o=A + 48 * MB, gate=None):
    return lib.kda_spec_verify(ctypes.byref(desc), A, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB,
                               S, gate, o, None)


def _commit(lib, desc, S=A + 40 * MB, acc=A + 56 * MB):
    return lib.kda_spec_commit(ctypes.byref(desc), A, A + MB, A + 2 * MB, A + 3 * MB, A + 4 * MB,
                               S, acc, None)


def test_spec_validation(lib):
    """Rejected on the host before any launch (fake pointers never touched)."""
    for bad in (dict(draft=0), dict(draft=kda.SPEC_MAX_DRAFT + 1), dict(batch=0),
                dict(io_dtype=5), dict(g_floor=-7.0), dict(scale=float("inf"))):
        assert _verify(lib, _spec(**bad)) == 1, bad
        assert _commit(lib, _spec(**bad)) == 1, bad
    assert _verify(lib, _spec(dk=96)) == 2
    assert _verify(lib, _spec(), o=None) == 1                  # verify needs outputs
    assert _commit(lib, _spec(), acc=None) == 1                # commit needs the counts
    assert _verify(lib, _spec(), S=A + 2 * MB) == 1            # S inside v
    assert _verify(lib, _spec(), o=A + 40 * MB + 64) == 1      # o inside S
    assert _commit(lib, _spec(), S=A + 40 * MB + 8) == 1       # S not 16-byte aligned
    assert _commit(lib, _spec(), acc=A + 40 * MB + 4096) == 1  # counts inside S


def _summary(lib, desc, S_loc=A + 40 * MB, M=A + 48 * MB, S0=None, cu_host=None, ws=A + 64 * MB,
             ws_bytes=1 << 20, q=A):
    cu_p = ctypes.cast(ctypes.c_void_p(A + 20 * MB), ctypes.POINTER(ctypes.c_int32))
    if cu_host is None:
        cu_host = (ctypes.c_int32 * 2)(0, desc.total_tokens)
    return lib.kda_segment_summary(ctypes.byref(desc), q, A + 4 * MB, A + 8 * MB, A + 12 * MB,
                                   A + 16 * MB, S0, cu_p, cu_host, S_loc, M, ws, ws_bytes, None)


def test_segment_summary_validation(lib):
    """Rejected on the host before any launch (fake pointers never touched)."""
    d = _desc()
    cu1 = (ctypes.c_int32 * 2)(0, 64)
    assert lib.kda_segment_summary_workspace_size(ctypes.byref(_desc(num_heads=0)), cu1, 1) == SIZE_MAX
    assert lib.kda_segment_summary_workspace_size(ctypes.byref(d), None, 1) == SIZE_MAX
    assert lib.kda_segment_summary_workspace_size(ctypes.byref(d), cu1, 1) % 256 == 0
    assert _summary(lib, _desc(io_dtype=kda.KDA_FP32)) == 2          # tensor-core shape only
    assert _summary(lib, _desc(dk=64)) == 2
    assert _summary(lib, _desc(chunk=16)) == 2
    assert _summary(lib, _desc(total_tokens=0)) == 1
    assert _summary(lib, d, S_loc=None) == 1
    assert lib.kda_segment_summary(ctypes.byref(d), A, A + 4 * MB, A + 8 * MB, A + 12 * MB,
                                   A + 16 * MB, None, None, (ctypes.c_int32 * 2)(0, 64),
                                   A + 40 * MB, None, A + 64 * MB, 1 << 20, None) == 1   # no cu_seqlens
    assert lib.kda_segment_summary(ctypes.byref(d), A, A + 4 * MB, A + 8 * MB, A + 12 * MB,
                                   A + 16 * MB, None,
                                   ctypes.cast(ctypes.c_void_p(A + 20 * MB), ctypes.POINTER(ctypes.c_int32)),
                                   None, A + 40 * MB, None, A + 64 * MB, 1 << 20, None) == 1  # no host copy
    assert _summary(lib, d, cu_host=(ctypes.c_int32 * 2)(0, 63)) == 1    # host seqlens disagree
    assert _summary(lib, d, q=A + 8) == 1                                 # q not 16-byte aligned
    assert _summary(lib, d, S_loc=A + 4 * MB + 64) == 1                   # S_loc inside k
    assert _summary(lib, d, M=A + 40 * MB + 4096) == 1                    # M overlaps S_loc
    assert _summary(lib, d, ws=None) == 3
    assert _summary(lib, d, ws_bytes=8) == 3
    assert _summary(lib, d, ws=A + 64 * MB + 16) == 3                     # not 256-byte aligned
    assert _summary(lib, d, ws=A + 40 * MB) == 1                          # workspace on S_loc


def test_state_combine_validation(lib):
    ok = dict(num_seqs=2, num_heads=2, dk=128, dv=128, num_summaries=3)
    S_in = A + 200 * MB
    for bad in (dict(num_seqs=0), dict(num_heads=0), dict(num_summaries=0), dict(dk=0)):
        assert lib.kda_state_combine(ctypes.byref(kda.CombineDesc(**{**ok, **bad})), A, S_in, None) == 1
    assert lib.kda_state_combine(ctypes.byref(kda.CombineDesc(**{**ok, "dk": 64, "dv": 64})), A, S_in,
                                 None) == 2
    d = kda.CombineDesc(**ok)
    assert lib.kda_state_combine(ctypes.byref(d), None, S_in, None) == 1
    assert lib.kda_state_combine(ctypes.byref(d), A, None, None) == 1
    assert lib.kda_state_combine(ctypes.byref(d), A + 4, S_in, None) == 1     # misaligned
    assert lib.kda_state_combine(ctypes.byref(d), A, A + MB, None) == 1        # S_in inside summaries


def test_chunk_bwd_validation(lib):
    """Rejected on the host before any launch (fake pointers never touched)."""
    d = _desc(total_tokens=64)
    cu_host = (ctypes.c_int32 * 2)(0, 64)
    assert lib.kda_chunk_bwd_workspace_size(ctypes.byref(d), None) == SIZE_MAX
    need = lib.kda_chunk_bwd_workspace_size(ctypes.byref(d), cu_host)
    assert need != SIZE_MAX and need % 256 == 0
    cu_p = ctypes.cast(ctypes.c_void_p(A + 20 * MB), ctypes.POINTER(ctypes.c_int32))

    def bwd(desc=d, cu_h=cu_host, dout=A + 30 * MB, dq=A + 32 * MB, gate=None, dgate=None, S0=None,
            dS0=None, ws=A + 256 * MB, ws_bytes=1 << 34):
        return lib.kda_chunk_bwd(ctypes.byref(desc), A, A + 4 * MB, A + 8 * MB, A + 12 * MB, A + 16 * MB,
                                 S0, cu_p, cu_h, gate, dout, None, dq, A + 34 * MB, A + 36 * MB,
                                 A + 38 * MB, A + 40 * MB, dgate, dS0, ws, ws_bytes, None)
    assert bwd(desc=_desc(total_tokens=64, dk=96)) == 2                 # head size outside {64, 128}
    assert bwd(cu_h=None) == 1
    assert bwd(dout=None) == 1
    assert bwd(dq=A + 4 * MB + 64) == 1                     # dq inside k
    assert bwd(gate=A + 50 * MB) == 1                       # gate without dgate
    assert bwd(S0=A + 60 * MB + 4) == 1                     # S0 not 16-byte aligned
    assert bwd(dS0=A + 32 * MB) == 1                        # dS0 on dq
    assert bwd(ws=None) == 3
    assert bwd(ws_bytes=need - 256) == 3
    assert bwd(ws=A + 8 * MB) == 1                          # workspace on v


def test_chunk_fwd_host_validation(lib):
    """Rejected on the host before any copy or launch (fake pointers never touched)."""
    d = _desc(num_seqs=2, total_tokens=10)
    cu_host = (ctypes.c_int32 * 3)(0, 4, 10)
    assert lib.kda_chunk_fwd_host_workspace_size(ctypes.byref(_desc(num_heads=0)), cu_host, 0, 0, 1) == SIZE_MAX
    assert lib.kda_chunk_fwd_host_workspace_size(ctypes.byref(d), None, 0, 0, 1) == SIZE_MAX
    full = lib.kda_chunk_fwd_host_workspace_size(ctypes.byref(d), cu_host, 1, 1, 1)
    need = lib.kda_chunk_fwd_host_workspace_size(ctypes.byref(d), cu_host, 0, 0, 0)   # as called below
    assert need != SIZE_MAX and need % 256 == 0 and full > need

    def host(desc=d, cu_h=cu_host, ws=A + 256 * MB, ws_bytes=need, o=A + 24 * MB):
        return lib.kda_chunk_fwd_host(ctypes.byref(desc), A, A + 4 * MB, A + 8 * MB, A + 12 * MB, A + 16 * MB,
                                      None, cu_h, None, o, None, ws, ws_bytes, None)
    assert host(cu_h=None) == 1
    assert host(cu_h=(ctypes.c_int32 * 3)(0, 4, 9)) == 1          # disagrees with total_tokens
    assert host(o=None) == 1
    assert host(desc=_desc(num_seqs=2, total_tokens=10, io_dtype=5)) == 1
    assert host(ws=None) == 3
    assert host(ws_bytes=need - 256) == 3
    assert host(ws=A + 256 * MB + 64) == 3                           # not 256-byte aligned


def _in_subprocess_env(env, code):
    """Run `code` (prints one integer) with extra environment variables: the
    planners read KDA_SEGMENTS when they run, so each case gets a fresh process."""
    import subprocess
    import sys
    out = subprocess.run([sys.executable, "-c", code], env={**os.environ, **env}, capture_output=True,
                         text=True, check=True, cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    return int(out.stdout.strip().splitlines()[-1])


_SUMMARY_WS = """
import ctypes
from gated_delta_rule_136_b200 import kda
lib = kda.load_library()
lengths = {lengths}
cu = [0]
for L in lengths: cu.append(cu[-1] + L)
d = kda.FwdDesc(total_tokens=cu[-1], num_seqs=len(lengths), num_heads={H}, dk=128, dv=128, io_dtype=kda.KDA_BF16,
                scale=0.088, g_floor=-5.0, chunk=0, max_seqlen=0)
print(lib.kda_segment_summary_workspace_size(ctypes.byref(d), (ctypes.c_int32 * len(cu))(*cu), 1))
"""


def test_summary_split_plan_sizes():
    """Host planning of the piece summary (no GPU: 148 SMs assumed).  A long
    piece with few heads is split (its sub-segment matrices need workspace);
    KDA_SEGMENTS=1 keeps one chain; forced counts that differ per sequence
    are sized by their sum."""
    DD = 128 * 128 * 4
    auto = _in_subprocess_env({}, _SUMMARY_WS.format(lengths=[131072], H=32))
    whole = _in_subprocess_env({"KDA_SEGMENTS": "1"}, _SUMMARY_WS.format(lengths=[131072], H=32))
    assert whole < DD and auto >= 32 * 2 * 2 * DD                  # at least 2 sub-segments each
    mixed = _in_subprocess_env({"KDA_SEGMENTS": "3"}, _SUMMARY_WS.format(lengths=[300, 1300], H=3))
    assert mixed >= (3 * 2 + 3 * 3) * 2 * DD                        # P = 2 and 3, S_loc and M each


def test_library_carries_nvtx_ranges():
    """The host code marks its launch sequences with NVTX ranges (plan, the
    split's two passes and scan, prefill, decode, speculative verify/commit,
    backward, summary, combine, host pipeline), so a profiler attached to the
    process can attribute kernels; the range names are compiled into the
    library."""
    blob = open(kda.library_path(), "rb").read()
    for name in ("kda.plan", "kda.prefill", "kda.split.pass1", "kda.split.scan", "kda.split.pass2",
                 "kda.decode", "kda.spec.verify", "kda.spec.commit", "kda.bwd", "kda.summary.chains",
                 "kda.summary.scan", "kda.combine", "kda.host.group", "kda.prefill.noalloc"):
        assert name.encode() + b"\0" in blob, name
