"""B200-native (sm_100a) Kimi Delta Attention forward: chunked prefill and
in-place decode behind a C ABI (``include/kda.h``), with a thin PyTorch
binding.  See ``kda.chunk_fwd`` and ``kda.decode_step``; ``kcp.kcp_chunk_fwd``
runs one long sequence context-parallel across the ranks of a process group."""
from .kda import (KDAError, chunk_bwd, chunk_fwd, chunk_fwd_host, chunk_fwd_snapshots, decode_step, device_status,  # noqa: F401
                  load_library, segment_summary, selftest_bounded_wait, spec_commit, spec_verify,
                  state_combine, workspace_size)
from .kcp import kcp_chunk_fwd, split_pieces  # noqa: F401

__all__ = ["chunk_fwd", "chunk_fwd_host", "chunk_bwd", "chunk_fwd_snapshots", "decode_step", "device_status", "load_library", "workspace_size",
           "selftest_bounded_wait", "spec_verify", "spec_commit", "segment_summary", "state_combine",
           "kcp_chunk_fwd", "split_pieces", "KDAError"]
