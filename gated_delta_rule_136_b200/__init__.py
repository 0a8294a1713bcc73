"""B200-native (sm_100a) Kimi Delta Attention forward: chunked prefill and
in-place decode behind a C ABI (``include/kda.h``), with a thin PyTorch
binding.  See ``kda.chunk_fwd`` and ``kda.decode_step``."""
from .kda import (KDAError, chunk_fwd, chunk_fwd_snapshots, decode_step, device_status,  # noqa: F401
                  load_library, selftest_bounded_wait, spec_commit, spec_verify, workspace_size)

__all__ = ["chunk_fwd", "chunk_fwd_snapshots", "decode_step", "device_status", "load_library", "workspace_size",
           "selftest_bounded_wait", "spec_verify", "spec_commit", "KDAError"]
