"""Python binding of libmmsp.so: ring-blockwise causal attention (the MM-SP
hot path) on one B200.

Argument marshalling only: every step runs in the CUDA kernels behind the C
ABI (include/mmsp.h). The functions keep the C names and accept torch CUDA
tensors (or raw device pointers as ints). There is no fallback: importing
fails loudly when the shared library has not been built.
"""
from ._binding import (  # noqa: F401
    MMSP_ACCUMULATE,
    MMSP_FINALIZE,
    MMSP_MAX_SEGMENTS,
    MmspError,
    STATUS,
    lib_path,
    mmsp_attn_bwd,
    mmsp_attn_bwd_noalloc,
    mmsp_attn_bwd_prepare,
    mmsp_attn_bwd_dkdv,
    mmsp_attn_bwd_dq,
    MMSP_NOALLOC_SCRATCH_BYTES,
    mmsp_attn_fwd,
    mmsp_bwd_workspace_bytes,
    mmsp_device_status,
    mmsp_doc_starts,
    mmsp_last_error,
    mmsp_lse_merge,
    mmsp_selftest_bounded_wait,
    mmsp_shard,
    mmsp_shard_rope,
    mmsp_shard_frames,
    mmsp_gather_rows,
    mmsp_ulysses_transpose,
    mmsp_version,
    exported_symbols,
)
