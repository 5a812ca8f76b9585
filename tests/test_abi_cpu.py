"""The C-ABI library loads and exports every symbol include/mmsp.h declares;
host-side validation rejects bad arguments before any launch (CPU only: no
compute call reaches the GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "mmsp.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mmsp_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import long_context_multimodal_b200 as m

    names = _header_functions()
    assert "mmsp_attn_fwd" in names and "mmsp_shard" in names and len(names) >= 9
    lib = ctypes.CDLL(m.lib_path())
    for n in names:
        assert hasattr(lib, n), n
    assert set(m.exported_symbols()) == set(names)
    assert "sm_100a" in m.mmsp_version()


def _einval(fn, *a, **k):
    import long_context_multimodal_b200 as m

    with pytest.raises(m.MmspError) as e:
        fn(*a, **k)
    assert e.value.status == 1, str(e.value)
    return str(e.value)


def test_attn_fwd_rejects_bad_arguments():
    import long_context_multimodal_b200 as m

    F = m.mmsp_attn_fwd
    p = 1 << 20  # a 16-byte-aligned stand-in pointer; nothing is launched
    ok = dict(q=p, k=p, v=p, N=4096, P=4, Hq=4, Hkv=4, d=64, scale=0.125, causal=1, step_begin=0, step_end=4,
              o_acc=p, lse=p, o_out=p, flags=m.MMSP_FINALIZE)
    for bad in [dict(N=4095), dict(N=4100, P=4), dict(P=0), dict(N=-2), dict(Hq=6, Hkv=4), dict(d=96),
                dict(d=256), dict(step_begin=3, step_end=2), dict(step_end=5), dict(q=p + 8), dict(lse=None),
                dict(scale=0.0), dict(scale=float("nan")), dict(causal=2), dict(flags=8),
                dict(flags=m.MMSP_ACCUMULATE, o_acc=None), dict(o_out=None), dict(N=1 << 31, P=1),
                dict(rank_begin=0, rank_end=0), dict(rank_begin=2, rank_end=1), dict(rank_begin=-1),
                dict(rank_end=5)]:
        args = dict(ok, **bad)
        _einval(F, **args)


def test_backward_stages_reject_bad_rank_ranges():
    import long_context_multimodal_b200 as m

    p = 1 << 20
    N, P, hq, hkv, d = 4096, 4, 4, 4, 128
    wsb = m.mmsp_bwd_workspace_bytes(N, P, hq, d)
    for rb, re in ((0, 0), (3, 2), (-1, 2), (0, 5)):
        msg = _einval(m.mmsp_attn_bwd_prepare, p, p, p, N, P, hq, d, p, wsb, rank_begin=rb, rank_end=re)
        assert "rank_begin" in msg
        _einval(m.mmsp_attn_bwd_dkdv, p, p, p, p, N, P, hq, hkv, d, 0.088, 1, p, p, p, wsb, rank_begin=rb,
                rank_end=re)
        _einval(m.mmsp_attn_bwd_dq, p, p, p, p, N, P, hq, hkv, d, 0.088, 1, p, None, p, wsb, rank_begin=rb,
                rank_end=re)


def test_shard_rejects_bad_arguments():
    import long_context_multimodal_b200 as m

    p = 1 << 20
    _einval(m.mmsp_shard, None, None, 10, 3)                                   # N % 2P
    _einval(m.mmsp_shard, [5, 4], [0, 1], 8, 2, local2global=p, modality_local=p)  # sum != N
    _einval(m.mmsp_shard, [8], [2], 8, 2, modality_local=p)                   # bad kind
    _einval(m.mmsp_shard, [0, 8], [0, 0], 8, 2, segid_local=p)               # empty segment
    _einval(m.mmsp_shard, None, None, 8, 2, modality_local=p)                 # table missing
    _einval(m.mmsp_shard, np.ones(4097, np.int32), np.zeros(4097, np.uint8), 4097 * 2, 1,
            rank_counts=p)                                                     # over capacity
    _einval(m.mmsp_shard, None, None, 8, 2, src=p, dst=None)                  # half a permute
    _einval(m.mmsp_shard, None, None, 8, 2, src=p, dst=p + 4096, row_bytes=6)  # row_bytes % 4
    _einval(m.mmsp_shard, None, None, 8, 2, src=p + 4, dst=p + 4096, row_bytes=32)  # misaligned
    _einval(m.mmsp_shard, None, None, 8, 2, src=p, dst=p + 64, row_bytes=16)  # overlap


def test_merge_and_bwd_reject_bad_arguments():
    import long_context_multimodal_b200 as m

    p = 1 << 20
    _einval(m.mmsp_lse_merge, p, p, p, p, p, p, 10, 2, 96)
    _einval(m.mmsp_lse_merge, p + 4, p, p, p, p, p, 10, 2, 64)
    _einval(m.mmsp_lse_merge, p, p, p, p, p, p, -1, 2, 64)
    _einval(m.mmsp_selftest_bounded_wait, 0)
    # backward stages validate their own arguments
    _einval(m.mmsp_attn_bwd_prepare, p, p, p, 4096, 4, 28, 128, None, 0)
    _einval(m.mmsp_attn_bwd_dkdv, p, p, p, p, 4096, 4, 28, 5, 128, 0.1, 1, p, p, p, 1 << 30)
    _einval(m.mmsp_attn_bwd_dq, p, p, p, p, 4095, 4, 28, 4, 128, 0.1, 1, p, None, p, 1 << 30)
    _einval(m.mmsp_attn_bwd_dq, p, p, p, p, 4096, 4, 28, 4, 128, 0.1, 1, p + 4, None, p, 1 << 30)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The binding has no fallback: a missing .so is an ImportError."""
    import importlib.util
    import shutil

    pkg = os.path.join(ROOT, "long_context_multimodal_b200")
    dst = tmp_path / "pkgcopy"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    spec = importlib.util.spec_from_file_location("pkgcopy", dst / "__init__.py",
                                                  submodule_search_locations=[str(dst)])
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_documents_and_rope_reject_bad_arguments():
    import long_context_multimodal_b200 as m

    p = 1 << 20
    # document starts: table must be valid and sum to N
    _einval(m.mmsp_doc_starts, [4, 4], 16, p)                     # sums to 8, not 16
    _einval(m.mmsp_doc_starts, [8, 0, 8], 16, p)                  # empty document
    _einval(m.mmsp_doc_starts, [16], 16, p + 2)                   # misaligned output
    _einval(m.mmsp_doc_starts, np.ones(4097, np.int32), 4097, p)  # over capacity
    # doc_start on the attention calls needs causal attention and alignment
    ok = dict(q=p, k=p, v=p, N=4096, P=4, Hq=4, Hkv=4, d=64, scale=0.125, causal=1, step_begin=0, step_end=4,
              o_acc=p, lse=p, o_out=p, flags=m.MMSP_FINALIZE)
    _einval(m.mmsp_attn_fwd, **dict(ok, causal=0), doc_start=p)
    _einval(m.mmsp_attn_fwd, **ok, doc_start=p + 2)
    ws = m.mmsp_bwd_workspace_bytes(4096, 4, 4, 128)
    _einval(m.mmsp_attn_bwd, p, p, p, p, p, p, 4096, 4, 4, 4, 128, 0.088, 0, p, p, p, None, p, ws, doc_start=p)
    # RoPE gather: head size, base, flags, alignment, overlap, sharding
    R = m.mmsp_shard_rope
    _einval(R, p, p + (1 << 24), 64, 2, 2, 48)                    # d not supported
    _einval(R, p, p + (1 << 24), 64, 2, 2, 512)
    _einval(R, p, p + (1 << 24), 64, 2, 2, 64, theta=1.0)         # base must exceed 1
    _einval(R, p, p + (1 << 24), 64, 2, 2, 64, theta=float("nan"))
    _einval(R, p, p + (1 << 24), 64, 3, 2, 64)                    # N % 2P
    _einval(R, p, p + (1 << 24), 64, 2, 0, 64)                    # no heads
    _einval(R, p + 8, p + (1 << 24), 64, 2, 2, 64)                # misaligned
    _einval(R, p, p + 64, 64, 2, 2, 64)                           # overlapping rows
    _einval(R, p, p + (1 << 24), 64, 2, 2, 64, doc_start=p + 1)   # misaligned document starts
