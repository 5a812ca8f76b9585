"""ctypes marshalling for libmmsp.so. Same names and argument order as the C
ABI in include/mmsp.h; tensors are passed by device pointer."""
from __future__ import annotations

import ctypes
import os
from ctypes import c_float, c_int32, c_int64, c_size_t, c_uint32, c_void_p

import numpy as np

MMSP_ACCUMULATE = 1
MMSP_FINALIZE = 2
MMSP_MAX_SEGMENTS = 4096
STATUS = {0: "MMSP_OK", 1: "MMSP_EINVAL", 2: "MMSP_EUNSUPPORTED", 3: "MMSP_ECUDA", 4: "MMSP_ETIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.path.join(_HERE, "libmmsp.so")


class MmspError(RuntimeError):
    def __init__(self, func: str, status: int, message: str):
        self.status = status
        super().__init__(f"{func} -> {STATUS.get(status, status)}: {message}")


def _load():
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build the CUDA library first "
            "(python long_context_multimodal_b200/build.py). There is no CPU fallback.")
    return ctypes.CDLL(path)


_lib = _load()

_SIGS = {
    "mmsp_shard": ([c_void_p, c_void_p, c_int32, c_int64, c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                    c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_void_p], c_int32),
    "mmsp_attn_fwd": ([c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_int32, c_int32, c_int32, c_float,
                       c_int32, c_int32, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_uint32, c_void_p,
                       c_void_p], c_int32),
    "mmsp_doc_starts": ([c_void_p, c_int32, c_int64, c_void_p, c_void_p], c_int32),
    "mmsp_shard_rope": ([c_void_p, c_void_p, c_int64, c_int32, c_int32, c_int32, ctypes.c_double, c_int32, c_void_p,
                         c_int32, c_void_p], c_int32),
    "mmsp_lse_merge": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_int32,
                        c_void_p], c_int32),
    "mmsp_shard_frames": ([c_void_p, c_void_p, c_int32, c_int64, c_int32, c_void_p, c_void_p, c_void_p, c_void_p],
                          c_int32),
    "mmsp_gather_rows": ([c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int32, c_void_p], c_int32),
    "mmsp_ulysses_transpose": ([c_void_p, c_void_p, c_int64, c_int32, c_int32, c_int64, c_int32, c_void_p], c_int32),
    "mmsp_attn_bwd": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_int32,
                       c_int32, c_int32, c_float, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                       c_size_t, c_void_p, c_void_p], c_int32),
    "mmsp_attn_bwd_prepare": ([c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_int32, c_int32, c_int32, c_int32,
                               c_void_p, c_size_t, c_void_p], c_int32),
    "mmsp_attn_bwd_dkdv": ([c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_int32, c_int32, c_int32,
                            c_float, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p,
                            c_void_p], c_int32),
    "mmsp_attn_bwd_dq": ([c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_int32, c_int32, c_int32,
                          c_float, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p,
                          c_void_p], c_int32),
    "mmsp_bwd_workspace_bytes": ([c_int64, c_int32, c_int32, c_int32], c_size_t),
    "mmsp_attn_bwd_noalloc": ([c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int32,
                               c_int32, c_int32, c_int32, c_float, c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_void_p, c_void_p], c_int32),
    "mmsp_last_error": ([], ctypes.c_char_p),
    "mmsp_device_status": ([c_void_p], c_int32),
    "mmsp_selftest_bounded_wait": ([c_int64, c_void_p], c_int32),
    "mmsp_version": ([], ctypes.c_char_p),
}
for _name, (_args, _ret) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _ret


def exported_symbols():
    """Names of the C ABI this binding declares (all must resolve in the .so)."""
    return list(_SIGS)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        if not x.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return x.data_ptr()
    raise TypeError(f"expected a tensor, an int pointer or None, got {type(x)}")


def _stream(stream):
    if stream is None:
        import torch

        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(name, rc):
    if rc != 0:
        raise MmspError(name, rc, _lib.mmsp_last_error().decode())
    return rc


def mmsp_last_error() -> str:
    return _lib.mmsp_last_error().decode()


def mmsp_version() -> str:
    return _lib.mmsp_version().decode()


def mmsp_shard(seg_len, seg_kind, N, P, local2global=None, global2local=None, modality_local=None,
               segid_local=None, rank_counts=None, src=None, dst=None, row_bytes=0, inverse=False, stream=None):
    """Index maps and/or row permute of the zigzag shard step (see mmsp.h)."""
    n_seg = 0
    sl = sk = None
    if seg_len is not None:
        sl_arr = np.ascontiguousarray(np.asarray(seg_len, dtype=np.int32))
        sk_arr = np.ascontiguousarray(np.asarray(seg_kind, dtype=np.uint8))
        n_seg = int(sl_arr.size)
        sl = sl_arr.ctypes.data_as(c_void_p)
        sk = sk_arr.ctypes.data_as(c_void_p)
    rc = _lib.mmsp_shard(sl, sk, n_seg, int(N), int(P), _ptr(local2global), _ptr(global2local),
                         _ptr(modality_local), _ptr(segid_local), _ptr(rank_counts), _ptr(src), _ptr(dst),
                         int(row_bytes), int(bool(inverse)), _stream(stream))
    return _check("mmsp_shard", rc)


def _ranks(P, rank_begin, rank_end):
    return int(rank_begin), int(P if rank_end is None else rank_end)


def mmsp_attn_fwd(q, k, v, N, P, Hq, Hkv, d, scale, causal, step_begin, step_end, o_acc, lse, o_out,
                  flags, doc_start=None, stream=None, rank_begin=0, rank_end=None):
    """Ring attention forward of the virtual ranks [rank_begin, rank_end)
    (default: every rank) over ring steps [step_begin, step_end)."""
    rb, re = _ranks(P, rank_begin, rank_end)
    rc = _lib.mmsp_attn_fwd(_ptr(q), _ptr(k), _ptr(v), int(N), int(P), int(Hq), int(Hkv), int(d), float(scale),
                            int(causal), int(step_begin), int(step_end), rb, re, _ptr(o_acc), _ptr(lse),
                            _ptr(o_out), int(flags), _ptr(doc_start), _stream(stream))
    return _check("mmsp_attn_fwd", rc)


def mmsp_shard_rope(src, dst, N, P, H, d, theta=1e7, interleaved=False, doc_start=None, inverse=False, stream=None):
    """Shard gather with RoPE applied (or the transposed scatter; see mmsp.h)."""
    rc = _lib.mmsp_shard_rope(_ptr(src), _ptr(dst), int(N), int(P), int(H), int(d), float(theta),
                              int(bool(interleaved)), _ptr(doc_start), int(bool(inverse)), _stream(stream))
    return _check("mmsp_shard_rope", rc)


def mmsp_doc_starts(doc_len, N, doc_start, stream=None):
    """doc_start[g] (device int32 [N]) from host document lengths."""
    dl = np.ascontiguousarray(np.asarray(doc_len, dtype=np.int32))
    rc = _lib.mmsp_doc_starts(dl.ctypes.data_as(c_void_p), int(dl.size), int(N), _ptr(doc_start), _stream(stream))
    return _check("mmsp_doc_starts", rc)


def mmsp_lse_merge(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, H, d, stream=None):
    rc = _lib.mmsp_lse_merge(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(o_out), _ptr(lse_out),
                             int(rows), int(H), int(d), _stream(stream))
    return _check("mmsp_lse_merge", rc)


def mmsp_shard_frames(seg_len, seg_kind, N, P, global2enc=None, local2enc=None, enc_counts=None, stream=None):
    """Frame-aligned, modality-balanced encoder shard maps (see mmsp.h)."""
    sl_arr = np.ascontiguousarray(np.asarray(seg_len, dtype=np.int32))
    sk_arr = np.ascontiguousarray(np.asarray(seg_kind, dtype=np.uint8))
    rc = _lib.mmsp_shard_frames(sl_arr.ctypes.data_as(c_void_p), sk_arr.ctypes.data_as(c_void_p), int(sl_arr.size),
                                int(N), int(P), _ptr(global2enc), _ptr(local2enc), _ptr(enc_counts),
                                _stream(stream))
    return _check("mmsp_shard_frames", rc)


def mmsp_gather_rows(src, dst, index, n_rows, row_bytes, scatter=False, stream=None):
    """dst[i] = src[index[i]] (or the scatter dst[index[i]] = src[i])."""
    rc = _lib.mmsp_gather_rows(_ptr(src), _ptr(dst), _ptr(index), int(n_rows), int(row_bytes), int(bool(scatter)),
                               _stream(stream))
    return _check("mmsp_gather_rows", rc)


def mmsp_ulysses_transpose(src, dst, S, H, P_u, row_bytes, unpack=False, stream=None):
    """Sequence <-> head transpose around the Ulysses all-to-all (see mmsp.h):
    pack [S][H] -> [P_u][S][H/P_u], or unpack the inverse."""
    rc = _lib.mmsp_ulysses_transpose(_ptr(src), _ptr(dst), int(S), int(H), int(P_u), int(row_bytes),
                                     int(bool(unpack)), _stream(stream))
    return _check("mmsp_ulysses_transpose", rc)


def mmsp_attn_bwd(q, k, v, o, dout, lse, N, P, Hq, Hkv, d, scale, causal, dq, dk, dv, dq_acc_opt,
                  workspace, workspace_bytes, doc_start=None, stream=None):
    rc = _lib.mmsp_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), int(N), int(P), int(Hq),
                            int(Hkv), int(d), float(scale), int(causal), _ptr(dq), _ptr(dk), _ptr(dv),
                            _ptr(dq_acc_opt), _ptr(workspace), int(workspace_bytes), _ptr(doc_start),
                            _stream(stream))
    return _check("mmsp_attn_bwd", rc)


def mmsp_attn_bwd_prepare(o, dout, lse, N, P, Hq, d, workspace, workspace_bytes, stream=None, rank_begin=0,
                          rank_end=None):
    rb, re = _ranks(P, rank_begin, rank_end)
    rc = _lib.mmsp_attn_bwd_prepare(_ptr(o), _ptr(dout), _ptr(lse), int(N), int(P), int(Hq), int(d), rb, re,
                                    _ptr(workspace), int(workspace_bytes), _stream(stream))
    return _check("mmsp_attn_bwd_prepare", rc)


def mmsp_attn_bwd_dkdv(q, k, v, dout, N, P, Hq, Hkv, d, scale, causal, dk, dv, workspace, workspace_bytes,
                       doc_start=None, stream=None, rank_begin=0, rank_end=None):
    rb, re = _ranks(P, rank_begin, rank_end)
    rc = _lib.mmsp_attn_bwd_dkdv(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), int(N), int(P), int(Hq), int(Hkv), int(d),
                                 float(scale), int(causal), rb, re, _ptr(dk), _ptr(dv), _ptr(workspace),
                                 int(workspace_bytes), _ptr(doc_start), _stream(stream))
    return _check("mmsp_attn_bwd_dkdv", rc)


def mmsp_attn_bwd_dq(q, k, v, dout, N, P, Hq, Hkv, d, scale, causal, dq, dq_acc_opt, workspace, workspace_bytes,
                     doc_start=None, stream=None, rank_begin=0, rank_end=None):
    rb, re = _ranks(P, rank_begin, rank_end)
    rc = _lib.mmsp_attn_bwd_dq(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), int(N), int(P), int(Hq), int(Hkv), int(d),
                               float(scale), int(causal), rb, re, _ptr(dq), _ptr(dq_acc_opt), _ptr(workspace),
                               int(workspace_bytes), _ptr(doc_start), _stream(stream))
    return _check("mmsp_attn_bwd_dq", rc)


def mmsp_attn_bwd_noalloc(q, k, v, o, dout, lse, N, P, Hq, Hkv, d, scale, causal, dq, dk, dv, dq_acc_opt,
                          doc_start=None, stream=None):
    """Backward with the library's own fixed scratch (no allocation anywhere;
    see include/mmsp.h for the capacity and the sharing rules)."""
    rc = _lib.mmsp_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), int(N), int(P),
                                    int(Hq), int(Hkv), int(d), float(scale), int(causal), _ptr(dq), _ptr(dk),
                                    _ptr(dv), _ptr(dq_acc_opt), _ptr(doc_start), _stream(stream))
    return _check("mmsp_attn_bwd_noalloc", rc)


MMSP_NOALLOC_SCRATCH_BYTES = 64 << 20


def mmsp_bwd_workspace_bytes(N, P, Hq, d) -> int:
    return int(_lib.mmsp_bwd_workspace_bytes(int(N), int(P), int(Hq), int(d)))


def mmsp_device_status(stream=None) -> int:
    """Synchronise the stream; raises MmspError on a recorded timeout."""
    return _check("mmsp_device_status", _lib.mmsp_device_status(_stream(stream)))


def mmsp_selftest_bounded_wait(max_cycles, stream=None):
    return _check("mmsp_selftest_bounded_wait", _lib.mmsp_selftest_bounded_wait(int(max_cycles), _stream(stream)))
