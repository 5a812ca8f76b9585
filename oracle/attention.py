"""Causal softmax attention by its definition, in fp64 (oracle; test
infrastructure only).

Forward, for every global row i and query head h, kv head kh = floor(h*Hkv/Hq):
    s_ij   = (q_i . k_j) * scale          for j <= i   (scale = 1/sqrt(d))
    LSE_i  = ln sum_{j<=i} exp(s_ij)
    O_i    = sum_{j<=i} exp(s_ij - LSE_i) v_j
Scale and (B,S,H,D) layout: "LongVILA Guide" (aifetchly), section
"Implementation", ``LongVILAMultiModalAttention.forward`` (scores divided by
head_dim ** 0.5; q/k/v viewed as (b, s, n_heads, head_dim)). The ring method
reaches exactly this result (up to rounding order), so the oracle does not
simulate the ring for forward parity; ``merge.ring_attention`` does, to pin
the merge.

Backward (the pages give none; a reading: the gradient of the definition
above), with P_ij = exp(s_ij - LSE_i) and D_i = sum_d dO_i * O_i:
    dV_j = sum_i P_ij dO_i            (summed over the q heads of kv head kh)
    dP_ij = dO_i . v_j
    dS_ij = P_ij (dP_ij - D_i)
    dQ_i = scale sum_j dS_ij k_j
    dK_j = scale sum_i dS_ij q_i      (summed over the q heads of kv head kh)

Inputs are numpy arrays (any float dtype; converted to fp64) of shape
[N, H, d]. Rows are processed in blocks only to bound memory; every block is
the plain formula, evaluated with fp64 torch CPU ops (matmul, exp, log,
max, sum) so that large sampled checks use every host core.
"""
from __future__ import annotations

import math

import numpy as np
import torch

NEG_INF = -np.inf


def _t(x):
    """fp64 CPU torch view of a numpy array (no copy when already fp64)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))


def kv_head(h: int, hq: int, hkv: int) -> int:
    """GQA mapping (reading): contiguous groups of Hq/Hkv query heads."""
    return (h * hkv) // hq


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def document_starts(doc_len):
    """doc_start[g] for a packed sequence given as document lengths: the
    position where the document holding g begins ("LongVILA Guide",
    section "Critical Operational Best Practices", dynamic sequence packing:
    several videos share one buffer and the attention mask resets between
    them). Written as a plain loop over documents."""
    out = []
    pos = 0
    for L in np.asarray(doc_len, np.int64).tolist():
        if L < 1:
            raise ValueError("document lengths must be >= 1")
        out.extend([pos] * L)
        pos += L
    return np.asarray(out, np.int64)


def _visible(jmax, rows, lo):
    """[R, jmax] mask: key j visible to row i iff lo_i <= j <= i (lo_i = 0
    without documents)."""
    rows_t = torch.as_tensor(np.asarray(rows, np.int64))
    j = torch.arange(jmax)[None, :]
    vis = j <= rows_t[:, None]
    if lo is not None:
        vis &= j >= torch.as_tensor(np.asarray(lo, np.int64))[:, None]
    return vis


def _rows_forward(qr, rows, K, V, scale, lo=None):
    """O and LSE for query vectors qr [R,d] at global positions rows [R]
    against keys K[:i+1], V[:i+1] (one head); with `lo`, only keys
    j >= lo_i of the row's own document. Plain formula in fp64 torch CPU ops
    (multi-threaded; same arithmetic as numpy)."""
    R = len(rows)
    d = V.shape[1]
    if R == 0:
        return np.zeros((R, d)), np.full(R, NEG_INF)
    jmax = int(np.max(rows)) + 1
    qr, K, V = _t(qr), _t(K[:jmax]), _t(V[:jmax])
    s = (qr @ K.T) * scale                                       # [R, jmax]
    visible = _visible(jmax, rows, lo)
    s = s.masked_fill(~visible, NEG_INF)
    m = s.max(dim=1).values
    lse = m + torch.log(torch.exp(s - m[:, None]).sum(dim=1))
    p = torch.exp(s - lse[:, None])                              # 0 where masked
    O = p @ V
    return O.numpy(), lse.numpy()


def causal_attention(q, k, v, scale=None, block: int = 512, doc_start=None):
    """Whole-sequence forward. Returns (O [N,Hq,d], LSE [N,Hq]) in fp64.

    doc_start (optional, [N] ints, global order): first position of each
    token's document in a packed sequence; key j is then visible to query i
    iff doc_start[i] <= j <= i (attention reset at document boundaries)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, hq, d = q.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((N, hq, d))
    LSE = np.zeros((N, hq))
    for h in range(hq):
        kh = kv_head(h, hq, hkv)
        for i0 in range(0, N, block):
            rows = np.arange(i0, min(N, i0 + block))
            lo = None if doc_start is None else np.asarray(doc_start)[rows]
            o, l = _rows_forward(q[rows, h], rows, k[:, kh], v[:, kh], scale, lo)
            O[rows, h] = o
            LSE[rows, h] = l
    return O, LSE


def attention_rows(q_rows, k, v, rows, scale=None, block: int = 64, doc_start=None):
    """Forward for selected global rows only.

    q_rows [R,Hq,d] holds the query vectors of global positions `rows` (the
    caller gathers them, so the whole Q need not be held in fp64); k, v are
    the whole [N,Hkv,d] tensors, converted to fp64 one kv head at a time.
    Returns (O [R,Hq,d], LSE [R,Hq]).
    """
    q_rows = _f64(q_rows)
    rows = np.asarray(rows, np.int64)
    R, hq, d = q_rows.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    jmax = int(rows.max()) + 1 if R else 0
    O = np.zeros((R, hq, d))
    LSE = np.zeros((R, hq))
    for kh in range(hkv):
        K = _f64(k[:jmax, kh])
        V = _f64(v[:jmax, kh])
        for h in range(hq):
            if kv_head(h, hq, hkv) != kh:
                continue
            for b0 in range(0, R, block):
                sel = np.arange(b0, min(R, b0 + block))
                lo = None if doc_start is None else np.asarray(doc_start)[rows[sel]]
                o, l = _rows_forward(q_rows[sel, h], rows[sel], K, V, scale, lo)
                O[sel, h] = o
                LSE[sel, h] = l
    return O, LSE


def _rows_backward(qr, dor, rows, K, V, scale, lo=None):
    """For one head and query rows: (O, LSE, D, dQ rows, P, dS) restricted to
    keys [0, max(rows)]; P and dS are [R, jmax]. fp64 torch CPU ops."""
    jmax = int(np.max(rows)) + 1
    qr, dor, K, V = _t(qr), _t(dor), _t(K[:jmax]), _t(V[:jmax])
    s = (qr @ K.T) * scale
    visible = _visible(jmax, rows, lo)
    s = s.masked_fill(~visible, NEG_INF)
    m = s.max(dim=1).values
    lse = m + torch.log(torch.exp(s - m[:, None]).sum(dim=1))
    p = torch.exp(s - lse[:, None])
    o = p @ V
    D = (dor * o).sum(dim=1)
    dp = dor @ V.T
    ds = p * (dp - D[:, None])
    dq = scale * (ds @ K)
    return o.numpy(), lse.numpy(), D.numpy(), dq.numpy(), p.numpy(), ds.numpy()


def causal_attention_bwd(q, k, v, do, scale=None, block: int = 512, doc_start=None):
    """Whole-sequence backward of the definition (doc_start as in
    causal_attention).

    Returns dict with O, LSE, D [N,Hq], dQ [N,Hq,d], dK, dV [N,Hkv,d] (fp64).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    N, hq, d = q.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.zeros((N, hq, d))
    LSE = np.zeros((N, hq))
    Dm = np.zeros((N, hq))
    dQ = np.zeros((N, hq, d))
    dK = np.zeros((N, hkv, d))
    dV = np.zeros((N, hkv, d))
    for h in range(hq):
        kh = kv_head(h, hq, hkv)
        for i0 in range(0, N, block):
            rows = np.arange(i0, min(N, i0 + block))
            lo = None if doc_start is None else np.asarray(doc_start)[rows]
            o, lse, D, dq, p, ds = _rows_backward(q[rows, h], do[rows, h], rows,
                                                  k[:, kh], v[:, kh], scale, lo)
            jmax = p.shape[1]
            O[rows, h] = o
            LSE[rows, h] = lse
            Dm[rows, h] = D
            dQ[rows, h] = dq
            dV[:jmax, kh] += p.T @ do[rows, h]
            dK[:jmax, kh] += scale * (ds.T @ q[rows, h])
    return {"O": O, "LSE": LSE, "D": Dm, "dQ": dQ, "dK": dK, "dV": dV}


def attention_bwd_rows(q_rows, k, v, do_rows, rows, scale=None, block: int = 64, doc_start=None):
    """dQ (and O, LSE) for selected global rows: row i needs only keys <= i.
    q_rows and do_rows [R,Hq,d] are the caller-gathered rows at `rows`;
    doc_start as in causal_attention."""
    q_rows, do_rows = _f64(q_rows), _f64(do_rows)
    rows = np.asarray(rows, np.int64)
    R, hq, d = q_rows.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    jmax = int(rows.max()) + 1 if R else 0
    dQ = np.zeros((R, hq, d))
    O = np.zeros((R, hq, d))
    LSE = np.zeros((R, hq))
    for kh in range(hkv):
        K = _f64(k[:jmax, kh])
        V = _f64(v[:jmax, kh])
        for h in range(hq):
            if kv_head(h, hq, hkv) != kh:
                continue
            for b0 in range(0, R, block):
                sel = np.arange(b0, min(R, b0 + block))
                lo = None if doc_start is None else np.asarray(doc_start)[rows[sel]]
                o, lse, _, dq, _, _ = _rows_backward(q_rows[sel, h], do_rows[sel, h], rows[sel], K, V, scale, lo)
                dQ[sel, h] = dq
                O[sel, h] = o
                LSE[sel, h] = lse
    return {"O": O, "LSE": LSE, "dQ": dQ}


def attention_bwd_keys(q_tail, k, v, do_tail, keys, scale=None, block: int = 64, doc_start=None):
    """dK and dV for selected global key positions.

    Key j receives contributions from rows i >= j only. q_tail and do_tail
    hold the rows [j0, N) of Q and dO, where j0 = min(keys) and N = len(k);
    those rows are computed in full (their LSE and D over keys <= i) and
    their terms are summed into the requested keys. Cheap only when the keys
    lie near the end. doc_start as in causal_attention.
    """
    keys = np.asarray(keys, np.int64)
    N = k.shape[0]
    hkv = k.shape[1]
    hq, d = q_tail.shape[1], q_tail.shape[2]
    j0 = int(keys.min())
    if q_tail.shape[0] != N - j0 or do_tail.shape[0] != N - j0:
        raise ValueError("q_tail/do_tail must hold rows [min(keys), N)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    q_tail, do_tail = _f64(q_tail), _f64(do_tail)
    dK = np.zeros((len(keys), hkv, d))
    dV = np.zeros((len(keys), hkv, d))
    for kh in range(hkv):
        K = _f64(k[:, kh])
        V = _f64(v[:, kh])
        for h in range(hq):
            if kv_head(h, hq, hkv) != kh:
                continue
            for i0 in range(j0, N, block):
                rows = np.arange(i0, min(N, i0 + block))
                lo = None if doc_start is None else np.asarray(doc_start)[rows]
                _, _, _, _, p, ds = _rows_backward(q_tail[rows - j0, h], do_tail[rows - j0, h], rows, K, V, scale,
                                                   lo)
                sel = np.nonzero(keys <= rows.max())[0]
                dV[sel, kh] += p[:, keys[sel]].T @ do_tail[rows - j0, h]
                dK[sel, kh] += scale * (ds[:, keys[sel]].T @ q_tail[rows - j0, h])
    return {"dK": dK, "dV": dV}
