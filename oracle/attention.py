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


def _scores(qr, rows, K, scale, lo=None):
    """s_ij = (q_i . k_j) * scale for the keys K[:jmax] (fp64 torch), with
    -inf where key j is not visible to the row: j > i (causal), or j < lo_i
    (before the row's document start). qr is [R, d]; rows [R] holds each
    vector's global position (rows may repeat when several heads of one
    position are stacked). Columns before min(rows) + 1 are visible to every
    row and columns from max(lo) on pass the document test, so the mask is
    only applied where it can remove a key."""
    jmax = K.shape[0]
    s = qr @ K.T
    s.mul_(scale)
    rows = np.asarray(rows, np.int64)
    j_first = int(rows.min()) + 1
    if j_first < jmax:
        s[:, j_first:].masked_fill_(torch.arange(j_first, jmax)[None, :] > torch.as_tensor(rows)[:, None], NEG_INF)
    if lo is not None:
        lo = np.asarray(lo, np.int64)
        j_last = int(lo.max())
        if j_last > 0:
            s[:, :j_last].masked_fill_(torch.arange(j_last)[None, :] < torch.as_tensor(lo)[:, None], NEG_INF)
    return s


def _softmax_rows(qr, rows, K, V, scale, lo=None):
    """Row softmax of the visible scores and the output: returns (P, O, LSE)
    with P_ij = exp(s_ij - m_i) / l_i, l_i = sum_j exp(s_ij - m_i),
    m_i = max_j s_ij, O = P V and LSE_i = m_i + ln l_i. fp64 torch."""
    p = _scores(qr, rows, K, scale, lo)
    m = p.max(dim=1).values
    p.sub_(m[:, None]).exp_()                                    # 0 where masked
    l = p.sum(dim=1)
    p.div_(l[:, None])
    return p, p @ V, m + torch.log(l)


def _rows_forward(qr, rows, K, V, scale, lo=None):
    """O and LSE for query vectors qr [R,d] at global positions rows [R]
    against keys K[:i+1], V[:i+1] (one head); with `lo`, only keys
    j >= lo_i of the row's own document."""
    R = len(rows)
    d = V.shape[1]
    if R == 0:
        return np.zeros((R, d)), np.full(R, NEG_INF)
    jmax = int(np.max(rows)) + 1
    _, O, lse = _softmax_rows(_t(qr), rows, _t(K[:jmax]), _t(V[:jmax]), scale, lo)
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


def _head_groups(hq, hkv):
    """The query heads that read each kv head: kv head kh -> list of h."""
    return [[h for h in range(hq) if kv_head(h, hq, hkv) == kh] for kh in range(hkv)]


BLOCK_BUDGET = 1 << 25  # elements of one fp64 score matrix (memory bound only)


def _row_block(n_vec, jmax, budget=BLOCK_BUDGET):
    """Rows per block so that a [rows * n_vec, jmax] fp64 score matrix stays
    within `budget` elements."""
    return max(1, budget // max(1, n_vec * jmax))


def _sorted_block(sorted_rows, b0, n_vec, block=None):
    """Number of rows of the next block starting at index b0 of ascending
    `sorted_rows`: `block` if given, else as many as keep the block's score
    matrix in budget (its last, largest row sets the key count)."""
    if block:
        return block
    nb = min(_row_block(n_vec, int(sorted_rows[b0]) + 1), len(sorted_rows) - b0)
    while nb > 1 and nb * n_vec * (int(sorted_rows[b0 + nb - 1]) + 1) > BLOCK_BUDGET:
        nb = (nb + 1) // 2
    return nb


def attention_rows(q_rows, k, v, rows, scale=None, block=None, doc_start=None):
    """Forward for selected global rows only.

    q_rows [R,Hq,d] holds the query vectors of global positions `rows` (the
    caller gathers them, so the whole Q need not be held in fp64); k, v are
    the whole [N,Hkv,d] tensors, converted to fp64 one kv head at a time.
    Returns (O [R,Hq,d], LSE [R,Hq]). block: rows per block (default: a
    memory budget).
    """
    out = attention_bwd_rows(q_rows, k, v, None, rows, scale=scale, block=block, doc_start=doc_start)
    return out["O"], out["LSE"]


def _rows_backward(qr, dor, rows, K, V, scale, lo=None):
    """For one head and query rows: (O, LSE, D, dQ rows, P, dS) restricted to
    keys [0, max(rows)]; P and dS are [R, jmax]."""
    o, lse, D, dq, p, ds = _rows_backward_t(_t(qr), _t(dor), rows, _t(K), _t(V), scale, lo)
    return o.numpy(), lse.numpy(), D.numpy(), dq.numpy(), p.numpy(), ds.numpy()


def _rows_backward_t(qr, dor, rows, K, V, scale, lo=None):
    """_rows_backward on fp64 torch tensors (K, V may hold more keys than
    max(rows) + 1; only those are read). Returns torch tensors."""
    jmax = int(np.max(rows)) + 1
    K, V = K[:jmax], V[:jmax]
    p, o, lse = _softmax_rows(qr, rows, K, V, scale, lo)
    D = (dor * o).sum(dim=1)
    ds = dor @ V.T                                               # dP
    ds.sub_(D[:, None]).mul_(p)                                  # dS = P (dP - D)
    dq = (ds @ K).mul_(scale)
    return o, lse, D, dq, p, ds


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


def attention_bwd_rows(q_rows, k, v, do_rows, rows, scale=None, block=None, doc_start=None):
    """dQ (and O, LSE) for selected global rows: row i needs only keys <= i.
    q_rows and do_rows [R,Hq,d] are the caller-gathered rows at `rows`
    (do_rows None: forward only, no dQ); doc_start as in causal_attention.
    The query heads that read one kv head are evaluated together (their
    vectors stacked as rows of one matrix), in blocks of rows sorted by
    position (`block` rows per block; default: a memory budget)."""
    q_rows = _f64(q_rows)
    rows = np.asarray(rows, np.int64)
    R, hq, d = q_rows.shape
    hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    order = np.argsort(rows, kind="stable")
    dQ = np.zeros((R, hq, d))
    O = np.zeros((R, hq, d))
    LSE = np.zeros((R, hq))
    if R == 0:
        return {"O": O, "LSE": LSE, "dQ": dQ}
    jmax_all = int(rows.max()) + 1
    if do_rows is not None:
        do_rows = _f64(do_rows)
    ds_all = None if doc_start is None else np.asarray(doc_start, np.int64)
    for kh, heads in enumerate(_head_groups(hq, hkv)):
        G = len(heads)
        K = _t(k[:jmax_all, kh])
        V = _t(v[:jmax_all, kh])
        srows = rows[order]
        b0 = 0
        while b0 < R:
            nb = _sorted_block(srows, b0, G, block)
            sel = order[b0:b0 + nb]
            b0 += nb
            rr = rows[sel]
            rep = np.repeat(rr, G)                      # position of each stacked vector
            lo = None if ds_all is None else ds_all[rep]
            qb = _t(q_rows[np.ix_(sel, heads)].reshape(-1, d))
            if do_rows is None:
                jmax = int(rr.max()) + 1
                _, o, lse = _softmax_rows(qb, rep, K[:jmax], V[:jmax], scale, lo)
            else:
                dob = _t(do_rows[np.ix_(sel, heads)].reshape(-1, d))
                o, lse, _, dq, _, _ = _rows_backward_t(qb, dob, rep, K, V, scale, lo)
                dQ[np.ix_(sel, heads)] = dq.reshape(len(sel), G, d).numpy()
            O[np.ix_(sel, heads)] = o.reshape(len(sel), G, d).numpy()
            LSE[np.ix_(sel, heads)] = lse.reshape(len(sel), G).numpy()
    return {"O": O, "LSE": LSE, "dQ": dQ}


def attention_bwd_keys(q_tail, k, v, do_tail, keys, scale=None, block=None, doc_start=None, kv_heads=None):
    """dK and dV for selected global key positions.

    Key j receives contributions from rows i >= j only. q_tail and do_tail
    hold the rows [j0, N) of Q and dO, where j0 = min(keys) and N = len(k);
    those rows are computed in full (their LSE and D over keys <= i) and
    their terms are summed into the requested keys. Cheap only when the keys
    lie near the end. doc_start as in causal_attention. kv_heads: the kv
    heads to compute (default all; the others stay 0). block: rows per
    block (default: a memory budget).
    Also returns the tail rows' O, LSE and dQ ("O_tail", ...).
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
    T = N - j0
    O = np.zeros((T, hq, d))
    LSE = np.zeros((T, hq))
    dQ = np.zeros((T, hq, d))
    ds_all = None if doc_start is None else np.asarray(doc_start, np.int64)
    keys_t = torch.as_tensor(keys)
    for kh, heads in enumerate(_head_groups(hq, hkv)):
        if kv_heads is not None and kh not in kv_heads:
            continue
        G = len(heads)
        K = _t(k[:, kh])
        V = _t(v[:, kh])
        dKk = torch.zeros((len(keys), d), dtype=torch.float64)
        dVk = torch.zeros((len(keys), d), dtype=torch.float64)
        i0 = j0
        while i0 < N:
            nb = block or _row_block(G, N)
            rows = np.arange(i0, min(N, i0 + nb))
            i0 += nb
            rep = np.repeat(rows, G)
            lo = None if ds_all is None else ds_all[rep]
            qb = _t(q_tail[np.ix_(rows - j0, heads)].reshape(-1, d))
            dob = _t(do_tail[np.ix_(rows - j0, heads)].reshape(-1, d))
            o, lse, _, dq, p, ds = _rows_backward_t(qb, dob, rep, K, V, scale, lo)
            O[np.ix_(rows - j0, heads)] = o.reshape(len(rows), G, d).numpy()
            LSE[np.ix_(rows - j0, heads)] = lse.reshape(len(rows), G).numpy()
            dQ[np.ix_(rows - j0, heads)] = dq.reshape(len(rows), G, d).numpy()
            sel = np.nonzero(keys <= rows.max())[0]
            if len(sel) == 0:
                continue
            ks = keys_t[torch.as_tensor(sel)]
            dVk[sel] += p[:, ks].T @ dob
            dKk[sel] += scale * (ds[:, ks].T @ qb)
        dK[:, kh] = dKk.numpy()
        dV[:, kh] = dVk.numpy()
    return {"dK": dK, "dV": dV, "O_tail": O, "LSE_tail": LSE, "dQ_tail": dQ}
