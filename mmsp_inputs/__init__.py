"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and lays out the packed video+text sequence.
It holds none of the method's arithmetic: no sharding, no attention, no merge.
Both sides (the CUDA library and the fp64 oracle) receive exactly the arrays
built here.

Workload recipe (stand-in for the pages' hour-long 1 fps video with 576 visual
tokens per frame and interleaved text; "LongVILA Guide", section "Problem",
item 1, and "Example Execution Workflow"):

* a sequence of F frames of 576 visual tokens and S text segments whose
  lengths (total T tokens, every length >= 1) are cut at S-1 distinct seeded
  points of [1, T);
* text segment s is placed immediately before frame floor(s*F/S), so the
  sequence opens with text;
* Q [N,Hq,d], K [N,Hkv,d], V [N,Hkv,d] and dO [N,Hq,d] are iid N(0,1) drawn in
  that order in fp32 and rounded to bf16; K rows of visual tokens are then
  multiplied by 2 (exact in bf16) so that attention is peaked.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np

FRAME_TOKENS = 576
TEXT = 0
VISUAL = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    frames: int
    text_tokens: int
    text_segments: int
    hq: int
    hkv: int
    d: int
    P: int
    backward: bool
    index: int  # seeds: layout 1000+index, tensors 2000+index, rows 3000+index

    @property
    def N(self) -> int:
        return self.frames * FRAME_TOKENS + self.text_tokens

    @property
    def C(self) -> int:
        return self.N // (2 * self.P)

    def fwd_flops(self) -> float:
        """Algorithmic causal flops: 4*d*Hq*N(N+1)/2 (visible pairs only)."""
        N = self.N
        return 4.0 * self.d * self.hq * N * (N + 1) / 2.0

    def fwd_bwd_flops(self) -> float:
        return 3.5 * self.fwd_flops()


# The five named workloads (sizes: frames x 576 + text = N; GQA Hq/Hkv; P virtual ranks).
WORKLOADS = {
    "n4k": Workload("n4k", 4, 1792, 4, 4, 4, 64, 4, False, 0),
    "n32k": Workload("n32k", 56, 512, 8, 28, 4, 128, 8, False, 1),
    "n128k": Workload("n128k", 224, 2048, 32, 28, 4, 128, 32, True, 2),
    "n512k": Workload("n512k", 906, 2432, 64, 28, 4, 128, 64, True, 3),
    "n1m": Workload("n1m", 1816, 2560, 128, 28, 4, 128, 128, True, 4),
}


def make_layout(frames: int, text_tokens: int, text_segments: int,
                seed: int) -> Tuple[np.ndarray, np.ndarray]:
    """Segment table in sequence order: (lengths int32, kinds uint8).

    Frames are single segments of 576 tokens (kind VISUAL). Text segment
    lengths come from S-1 distinct cut points drawn from [1, T) without
    replacement, so every length is >= 1 and they sum to T.
    """
    F, T, S = frames, text_tokens, text_segments
    if S > T:
        raise ValueError("more text segments than text tokens")
    rng = np.random.default_rng(seed)
    if S > 0:
        cuts = np.sort(rng.choice(np.arange(1, T), S - 1, replace=False)) if S > 1 else np.zeros(0, np.int64)
        bounds = np.concatenate([[0], cuts, [T]])
        text_len = np.diff(bounds)
    else:
        text_len = np.zeros(0, np.int64)
    # text segment s goes right before frame floor(s*F/S)
    before = {}
    for s in range(S):
        f = (s * F) // S if F > 0 else 0
        before.setdefault(f, []).append(s)
    lens: List[int] = []
    kinds: List[int] = []
    for f in range(max(F, 1)):
        for s in before.get(f, []):
            lens.append(int(text_len[s]))
            kinds.append(TEXT)
        if f < F:
            lens.append(FRAME_TOKENS)
            kinds.append(VISUAL)
    return np.asarray(lens, np.int32), np.asarray(kinds, np.uint8)


def workload_layout(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    return make_layout(w.frames, w.text_tokens, w.text_segments, 1000 + w.index)


def token_kinds(seg_len: np.ndarray, seg_kind: np.ndarray) -> np.ndarray:
    """Per-token kind in global order (input construction only)."""
    return np.repeat(seg_kind.astype(np.uint8), seg_len.astype(np.int64))


def random_segments(N: int, seed: int, max_len: int = 700) -> Tuple[np.ndarray, np.ndarray]:
    """A seeded random segment table summing to N (for edge-case tests)."""
    rng = np.random.default_rng(seed)
    lens, kinds = [], []
    left = N
    while left > 0:
        L = int(min(left, rng.integers(1, max_len + 1)))
        lens.append(L)
        kinds.append(int(rng.integers(0, 2)))
        left -= L
    return np.asarray(lens, np.int32), np.asarray(kinds, np.uint8)


def packed_documents(N: int, seed: int, max_frames: int = 6, text_max: int = 300
                     ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """A seeded packed buffer of N tokens made of several short videos, each
    a document of (prompt text, f frames of FRAME_TOKENS visual tokens,
    answer text); the last document is cut at N. Returns (doc_len, seg_len,
    seg_kind): the document lengths and the matching segment table."""
    rng = np.random.default_rng(seed)
    docs, lens, kinds = [], [], []
    left = N
    while left > 0:
        parts = [(int(rng.integers(1, text_max + 1)), TEXT)]
        parts += [(FRAME_TOKENS, VISUAL)] * int(rng.integers(1, max_frames + 1))
        parts.append((int(rng.integers(1, 65)), TEXT))
        used = 0
        for L, kind in parts:
            L = min(L, left - used)
            if L <= 0:
                break
            lens.append(L)
            kinds.append(kind)
            used += L
        docs.append(used)
        left -= used
    return np.asarray(docs, np.int32), np.asarray(lens, np.int32), np.asarray(kinds, np.uint8)


def make_tensors(N: int, hq: int, hkv: int, d: int, seed: int, visual_mask,
                 device="cpu", with_dout: bool = False):
    """Q, K, V (and dO) as bf16 torch tensors [N, H, d], drawn in that order.

    `visual_mask` is a bool/uint8 array of length N in global token order; K
    rows of visual tokens are multiplied by 2 after rounding (exact in bf16).
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = torch.randn((N, hq, d), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((N, hkv, d), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((N, hkv, d), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    do = None
    if with_dout:
        do = torch.randn((N, hq, d), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    vm = torch.as_tensor(np.asarray(visual_mask, dtype=np.bool_)).to(device)
    k[vm] = k[vm] * 2
    return q, k, v, do


def workload_tensors(w: Workload, device="cpu", with_dout: Optional[bool] = None):
    seg_len, seg_kind = workload_layout(w)
    vis = token_kinds(seg_len, seg_kind) == VISUAL
    if with_dout is None:
        with_dout = w.backward
    return make_tensors(w.N, w.hq, w.hkv, w.d, 2000 + w.index, vis, device, with_dout)


def sample_rows(N: int, C: int, count: int, seed: int) -> np.ndarray:
    """Seeded global query positions: `count` distinct random positions
    other than the forced edges (0, N-1 and every chunk start), plus those
    edges; sorted."""
    import torch

    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    forced = np.unique(np.concatenate([[0, N - 1], np.arange(0, N, C, dtype=np.int64)]))
    free = np.setdiff1d(np.arange(N, dtype=np.int64), forced)
    count = min(count, len(free))
    r = free[torch.randperm(len(free), generator=g)[:count].numpy()]
    return np.sort(np.concatenate([r, forced]))


def sample_keys(N: int, window: int, count: int, seed: int) -> np.ndarray:
    """Seeded key positions: `count` distinct positions drawn from the last
    `window` of the sequence (always including N-1), sorted."""
    import torch

    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    window = min(window, N)
    r = N - window + torch.randperm(window - 1, generator=g)[:max(0, count - 1)].numpy().astype(np.int64)
    return np.sort(np.concatenate([r, [N - 1]]))
