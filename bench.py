"""Benchmark: ring-blockwise causal attention (MM-SP hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload n512k] [--impl reference]

One step is one pass of the whole hot path over one synthetic sequence:
zigzag shard maps, gather of Q/K/V/dO into rank-local order, attention
forward over every virtual rank and ring step (merge fused), backward, and
the inverse scatter of O/dQ/dK/dV -- all through the C ABI of libmmsp.so.
Throughput is algorithmic causal flops (forward 4*d*Hq*N(N+1)/2, forward +
backward 3.5x that) per second.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
sequence (weak scaling, no collective on the data path); time is the max
over ranks. `--impl reference` times the fp64 CPU oracle on a bounded row
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import signal
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import mmsp_inputs as mi  # noqa: E402

METRIC = "causal ring-attention TFLOP/s fwd & fwd+bwd at N=32K–1M; % of B200 BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "long_context_multimodal_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(profile_md, source_files):
    """Per-launch DRAM bytes recorded from an ncu capture, or None when the
    summary is missing or the kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", profile_md)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"source_sha:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != kernel_source_hash(source_files):
        return None
    return float(m.group(1))


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 8:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        mx = [num(r[1]) for r in rows if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower().startswith("active")})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


_KV_CACHE = {}
PARITY_ROWS = 4096  # the seeded query rows the full-size parity tests check


def parity_rows(w, count, part=0):
    """`count` query positions spread evenly over the seeded 4,096-row sample
    the full-size parity tests use (mmsp_inputs.sample_rows with seed
    3000 + index, forced chunk starts included); `part` picks a different
    interleaved subset."""
    sample = mi.sample_rows(w.N, w.C, PARITY_ROWS, 3000 + w.index)
    stride = max(1, len(sample) // max(1, count))
    return np.sort(sample[(part % stride)::stride][:count])


def cpu_sample_inputs(w, rows_count, seed):
    """Rows of the workload for the CPU oracle without building all of Q:
    K, V whole and Q, dO at rows of the parity sample (same recipe and
    distribution, CPU generator)."""
    import torch

    rows = parity_rows(w, rows_count, seed)
    g = torch.Generator().manual_seed(2000 + w.index + seed)
    bf = lambda *s: torch.randn(s, generator=g).to(torch.bfloat16)
    if w.name not in _KV_CACHE:
        gk = torch.Generator().manual_seed(2000 + w.index)
        vis = torch.as_tensor(mi.token_kinds(*mi.workload_layout(w)) == mi.VISUAL)
        k = torch.randn((w.N, w.hkv, w.d), generator=gk).to(torch.bfloat16)
        v = torch.randn((w.N, w.hkv, w.d), generator=gk).to(torch.bfloat16)
        k[vis] = k[vis] * 2
        _KV_CACHE[w.name] = (k.float().numpy(), v.float().numpy())
    kc, vc = _KV_CACHE[w.name]
    qr, dor = bf(len(rows), w.hq, w.d), bf(len(rows), w.hq, w.d)
    return rows, qr.float().numpy(), kc, vc, dor.float().numpy()


def oracle_sample(w, rows_count, seed, inputs=None):
    """fp64 oracle (forward + dQ backward) on a bounded sample of query rows
    of workload w; returns (algorithmic flops of the sample, seconds, threads)."""
    import torch

    from oracle import attention as A

    rows, qr, kc, vc, dor = inputs if inputs is not None else cpu_sample_inputs(w, rows_count, seed)
    torch.set_num_threads(host_cores())
    t0 = time.perf_counter()
    A.attention_bwd_rows(qr, kc, vc, dor, rows)
    dt = time.perf_counter() - t0
    # each sampled row i: forward 4*d*(i+1) flops per head, forward+backward 3.5x
    flops = 3.5 * 4.0 * w.d * w.hq * float(np.sum(rows + 1))
    return flops, dt, torch.get_num_threads()


def host_cores():
    """Cores this process may run on (its CPU affinity set)."""
    return len(os.sched_getaffinity(0))


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = mi.WORKLOADS[args.workload]
    rows = args.ref_rows
    sample = (f"{rows} query rows x all {w.hq} heads of {w.name} (N={w.N}), an interleaved subset of the "
              f"{PARITY_ROWS} seeded rows the parity tests check (a different subset each step): forward + dQ "
              f"backward in fp64")
    for i in range(args.warmup):
        oracle_sample(w, max(4, rows // 8), 100 + i)
    vals, secs = [], 0.0
    threads = 1
    for i in range(args.steps):
        fl, dt, threads = oracle_sample(w, rows, 1000 + i)
        vals.append(fl / dt / 1e12)
        secs += dt
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus, args.mode),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, gpus, mode="split"):
    if gpus == 1:
        par = f"one GPU holds all {w.P} virtual ranks of the ring"
        batch = 1
    elif mode == "split":
        par = (f"one sequence; its {w.P} virtual ranks split over {gpus} GPUs ({w.P // gpus} each), K/V, Q, dO and "
               f"the prepared (LSE, D) rows all-gathered with NCCL")
        batch = 1
    else:
        par = f"{gpus} independent sequences, one per GPU; all {w.P} virtual ranks on each GPU"
        batch = gpus
    return {"workload": w.name, "N": w.N, "frames": w.frames, "frame_tokens": mi.FRAME_TOKENS,
            "text_tokens": w.text_tokens, "text_segments": w.text_segments, "Hq": w.hq, "Hkv": w.hkv, "d": w.d,
            "P_virtual_ranks": w.P, "causal": True, "global_batch": batch, "seq_len": w.N,
            "parallelism": par, "l2": "inputs larger than L2 (Q alone is N*Hq*d*2 bytes)"}


def max_over_ranks(values, ws, device=None):
    """Element-wise max of per-rank timings (the job takes as long as its
    slowest rank)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if ws > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(flops_per_step, sequences, ms_per_step):
    """Whole-job TFLOP/s: `sequences` sequences of `flops_per_step` each per
    step (one per GPU for replicas, one in all for a split ring)."""
    return flops_per_step * sequences / (ms_per_step * 1e-3) / 1e12


class Path:
    """Device buffers and the C-ABI calls of one hot-path step."""

    def __init__(self, w, device, seed_offset=0, owned=None, group=None):
        import torch

        import long_context_multimodal_b200 as m

        self.m = m
        self.w = w
        self.dev = device
        # owned: the virtual ranks this GPU computes when the ring is split
        # across GPUs (split.RankRange), or None for the whole ring
        self.owned = owned
        self.group = group
        N, P, hq, hkv, d = w.N, w.P, w.hq, w.hkv, w.d
        self.seg_len, self.seg_kind = mi.workload_layout(w)
        vis = mi.token_kinds(self.seg_len, self.seg_kind) == mi.VISUAL
        self.q, self.k, self.v, self.do = mi.make_tensors(N, hq, hkv, d, 2000 + w.index + 100 * seed_offset, vis,
                                                          device=device, with_dout=True)
        e = lambda *s, dt=torch.bfloat16: torch.empty(s, dtype=dt, device=device)
        self.ql, self.kl, self.vl, self.dol = e(N, hq, d), e(N, hkv, d), e(N, hkv, d), e(N, hq, d)
        self.ol, self.dql, self.dkl, self.dvl = e(N, hq, d), e(N, hq, d), e(N, hkv, d), e(N, hkv, d)
        self.o, self.dq, self.dk, self.dv = e(N, hq, d), e(N, hq, d), e(N, hkv, d), e(N, hkv, d)
        self.lse = e(N, hq, dt=torch.float32)
        self.l2g = e(N, dt=torch.int32)
        self.g2l = e(N, dt=torch.int32)
        self.mod = e(N, dt=torch.uint8)
        self.segid = e(N, dt=torch.int32)
        self.counts = e(P, 2, dt=torch.int32)
        self.ws_bytes = m.mmsp_bwd_workspace_bytes(N, P, hq, d)
        self.ws = e(self.ws_bytes, dt=torch.uint8)
        self.scale = 1.0 / math.sqrt(d)
        self.launches_per_step = 2 + 4 + 1 + 3 + 4  # maps+counts, 4 gathers, fwd, bwd x3, 4 scatters

    def _exchange(self, *tensors):
        """Split ring: every GPU's owned rows of these rank-local tensors to
        every GPU (NCCL all-gather); nothing for the whole ring on one GPU."""
        if self.owned is None:
            return
        from long_context_multimodal_b200 import split

        for t in tensors:
            split.all_gather_rows(t, self.owned, self.group)

    def _exchange_workspace(self):
        if self.owned is None:
            return
        import torch.distributed as dist

        from long_context_multimodal_b200 import split

        w = self.w
        C = w.N // (2 * w.P)
        slab = w.hq * 2 * ((C + 127) // 128 * 128)
        for arr in split.workspace_slabs(self.ws, w.P, w.hq, C):
            own = arr[self.owned.begin * slab:self.owned.end * slab].contiguous()
            dist.all_gather_into_tensor(arr, own, group=self.group)

    def step(self, stream, ev=None, io=None):
        """One hot-path step. io: (inputs q, k, v, dO; outputs O, dQ, dK,
        dV) in global order, default this path's own buffers."""
        m, w = self.m, self.w
        N, P = w.N, w.P
        q, k, v, do, o, dq, dk, dv = io if io is not None else (self.q, self.k, self.v, self.do, self.o, self.dq,
                                                                  self.dk, self.dv)
        rk = {} if self.owned is None else {"rank_begin": self.owned.begin, "rank_end": self.owned.end}
        m.mmsp_shard(self.seg_len, self.seg_kind, N, P, self.l2g, self.g2l, self.mod, self.segid, self.counts,
                     stream=stream)
        for src, dst in ((q, self.ql), (k, self.kl), (v, self.vl), (do, self.dol)):
            m.mmsp_shard(None, None, N, P, src=src, dst=dst, row_bytes=src[0].numel() * 2, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        self._exchange(self.kl, self.vl)
        m.mmsp_attn_fwd(self.ql, self.kl, self.vl, N, P, w.hq, w.hkv, w.d, self.scale, 1, 0, P, None, self.lse,
                        self.ol, m.MMSP_FINALIZE, stream=stream, **rk)
        if ev is not None:
            ev[1].record(stream)
        # the backward's three stages (what mmsp_attn_bwd runs), so that the
        # dominant dK/dV kernel can be timed on its own
        m.mmsp_attn_bwd_prepare(self.ol, self.dol, self.lse, N, P, w.hq, w.d, self.ws, self.ws_bytes, stream=stream,
                                **rk)
        self._exchange_workspace()
        self._exchange(self.ql, self.dol)
        if ev is not None:
            ev[2].record(stream)
        m.mmsp_attn_bwd_dkdv(self.ql, self.kl, self.vl, self.dol, N, P, w.hq, w.hkv, w.d, self.scale, 1, self.dkl,
                             self.dvl, self.ws, self.ws_bytes, stream=stream, **rk)
        if ev is not None:
            ev[3].record(stream)
        m.mmsp_attn_bwd_dq(self.ql, self.kl, self.vl, self.dol, N, P, w.hq, w.hkv, w.d, self.scale, 1, self.dql, None,
                           self.ws, self.ws_bytes, stream=stream, **rk)
        if ev is not None:
            ev[4].record(stream)
        for src, dst in ((self.ol, o), (self.dql, dq), (self.dkl, dk), (self.dvl, dv)):
            m.mmsp_shard(None, None, N, P, src=src, dst=dst, row_bytes=src[0].numel() * 2, inverse=True,
                         stream=stream)


def document_masked(m, path, w, dev, stream, time_calls, peak):
    """Forward and backward of the packed-document variant: the workload's
    N tokens as a buffer of short videos (mmsp_inputs.packed_documents),
    every document's attention causal and isolated. Algorithmic flops count
    the visible pairs, 4 d Hq sum_docs L (L + 1) / 2 for the forward and
    2.5x that for the backward (prepare + dK/dV + dQ)."""
    import torch

    doc_len, _, _ = mi.packed_documents(w.N, 3000 + w.index)
    ds = torch.empty(w.N, dtype=torch.int32, device=dev)
    m.mmsp_doc_starts(doc_len, w.N, ds, stream=stream)
    L = doc_len.astype(np.float64)
    flops = 4.0 * w.d * w.hq * float((L * (L + 1) / 2).sum())
    N, P = w.N, w.P

    def fwd():
        m.mmsp_attn_fwd(path.ql, path.kl, path.vl, N, P, w.hq, w.hkv, w.d, path.scale, 1, 0, P, None, path.lse,
                        path.ol, m.MMSP_FINALIZE, doc_start=ds, stream=stream)

    def bwd():
        m.mmsp_attn_bwd_prepare(path.ol, path.dol, path.lse, N, P, w.hq, w.d, path.ws, path.ws_bytes, stream=stream)
        m.mmsp_attn_bwd_dkdv(path.ql, path.kl, path.vl, path.dol, N, P, w.hq, w.hkv, w.d, path.scale, 1, path.dkl,
                             path.dvl, path.ws, path.ws_bytes, doc_start=ds, stream=stream)
        m.mmsp_attn_bwd_dq(path.ql, path.kl, path.vl, path.dol, N, P, w.hq, w.hkv, w.d, path.scale, 1, path.dql,
                           None, path.ws, path.ws_bytes, doc_start=ds, stream=stream)

    ms = time_calls(fwd)
    bms = time_calls(bwd, reps=3)
    m.mmsp_device_status(stream)
    fwd_line = {"documents": int(doc_len.size), "mean_tokens": float(L.mean()), "ms": ms,
                "algorithmic_flops": flops, "tflops": flops / (ms * 1e-3) / 1e12,
                "frac_of_peak": flops / (ms * 1e-3) / 1e12 / peak}
    bwd_line = {"documents": int(doc_len.size), "ms": bms, "algorithmic_flops": 2.5 * flops,
                "tflops": 2.5 * flops / (bms * 1e-3) / 1e12, "frac_of_peak": 2.5 * flops / (bms * 1e-3) / 1e12 / peak}
    return fwd_line, bwd_line


def hbm_kernels(m, path, w, dev, stream, time_calls, hbm_peak):
    """The bandwidth-bound kernels timed alone at the workload's size, as
    achieved GB/s of their algorithmic bytes: the zigzag maps (two int32
    maps, uint8 modality, int32 segment id: 13 B per token), the plain row
    gather of Q (read + write, 2 * Hq * d * 2 B per token), and the
    standalone LSE merge of two fp32 partials over every (row, head) of the
    sequence (read 2 d + 2, write d + 1 fp32: 1,548 B per row-head at
    d = 128)."""
    import torch

    N, P, hq, d = w.N, w.P, w.hq, w.d

    def line(name, nbytes, ms):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"kernel": name, "bound": "hbm", "bytes_per_launch": nbytes, "ms": ms, "achieved": gbs,
                "unit": "GB/s", "peak": hbm_peak, "frac": gbs / hbm_peak}

    def graph_ms(call, reps=20):
        """Device time per launch of `call`, captured `reps` times in a CUDA
        graph and replayed back to back (for launches shorter than the host
        work of one call: there, back-to-back calls leave the GPU idle)."""
        cs = torch.cuda.Stream(device=dev)
        cs.wait_stream(torch.cuda.current_stream(dev))
        call(cs)
        torch.cuda.synchronize(dev)
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph, stream=cs):
            for _ in range(reps):
                call(cs)
        with torch.cuda.stream(cs):
            gph.replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(cs)
            gph.replay()
            b.record(cs)
        b.synchronize()
        del gph
        return a.elapsed_time(b) / reps

    out = {}
    maps_call = lambda st: m.mmsp_shard(path.seg_len, path.seg_kind, N, P, path.l2g, path.g2l, path.mod, path.segid,
                                        None, stream=st)
    host_ms = time_calls(lambda: maps_call(stream), reps=20)
    try:
        ms, how = graph_ms(maps_call), "CUDA graph of 20 launches replayed back to back (device time)"
    except Exception as exc:  # noqa: BLE001
        ms, how = host_ms, f"events around 20 calls, host work included (graph capture failed: {type(exc).__name__})"
    out["shard_maps"] = line("shard_maps_kernel", 13.0 * N, ms)
    out["shard_maps"].update(timing=how, ms_per_call_with_host=host_ms)
    ms = time_calls(lambda: m.mmsp_shard(None, None, N, P, src=path.q, dst=path.ql, row_bytes=hq * d * 2,
                                         stream=stream), reps=10)
    out["shard_gather_q"] = line("shard_rows_kernel (Q)", 2.0 * N * hq * d * 2, ms)
    g = torch.Generator(device=dev).manual_seed(11)
    oa = torch.randn((N, hq, d), device=dev, generator=g)
    ob = torch.randn((N, hq, d), device=dev, generator=g)
    la = torch.randn((N, hq), device=dev, generator=g)
    lb = torch.randn((N, hq), device=dev, generator=g)
    ms = time_calls(lambda: m.mmsp_lse_merge(oa, la, ob, lb, oa, la, N, hq, d, stream=stream), reps=10)
    out["lse_merge"] = line("lse_merge_kernel<128> (in place)", float(N * hq * (3 * d * 4 + 3 * 4)), ms)
    m.mmsp_device_status(stream)
    del oa, ob, la, lb
    torch.cuda.empty_cache()
    return out


def run_gpu(args):
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
    w = mi.WORKLOADS[args.workload]
    split_ring = ws > 1 and args.mode == "split"
    owned = None
    if split_ring:
        from long_context_multimodal_b200 import split

        owned = split.owned_ranks(w.P, ws, rank, w.N // (2 * w.P))
    # a split ring computes one sequence (the same seed on every GPU); the
    # replicas compute one independent sequence per GPU
    path = Path(w, dev, seed_offset=0 if split_ring else rank, owned=owned)
    m = path.m
    sequences = 1 if split_ring else ws
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        path.step(stream)
    m.mmsp_device_status(stream)

    # ---------------- device-resident timing
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(cvd.split(",")[local] if cvd else local)
    if rank == 0:
        sampler.start()
    barrier()
    t_start.record(stream)
    for i in range(args.steps):
        path.step(stream, evs[i])
    t_end.record(stream)
    barrier()
    clocks = sampler.stop() if rank == 0 else None
    m.mmsp_device_status(stream)
    ms_total = t_start.elapsed_time(t_end)
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd_ms = float(np.mean([e[1].elapsed_time(e[4]) for e in evs]))
    dkdv_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))
    dq_ms = float(np.mean([e[3].elapsed_time(e[4]) for e in evs]))
    rows = slice(None) if owned is None else owned.rows  # the rank-local rows this GPU computed
    ok = all(bool(torch.isfinite(t[rows].float()).all()) for t in (path.ol, path.dql, path.dkl, path.dvl))

    # ---------------- end to end through the C ABI with host buffers: every
    # step copies its inputs from pinned host memory and its outputs back,
    # on a copy stream, double-buffered so that step i+1's inputs arrive
    # and step i's outputs leave while step i+1 computes
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    dev_in = [(path.q, path.k, path.v, path.do), tuple(torch.empty_like(t) for t in (path.q, path.k, path.v, path.do))]
    dev_out = [(path.o, path.dq, path.dk, path.dv), tuple(torch.empty_like(t) for t in (path.o, path.dq, path.dk,
                                                                                         path.dv))]
    h_in = [pin(t) for t in dev_in[0]]
    for h, t in zip(h_in, dev_in[0]):
        h.copy_(t)
    h_out = [pin(t) for t in dev_out[0]]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    e_steps = max(1, args.e2e_steps if args.e2e_steps is not None else args.steps)
    copy_stream = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)

    def h2d_copy(b):
        with torch.cuda.stream(copy_stream):
            for h, t in zip(h_in, dev_in[b]):
                t.copy_(h, non_blocking=True)
        done = ev()
        done.record(copy_stream)
        return done

    inputs_ready = [h2d_copy(0), None]
    step_done = [None, None]   # step that last read/wrote buffer set b
    outputs_read = [None, None]
    for i in range(e_steps):
        b = i % 2
        stream.wait_event(inputs_ready[b])
        if outputs_read[b] is not None:
            stream.wait_event(outputs_read[b])  # step i-2's outputs have left
        path.step(stream, io=dev_in[b] + dev_out[b])
        step_done[b] = ev()
        step_done[b].record(stream)
        if i + 1 < e_steps:
            nb = 1 - b
            if step_done[nb] is not None:
                copy_stream.wait_event(step_done[nb])  # step i-1 has read its inputs
            inputs_ready[nb] = h2d_copy(nb)
        copy_stream.wait_event(step_done[b])
        with torch.cuda.stream(copy_stream):
            for h, t in zip(h_out, dev_out[b]):
                h.copy_(t, non_blocking=True)
        outputs_read[b] = ev()
        outputs_read[b].record(copy_stream)
    stream.wait_event(outputs_read[(e_steps - 1) % 2])
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    m.mmsp_device_status(stream)
    del dev_in, dev_out

    # ---------------- the RoPE-fused shard gather of Q (theta = 1e7), timed
    # on its own next to the plain gather it replaces (not part of the step:
    # the configured workload gives Q and K directly)
    def time_calls(fn, reps=5):
        fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / reps

    rope_ms = time_calls(lambda: m.mmsp_shard_rope(path.q, path.ql, w.N, w.P, w.hq, w.d, 1e7, False, stream=stream))
    plain_ms = time_calls(lambda: m.mmsp_shard(None, None, w.N, w.P, src=path.q, dst=path.ql,
                                               row_bytes=w.hq * w.d * 2, stream=stream))
    m.mmsp_device_status(stream)

    # ---------------- max over ranks
    ms_total, e2e_ms, fwd_ms, bwd_ms, dkdv_ms, dq_ms = max_over_ranks(
        [ms_total, e2e_ms, fwd_ms, bwd_ms, dkdv_ms, dq_ms], ws, dev)
    ms_step = ms_total / args.steps
    flops = w.fwd_bwd_flops()
    value = job_throughput(flops, sequences, ms_step)
    per_gpu = sequences / ws  # share of one sequence's work each GPU does
    if rank == 0:
        peaks, src = load_peaks()
        peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        # dominant kernel (ncu launch list): the dK/dV kernel; its algorithmic
        # work is the four GEMM-equivalents S^T, dP^T, dV, dK = 2x forward
        dkdv_flops = 2.0 * w.fwd_flops() * per_gpu
        achieved = dkdv_flops / (dkdv_ms * 1e-3) / 1e12
        traffic = profiled_traffic(f"attn_bwd_dkdv_{w.name}.md", ["attn_bwd.cuh", "ptx.cuh", "ring.cuh"])
        hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        rope_bytes = 2.0 * w.N * w.hq * w.d * 2  # read + write of Q, bf16
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if split_ring else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w, ws, args.mode),
            "fwd_tflops": w.fwd_flops() * per_gpu / (fwd_ms * 1e-3) / 1e12,
            "fwd_bwd_tflops": value / ws,
            "frac_of_bf16_peak": {"fwd": w.fwd_flops() * per_gpu / (fwd_ms * 1e-3) / 1e12 / peak,
                                  "fwd_bwd": value / ws / peak, "peak_tflops": peak,
                                  "peak_kind": f"bf16_tflops_sustained ({src})"},
            "roofline": {"kernel": "attn_bwd_dkdv_kernel (mmsp_attn_bwd_dkdv)",
                         "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_flops_per_launch": dkdv_flops, "launch_ms": dkdv_ms,
                         "peak_source": ("MEASURED_PEAKS.json bf16_tflops_sustained (measured)" if src == "measured"
                                         else "profiling recipe fallback, bf16 sustained (no MEASURED_PEAKS.json)")},
            "bwd_tflops": 2.5 * w.fwd_flops() * per_gpu / (bwd_ms * 1e-3) / 1e12,
            "kernel_ms": {"attn_fwd": fwd_ms, "attn_bwd_dkdv": dkdv_ms, "attn_bwd_dq": dq_ms,
                          "bwd_total": bwd_ms},
            "e2e": {"value": flops * sequences / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "rope_gather": {"kernel": "shard_rope_kernel<128, half pairs> on Q, theta = 1e7", "bound": "hbm",
                            "achieved": rope_bytes / (rope_ms * 1e-3) / 1e9, "unit": "GB/s",
                            "peak": hbm_peak, "frac": rope_bytes / (rope_ms * 1e-3) / 1e9 / hbm_peak,
                            "bytes_per_launch": rope_bytes, "ms": rope_ms, "plain_gather_ms": plain_ms},
            "gpu_launches": path.launches_per_step * args.steps,
            "clocks": clocks,
            "outputs_finite": ok,
        }
        if ws == 1 and not args.no_cpu_baseline:
            rows = parity_rows(w, args.ref_rows)
            ridx = torch.as_tensor(rows, device=dev)
            inp = (rows, path.q[ridx].float().cpu().numpy(), path.k.float().cpu().numpy(),
                   path.v.float().cpu().numpy(), path.do[ridx].float().cpu().numpy())
            fl, dt, threads = oracle_sample(w, len(rows), 7, inputs=inp)
            line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                    "sample": f"{len(rows)} of the {PARITY_ROWS} seeded parity rows (evenly "
                                              f"spread) x {w.hq} heads of {w.name}: fp64 forward + dQ "
                                              f"backward ({dt:.1f} s)"}
        # rank 0 alone, after the timed steps (the other ranks wait at the
        # final barrier): the bandwidth-bound kernels and the packed-document
        # variant on rank 0's buffers, each guarded so that a problem here is
        # reported in the line instead of losing it
        try:
            line.update(hbm_kernels(m, path, w, dev, stream, time_calls, hbm_peak))
        except Exception as exc:  # noqa: BLE001
            line["hbm_kernels_error"] = f"{type(exc).__name__}: {exc}"
        try:
            line["document_masked_fwd"], line["document_masked_bwd"] = document_masked(m, path, w, dev, stream,
                                                                                       time_calls, peak)
        except Exception as exc:  # noqa: BLE001
            line["document_masked_fwd"] = {"error": f"{type(exc).__name__}: {exc}"}
        mhz = (clocks or {}).get("sm_mhz")
        if mhz:
            # the sustained peak was measured at a different SM clock than
            # the one under this run's power cap: per-clock fractions
            # against the nominal dense bf16 peak (2,250 TFLOP/s at the
            # 1,965 MHz maximum clock) take the clock out of the comparison
            nominal_per_ghz = 2250.0 / 1.965
            line["per_clock"] = {"sm_mhz": mhz, "nominal_bf16_tflops_per_ghz": nominal_per_ghz,
                                 "fwd_tflops_per_ghz": line["fwd_tflops"] / (mhz / 1e3),
                                 "fwd_bwd_tflops_per_ghz": line["fwd_bwd_tflops"] / (mhz / 1e3),
                                 "fwd_frac": line["fwd_tflops"] / (mhz / 1e3) / nominal_per_ghz,
                                 "fwd_bwd_frac": line["fwd_bwd_tflops"] / (mhz / 1e3) / nominal_per_ghz}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="n512k", choices=list(mi.WORKLOADS))
    ap.add_argument("--mode", default="split", choices=["split", "replicas"],
                    help="N > 1 GPUs: split one sequence's virtual ranks over the GPUs (strong scaling), or run "
                         "one independent sequence per GPU (weak scaling)")
    ap.add_argument("--impl", default="mmsp", choices=["mmsp", "reference"])
    ap.add_argument("--ref-rows", type=int, default=384)
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
