"""Host-side logic of bench.py on CPU: the max-over-ranks reduction with two
gloo ranks, whole-job throughput, and the reference (oracle) arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    vals = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 1.0 * rank], ws)
    out.put((rank, vals))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [11.0, 5.0, 1.0]


def test_job_throughput_is_whole_job():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.job_throughput(2e15, 4, 1000.0) == pytest.approx(8000.0)


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "n4k",
                        "--steps", "1", "--warmup", "3", "--ref-rows", "16"], capture_output=True, text=True,
                       timeout=600, env=env)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["workload"] == "n4k"


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "n4k",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and "{" not in r.stdout


def test_cpu_baseline_rows_come_from_the_parity_sample():
    """The oracle timed as the CPU baseline runs on rows of the seeded sample
    the full-size parity tests check: a sorted subset of the requested size,
    spread over the sequence, and a different subset for another part."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import bench
    import mmsp_inputs as mi

    w = mi.WORKLOADS["n128k"]
    sample = mi.sample_rows(w.N, w.C, bench.PARITY_ROWS, 3000 + w.index)
    a = bench.parity_rows(w, 384)
    b = bench.parity_rows(w, 384, part=1)
    assert len(a) == 384 and len(b) == 384
    assert np.all(np.diff(a) > 0) and np.isin(a, sample).all() and np.isin(b, sample).all()
    assert not np.array_equal(a, b)
    assert a[0] < w.N // 8 and a[-1] > w.N - w.N // 8  # spread over the sequence
    assert len(bench.parity_rows(w, 10 * len(sample))) == len(sample)  # at most the whole sample
