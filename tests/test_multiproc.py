"""Multi-process host logic of the N-GPU benchmark path, on CPU with gloo.

Requests and heads are independent, so N GPUs run N independent shards with
no exchange on the data path; the only collectives are the barrier and the
maximum of the timed interval over ranks.  These tests run two gloo ranks.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(values[rank], dist)
        dist.barrier()
        out_q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    values = [0.125, 0.5]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 0.5, 1: 0.5}


def test_max_over_ranks_without_process_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5


def test_ranks_serve_independent_requests():
    """Weak scaling: each rank draws its own requests (different inputs)."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    w = W.WORKLOADS[1]
    a = W.gdn_inputs(w, bench.rank_input_step(3, 0), B=2)
    b = W.gdn_inputs(w, bench.rank_input_step(3, 1), B=2)
    assert not np.array_equal(a["v"], b["v"])
    assert len({bench.rank_input_step(t, r) for t in range(1000) for r in range(8)}) == 8000


@pytest.mark.slow
def test_reference_arm_under_torchrun_prints_one_line():
    """`bench.py --impl reference` launched like the multi-GPU run: rank 0 alone
    times the oracle and prints one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_emit_appends_jsonl_records(tmp_path):
    """--jsonl: each result line is printed and appended to the file."""
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    path = tmp_path / "r.jsonl"
    args = argparse.Namespace(jsonl=str(path))
    bench.emit({"metric": "head-updates/s", "value": 1.0}, args)
    bench.emit({"metric": "head-updates/s", "value": 2.0}, args)
    recs = [json.loads(l) for l in path.read_text().splitlines()]
    assert [r["value"] for r in recs] == [1.0, 2.0]
    bench.emit({"value": 3.0}, argparse.Namespace(jsonl=None))   # no file: print only
    assert len(path.read_text().splitlines()) == 2


def test_sweep_rows_name_known_workloads():
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    for name, rounding, window, key_axis in bench.SWEEP:
        assert name in W.BY_NAME
        assert rounding is None or rounding in bench.ROUNDING
        assert window in (0, 4, 8, 16) and not (window and key_axis)


def test_algorithmic_bytes_match_the_hand_counts():
    """The roofline numerator: bytes one head update must move (codes and scales
    read and written, inputs, gates, fp32 output), counted by hand per format.
    GDN d=128 bf16: codes 2*16384 (INT8) or 2*8192 (INT4), scales 2*512,
    q/k/v 3*256 + alpha/beta 8, output 512."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    gdn = W.BY_NAME["gdn_b64_h16_d128_int8_sr"]
    assert bench.algorithmic_bytes_per_head(gdn, 8) == 32768 + 1024 + 776 + 512 == 35080
    assert bench.algorithmic_bytes_per_head(gdn, 4) == 16384 + 1024 + 776 + 512 == 18696
    # full-precision state: 4-byte values in both directions, no scales
    assert bench.algorithmic_bytes_per_head(gdn, 32) == 2 * 65536 + 776 + 512 == 132360
    mamba = W.BY_NAME["mamba2_b128_h80_p64_n128_int8_sr"]
    # Mamba-2 N=128, P=64: codes 2*8192, scales 2*256, x 128 + dt 4, output 256
    assert bench.algorithmic_bytes_per_head(mamba, 8) == 16384 + 512 + 132 + 256 == 17284
    # per step: every head, plus B and C once per request (ngroups = 1) and A, D per head
    assert bench.step_bytes(mamba, [8] * mamba.H) == (17284 * mamba.H + 2 * 128 * 2) * mamba.B + 8 * mamba.H
    # the benchmark workload: 1024 head updates of 35080 bytes
    assert bench.step_bytes(gdn, [8] * gdn.H) == 1024 * 35080 == 35921920
    # key-axis groups: one scale per key row (d_k of them)
    import dataclasses
    wide = dataclasses.replace(gdn, dk=64, dv=128)
    assert (bench.algorithmic_bytes_per_head(wide, 8, key_axis=True)
            == bench.algorithmic_bytes_per_head(wide, 8) - 2 * 4 * (128 - 64))
