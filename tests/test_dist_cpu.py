"""The multi-GPU path of bench.py on CPU: two gloo ranks.

With N GPUs the benchmark runs N independent replicas (each GPU serves its own
memory bank and queries; no data-path collective). The job's step time is the
maximum over ranks and its throughput counts every rank's units; the
reference arm runs on rank 0 only.
"""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        value, ms = bench.combine_ranks(10.0 + 3.0 * rank, 1000.0, world, device="cpu")
        q.put((rank, value, ms))
    finally:
        dist.destroy_process_group()


def test_replicas_take_max_time_and_sum_units():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, ms in res:
        assert ms == pytest.approx(13.0)
        assert value == pytest.approx(1000.0 * 2 / 13e-3)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""



def test_reference_arm_prints_the_contract_line():
    """Rank 0 of the reference arm times the oracle and prints one JSON line
    with the contract's keys; its cpu_baseline and e2e repeat the line's value."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"]:
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}

def _gather_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from routed_sparse_attention_msa_b200 import memory_parallel as mp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ids = torch.full((3, 4), rank, dtype=torch.int32)
        sc = torch.full((3, 4), 0.5 * rank, dtype=torch.float32)
        all_ids, all_sc = mp.gather_candidates(ids, sc)
        q.put((rank, all_ids.tolist(), all_sc.tolist()))
    finally:
        dist.destroy_process_group()


def test_memory_parallel_candidate_gather_on_gloo():
    """Every rank receives every rank's [S, k] candidates, stacked by rank."""
    pytest.importorskip("routed_sparse_attention_msa_b200")
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for rank, ids, sc in sorted(q.get(timeout=10) for _ in range(world)):
        assert [row[0][0] for row in ids] == [0, 1]
        assert [row[0][0] for row in sc] == [0.0, 0.5]


def test_shard_ranges_balance_chunks():
    from routed_sparse_attention_msa_b200 import memory_parallel as mpar
    import synth
    dco, _ = synth.workload("10m").index()
    r = mpar.shard_ranges(dco, 8)
    assert r[0][0] == 0 and r[-1][1] == dco.size - 1
    assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
    counts = [int(dco[b] - dco[a]) for a, b in r]
    assert max(counts) - min(counts) <= 2 * int(np.diff(dco).max())
    assert mpar.shard_ranges(np.array([0, 5, 5, 9]), 5)[-1] == (3, 3)  # more shards than documents
