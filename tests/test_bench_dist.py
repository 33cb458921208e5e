"""bench.py's host-side logic: algorithmic work counts, and the multi-rank timing
plumbing (barrier, max over ranks, whole-job aggregation) on CPU with gloo,
world_size 2."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from synth import WORKLOADS


def test_algorithmic_counts():
    nb, fl = bench.algorithmic(WORKLOADS["gdn_prefill"])
    th = 4096 * 32
    assert fl == th * 180224
    assert nb == th * 1032 + 32 * 128 * 128 * 4           # + final state write
    nb, _ = bench.algorithmic(WORKLOADS["kda_prefill"])
    assert nb == th * 1540 + 32 * 128 * 128 * 4
    nb, _ = bench.algorithmic(WORKLOADS["decode_gdn"])
    assert nb == 2 * 256 * 32 * 128 * 128 * 4 * 512        # state read + write per step
    nb, _ = bench.algorithmic(WORKLOADS["kda_long"])
    assert nb == 4 * 65536 * 32 * 1540 + 2 * 4 * 32 * 128 * 128 * 4


def test_aggregate_single_rank():
    assert bench.aggregate(1000, 500.0, 1) == pytest.approx(2000.0)
    assert bench.max_over_ranks(3.5, False, torch.device("cpu")) == 3.5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_env()
    active = bench.dist_init(w, "gloo")
    bench.barrier(active, torch.device("cpu"))
    my_ms = 100.0 + 50.0 * r                       # rank 1 is the slow one
    mx = bench.max_over_ranks(my_ms, active, torch.device("cpu"))
    value = bench.aggregate(tokens_per_rank=4096, max_ms=mx, world=w)
    bench.barrier(active, torch.device("cpu"))
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, active, mx, value))


def test_two_rank_gloo_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for r, active, mx, value in res:
        assert active
        assert mx == 150.0                          # max over ranks, not the local time
        assert value == pytest.approx(4096 * 2 / 0.150)


def test_verify_algorithmic_bytes_count_state_and_snapshots():
    """A verify call reads the state once and writes one full snapshot per token."""
    import bench
    from synth import WORKLOADS
    w = WORKLOADS["verify_gdn"]
    state = w.B * w.H * w.dv * w.dk * 4
    nb, flops = bench.algorithmic(w)
    assert (1 + w.T) * state < nb < (1 + w.T) * state * 1.02
    assert flops == w.B * w.T * w.H * 6 * w.dk * w.dv


def test_traffic_records_name_their_sources_and_captures():
    """Every DRAM-traffic record in profiles/traffic.json names source files that exist
    and the committed summary it came from; a record is used only while the digest of
    those sources is unchanged."""
    import json
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    recs = json.load(open(os.path.join(root, "profiles", "traffic.json")))
    assert recs
    for key, rec in recs.items():
        srcs = rec["source"] if isinstance(rec["source"], list) else [rec["source"]]
        for src in srcs:
            assert os.path.exists(os.path.join(root, src)), (key, src)
        assert os.path.exists(os.path.join(root, rec["capture"])), key
        assert rec["dram_bytes_per_launch"] > 0
        current = bench.source_sha(rec["source"]) == rec["source_sha"]
        assert (bench.load_traffic(key) is not None) == current, key
    assert bench.load_traffic("no such kernel") is None
