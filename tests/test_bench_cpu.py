"""Host-side plumbing of bench.py: max-over-ranks timing and summed units over
a 2-rank gloo group on CPU (the N > 1 path without GPUs)."""
from __future__ import annotations

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = bench.dist_env()
        bench.barrier(w)
        ms, units = bench.aggregate(10.0 + 5.0 * rank, 8.0 * (rank + 1), w)
        q.put((r, lr, w, ms, units))
    finally:
        dist.destroy_process_group()


def test_aggregate_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, lr, w, ms, units) in enumerate(res):
        assert (rank, lr, w) == (r, r, 2)
        assert ms == 15.0 and units == 24.0


def test_aggregate_single_rank_is_identity():
    assert bench.aggregate(3.5, 8.0, 1) == (3.5, 8.0)


def test_profiled_traffic_requires_matching_sources(tmp_path, monkeypatch):
    import json
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    (tmp_path / "traffic_gate_decode_bf16.json").write_text(json.dumps(
        {"source_hash": "stale", "dram_bytes_per_launch": 1.0}))
    assert bench.profiled_traffic("gate", "decode_bf16") is None
    (tmp_path / "traffic_gate_decode_bf16.json").write_text(json.dumps(
        {"source_hash": bench.source_hash("gate"), "dram_bytes_per_launch": 123.0}))
    assert bench.profiled_traffic("gate", "decode_bf16") == 123.0


def test_warmup_floor():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "1"])
