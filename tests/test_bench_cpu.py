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


def test_work_model_decode_matches_byte_formula():
    import synth
    wl = synth.WORKLOADS["decode_bf16"]
    st = {"union": 8163, "nnz": 12000, "block_rows": 8163, "n_overflow": 0}
    b, f = bench.step_work(wl, 8, st)
    P = wl.d_ff // 128
    twell = 8 * P * (2 + 32 * 4)
    assert b == wl.d_ff * wl.d_model * 2 + 8163 * 2 * wl.d_model * 2 + 8 * wl.d_model * (2 + 4) + 2 * twell
    assert f == 2 * 8 * wl.d_model * wl.d_ff + 4 * 12000 * wl.d_model
    w = bench.kernel_work(wl, 8, "rows", st)
    assert set(w) == {"gate", "updown_rows", "fallback_h", "down", "decode_fused"}
    # the single launch moves the step's bytes with the TwELL records and keep
    # masks written once (nothing reads them back inside it)
    assert w["decode_fused"]["bytes"] == b - twell + 8 * P * 16
    # an overflow token's kept rows stream with the others in the single launch
    st2 = dict(st, n_overflow=1, union_all=9000, nnz_all=12500)
    w2 = bench.kernel_work(wl, 8, "rows", st2)
    assert w2["decode_fused"]["bytes"] == w["decode_fused"]["bytes"] + (9000 - 8163) * 2 * wl.d_model * 2
    assert w2["decode_fused"]["flops"] == 2 * 8 * wl.d_model * wl.d_ff + 4 * 12500 * wl.d_model
    # no overflow: the dense channel moves nothing
    assert w["fallback_h"]["bytes"] == 0 and w["down"]["flops"] == 0
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    r = bench.roofline_of(w["gate"], 0.030, peaks, "measured")
    assert r["bound"] == "hbm" and abs(r["achieved"] - w["gate"]["bytes"] / 30e-6 / 1e9) < 0.1


def test_work_model_prefill_gate_is_tensor_bound():
    import synth
    wl = synth.WORKLOADS["prefill_bf16"]
    st = {"union": 8192, "nnz": 4096 * 99, "block_rows": 300000, "n_overflow": 400}
    w = bench.kernel_work(wl, 4096, "rows", st)
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    r = bench.roofline_of(w["gate"], 0.2, peaks, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert w["gate"]["flops"] == 2 * 4096 * 2048 * 8192
    assert w["fallback_h"]["flops"] == 2 * 400 * 2048 * 8192


def test_work_model_tile_path_kernels():
    import synth
    for name, extra in (("lopa_bf16", {"gate_lowrank_z", "fallback_h", "tile_fused"}), ("wina_bf16", {"wina_topk"})):
        wl = synth.WORKLOADS[name]
        st = {"union": 14000, "nnz": 32 * 1400, "block_rows": 4 * 14000, "n_overflow": 1}
        w = bench.kernel_work(wl, 32, "tiles", st)
        assert {"gate", "router", "tile_h", "down"} | extra == set(w)


def test_reference_arm_tiny_workload(capsys):
    import json
    bench.main(["--impl", "reference", "--workload", "tiny_fp32", "--steps", "2", "--warmup", "3"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["steps"] == 2 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["config"]["tokens_per_step"] == 64


def test_tokens_option():
    import json
    with pytest.raises(SystemExit):
        bench.main(["--tokens", "0"])
    # the reference arm takes the override like the GPU arm does
    import io
    import contextlib
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny_fp32", "--tokens", "16", "--steps", "2",
                    "--warmup", "3"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["config"]["tokens_per_step"] == 16 and "tokens=16" in line["config"]["workload"]
