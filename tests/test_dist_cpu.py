"""Multi-process path of the benchmark on CPU (gloo, world size 2): every rank
runs the same workload as an independent replica, times are reduced with a
max over ranks, and the whole-job value is all ranks' bytes over that max."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # Rank-dependent "device times": the reduction must return the max.
        mine = [1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)]
        got = bench.reduce_max(mine, torch.device("cpu"))
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_aggregate_gloo_world2():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1] == [2.0, 10.0, 1.0]
    value, t = bench.aggregate([res[0][0]] * world, [1e9] * world)
    assert t == 2.0 and abs(value - 2e9 / 2e-3 / 1e9) < 1e-9


def test_single_process_reduce_is_identity():
    assert bench.reduce_max([3.0, 4.0], torch.device("cpu")) == [3.0, 4.0]


def test_step_bytes_accounting():
    g, q = bench.step_bytes()
    per = sum(o * k // 4 + 4 * o + k + 4 + 4 * o for _, o, k in bench.SHAPES)
    assert g == 30 * per
    assert q == 30 * sum(5 * k + 4 for _, _, k in bench.SHAPES)


def test_read_traffic_scales_and_checks_the_source_digest(tmp_path, monkeypatch):
    # The roofline's traffic comes from a committed ncu record; it is scaled to
    # the launch's algorithmic bytes and reported as null once the kernel's
    # sources differ from those the record was taken on.
    csrc = tmp_path / "ternary_weight_absmax_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_text("// kernel, first version\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"k": {"dram_bytes": 1000, "algorithmic_bytes": 500, "case": "a small case",
                 "sources": ["k.cu"], "source_digest": bench.source_digest("k.cu")}}
    import json
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.read_traffic("k", 500)[0] == 1000
    traffic, note = bench.read_traffic("k", 1500)
    assert traffic == 3000 and "scaled" in note
    assert bench.read_traffic("other", 500) == (None, "no ncu capture on record")
    src.write_text("// kernel, changed\n")
    assert bench.read_traffic("k", 500) == (None, "kernel changed since the ncu capture")


def test_headline_bytes_per_step():
    # codes out*K/4 + a fp32 scale per row + fp32 x + fp32 y, over the 120 linears
    per = sum(o * k // 4 + 4 * o + 4 * k + 4 * o for _, o, k in bench.SHAPES)
    assert bench.fused_step_bytes() == 30 * per == 528230400
