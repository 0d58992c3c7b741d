"""The multi-rank path of bench.py on CPU ranks (gloo, world size 2).

Decode shards by sequence with no data-path collective: each rank runs its
own batch (weak scaling), and the only cross-rank step is the max over ranks
of the timed region. These tests run that logic with two gloo ranks.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from paged_kv_cache_335_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        dist.init_process_group("gloo", rank=rank, world_size=world)
        r, lr, ws = bench.dist_env()
        local_ms = 10.0 + 5.0 * rank                        # rank 1 is the slow one
        mx = bench.dist_max(local_ms, "cpu")
        wl = W.tiny()
        vals = W.make_values(wl, "cpu", seed_offset=rank)   # the bench seeds ranks apart
        digest = float(vals["q"].double().sum())
        value = bench.weak_scaling_value(1000, 4, ws, mx)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, r, ws, mx, digest, value, tuple(vals["k_cache"].shape)))
    except Exception as e:  # pragma: no cover
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_max_time_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    out = sorted(out)
    assert all(o[1] != "error" for o in out), out
    (_, r0, ws0, mx0, d0, v0, sh0), (_, r1, ws1, mx1, d1, v1, sh1) = out
    assert (r0, r1) == (0, 1) and ws0 == ws1 == 2
    assert mx0 == mx1 == 15.0                               # max over ranks, seen by both
    assert v0 == v1 == pytest.approx(2 * 1000 * 4 / 0.015 / 1e9)
    assert sh0 == sh1 and d0 != d1                           # same shapes, different data


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        config, steps, warmup = "tiny", 1, 0
    assert bench.reference_arm(A()) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_rank0_prints_one_line(monkeypatch, capsys):
    import json
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class A:
        config, steps, warmup = "tiny", 2, 1
    assert bench.reference_arm(A()) == 0
    lines = capsys.readouterr().out.strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_oracle_sample_is_bounded():
    wl = W.make("llama7b")
    gbs, secs, desc, nbytes = bench.oracle_sample(wl, 0.5, 2)
    assert gbs > 0 and nbytes > 0 and "of 64 sequences" in desc
