"""The bench's multi-GPU plumbing on CPU: two gloo ranks, no GPU.

The path shards with no exchange step -- each GPU runs an independent problem, or owns a
share of one problem's heads -- so the process group only carries the start/stop barrier,
the max-over-ranks reduction of the timed region and the sum of the ranks' executed work.
These tests run that plumbing as two processes on the host.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_25_b200 import synth
    w, r, local, pg = bench.dist_setup(None)
    assert (w, r, local) == (world, rank, rank) and pg is not None
    bench.barrier(pg)
    # the timed region is the slowest rank's
    out[rank] = bench.max_over_ranks(1.5 + rank, pg)
    # each rank draws its own problem (different seeds), as the bench does
    wl = synth.WORKLOADS["tiny"]
    q, _, _ = synth.draw_qkv(wl.scaled(seed=wl.seed + 7919 * rank))
    out[world + rank] = float(q.double().sum())
    # --split heads: every rank draws the one problem and keeps its heads; the shares
    # cover the heads once, and the executed work adds up over the ranks
    h0, h1 = bench.head_range(rank, world, wl.heads)
    qf, _, _ = synth.draw_qkv(wl)
    mine = qf[:, :, h0:h1].contiguous()
    out[2 * world + rank] = float(mine.double().sum())
    out[3 * world + rank] = bench.sum_over_ranks(float(h1 - h0), pg)
    bench.barrier(pg)
    pg.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_draw_independent_problems():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Array("d", 4 * world)
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert list(out[:world]) == [1.5 + world - 1] * world
    assert out[world] != out[world + 1]
    # the head shares of one problem add up to the whole problem
    from block_sparse_attention_25_b200 import synth
    wl = synth.WORKLOADS["tiny"]
    qf, _, _ = synth.draw_qkv(wl)
    assert abs(out[2 * world] + out[2 * world + 1] - float(qf.double().sum())) < 1e-9
    assert list(out[3 * world:]) == [float(wl.heads)] * world


def test_head_ranges_partition_the_heads():
    sys.path.insert(0, ROOT)
    import bench
    for heads, world in ((40, 1), (40, 2), (40, 4), (40, 8), (24, 8), (12, 4)):
        seen = []
        for r in range(world):
            h0, h1 = bench.head_range(r, world, heads)
            assert h1 - h0 == heads // world
            seen += list(range(h0, h1))
        assert seen == list(range(heads))
    with pytest.raises(ValueError):
        bench.head_range(0, 3, 40)


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    w, r, local, pg = bench.dist_setup(None)
    assert (w, r, local, pg) == (1, 0, 0, None)
    assert bench.max_over_ranks(3.25, pg) == 3.25


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0(tmp_path):
    """bench.py --impl reference launched as two gloo ranks: rank 0 times the oracle and
    prints the JSON line, rank 1 exits without work, and both leave cleanly."""
    import json
    import subprocess
    port = _free_port()
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "1", "--cpu-sample-rows", "2", "--config", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
