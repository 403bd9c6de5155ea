"""The multi-rank path of bench.py (replicas: the layer shards by batch with no
exchange), exercised on the CPU: two gloo ranks agree on the slowest rank's
time, the job throughput counts every rank's tokens, each rank draws its own
batch with the same weights, and the reference arm prints on rank 0 only."""

import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks([2.5, 7.0][rank], dist, "cpu")
        cfg = synth.get_config("tiny_bf16_T64")
        x, w_router, bias = bench.replica_inputs(cfg, rank, "cpu")
        assert bench.replica_config(cfg, rank).T == cfg.T
        q.put((rank, slowest, float(x.float().sum()), float(w_router.float().sum()),
               float(bias.float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_replicas_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    (_, m0, x0, r0, w0), (_, m1, x1, r1, w1) = results
    assert m0 == m1 == 7.0              # every rank reports the slowest rank's time
    assert x0 != x1                     # each rank runs its own batch
    assert (r0, w0) == (r1, w1)         # with the same router weights and bias


def test_job_throughput_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_tokens_per_s(2048, 4, 0.5) == pytest.approx(4 * 2048 / 0.5e-3)
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
         "--config", "tiny_bf16_T64", "--steps", "1", "--warmup", "0", "--ref-tokens", "8"],
        capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    if rank:
        assert lines == []
    else:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["n_gpus"] == 2
        assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
