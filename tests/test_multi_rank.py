"""The N > 1 host logic of bench.py on CPU: two gloo ranks (replicas run
their own seeded copies of the layer; the job time is the slowest rank's),
and the reference arm under two ranks (rank 0 alone runs and prints)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    from block_scaled_fp8_fp8blk_b200 import synth, workloads as W
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = bench.replica_workload(W.TINY, rank)
        x = synth.bf16_bits(wl.x_bf16())
        digest = torch.tensor([int(x.astype("int64").sum() % (1 << 31)), wl.seed], dtype=torch.int64)
        gathered = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(gathered, digest)
        slowest = bench.max_over_ranks(10.0 * rank + 5.0, world, "cpu")
        out[rank] = (gathered[0].tolist(), gathered[1].tolist(), slowest)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_and_max_time():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        r0, r1 = out[0], out[1]
    assert r0[:2] == r1[:2]                       # both ranks saw the same gather
    a, b = r0[0], r0[1]
    assert a[1] == b[1] - 1 and a[0] != b[0]      # distinct seeds, distinct inputs
    assert r0[2] == r1[2] == 15.0                 # max over ranks: 10 * 1 + 5


def test_reference_arm_runs_on_rank_zero_only():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--workload", "tiny_m64_k256_n384"]
    outs = []
    for rank in (1, 0):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
        r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    assert outs[0] == ""                          # rank 1: no work, no line
    line = json.loads(outs[1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
