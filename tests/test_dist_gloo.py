"""Multi-rank host logic on CPU with world_size-2 gloo process groups.

The GPU path has no collective (rows are independent); what runs across ranks
is host logic: the row partition, the max-over-ranks timing reduction, and
the benchmark's rank-0-only reporting.  These run here as gloo ranks.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from conftest import ROOT

WORLD = 2


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from w4a4_mxfp4_post_b200 import shard, synth

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        M, d = 37, 96
        x = synth.activation("pixart", M, d, 7)
        F = synth.factors(d // 32, 7)
        r0, r1 = shard.row_range(M, world, rank)
        c, s = oracle.kq_quantize(x[r0:r1], F)
        # gather variable-size shards (pad to the largest)
        n = torch.tensor([r1 - r0])
        sizes = [torch.zeros(1, dtype=torch.long) for _ in range(world)]
        dist.all_gather(sizes, n)
        mx = int(max(t.item() for t in sizes))
        pc = torch.zeros((mx, d // 2), dtype=torch.uint8)
        pc[: r1 - r0] = torch.from_numpy(c)
        ps = torch.zeros((mx, d // 32), dtype=torch.uint8)
        ps[: r1 - r0] = torch.from_numpy(s)
        gc = [torch.zeros_like(pc) for _ in range(world)]
        gs = [torch.zeros_like(ps) for _ in range(world)]
        dist.all_gather(gc, pc)
        dist.all_gather(gs, ps)
        # max over ranks of per-rank timings
        mine = [1.0 + rank, 10.0 - rank, 0.5 * rank]
        red = bench.allreduce_max(dist, mine, "cpu")
        bench.barrier(dist)
        if rank == 0:
            codes = np.concatenate([g[: int(k.item())].numpy() for g, k in zip(gc, sizes)])
            scales = np.concatenate([g[: int(k.item())].numpy() for g, k in zip(gs, sizes)])
            cr, sr = oracle.kq_quantize(x, F)
            q.put({"codes_equal": bool(np.array_equal(codes, cr)), "scales_equal": bool(np.array_equal(scales, sr)),
                   "max": red})
    finally:
        dist.destroy_process_group()


def test_row_shards_and_max_reduce_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, WORLD, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = q.get(timeout=10)
    assert res["codes_equal"] and res["scales_equal"]
    assert res["max"] == [2.0, 10.0, 0.5]


def test_row_range_partition():
    from w4a4_mxfp4_post_b200 import shard

    for M in (0, 1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            rs = [shard.row_range(M, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [r1 - r0 for r0, r1 in rs]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.row_range(4, 2, 2)


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched as 2 ranks: rank 0 prints one JSON line, rank 1 exits 0."""
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(WORLD),
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", str(WORLD),
           "--steps", "3", "--warmup", "3", "--ref-seconds", "2"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == WORLD and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
