"""Host logic of the N > 1 path, on CPU with gloo, world size 2: each rank runs
its own token batch (different seeds, same experts), the only collective is the
max of the per-rank timings, and the reference arm prints from rank 0 only."""
import json
import os
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import synth

    got = bench.max_over_ranks([10.0 + rank, 5.0 - rank], "cpu")
    wl = synth.workload("tiny")
    x = synth.host_x(wl, seed=bench.rank_seed(rank))
    out.put((rank, got, x[:2].copy(), synth.host_w13(wl)[:1, :2].copy()))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_per_rank_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, g0, x0, w0), (r1, g1, x1, w1) = res
    assert g0 == g1 == [11.0, 5.0]           # max over ranks, element-wise
    assert not np.array_equal(x0, x1)          # each rank its own tokens
    assert np.array_equal(w0, w1)              # the same experts everywhere


def test_reference_arm_prints_on_rank0_only():
    port = 30500 + os.getpid() % 1000
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
