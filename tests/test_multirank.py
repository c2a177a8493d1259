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


def _ep_worker(rank, world, port, out):
    """Expert-parallel exchange logic: counts all-gathered over the process
    group, every rank's plan, and a cross-check that each owner's receive
    layout is exactly what the senders will write (world size 2, gloo)."""
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import sparse_moe_layer_beam_b200 as bm

    cfg = bm.beam_cfg()
    E, El, K = cfg.n_experts, cfg.n_experts // world, cfg.top_k
    t_local = 50 + 30 * rank
    rng = np.random.default_rng(100 + rank)
    ids = np.stack([rng.choice(E, size=K, replace=False) for _ in range(t_local)])
    counts = np.bincount(ids.ravel(), minlength=E).astype(np.int32)
    gathered = [torch.zeros(E, dtype=torch.int32) for _ in range(world)]
    dist.all_gather(gathered, torch.from_numpy(counts))
    counts_all = torch.stack(gathered).numpy()
    ep = bm.ep_cfg(world, rank, 80, world * 80 * K)
    send_base, recv_counts, recv_rows = bm.beam_moe_ep_plan(cfg, ep, counts_all)
    sends = [torch.zeros(E, dtype=torch.int32) for _ in range(world)]
    dist.all_gather(sends, torch.from_numpy(send_base))
    sends = torch.stack(sends).numpy()
    # this rank as owner: every source's rows for each local expert are one
    # contiguous run, in expert then source order, tiling [0, recv_rows)
    row, ok = 0, True
    for j in range(El):
        e = rank * El + j
        for s in range(world):
            ok &= bool(sends[s, e] == row)
            row += counts_all[s, e]
    ok &= row == recv_rows == int(recv_counts.sum())
    out.put((rank, ok, int(recv_rows), int(counts_all.sum())))
    dist.barrier()
    dist.destroy_process_group()


def test_expert_parallel_plan_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + os.getpid() % 1000
    procs = [ctx.Process(target=_ep_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ok0, rows0, tot0), (r1, ok1, rows1, tot1) = res
    assert ok0 and ok1
    assert tot0 == tot1 == (50 + 80) * 8        # every assignment of both ranks
    assert rows0 + rows1 == tot0                 # received exactly once, by its owner


class _FakeWs:
    """Stands in for a workspace tensor on a CPU-only rank."""

    def __init__(self, addr, nbytes):
        self.addr, self.nbytes = addr, nbytes

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


def _ipc_worker(rank, world, port, out):
    """The peer-workspace exchange over a real process group (gloo): every rank
    exports, the blobs are all-gathered, every other rank's blob is imported
    once, the own slot stays local, and close() releases exactly what was
    opened. Export / import / release are fakes (no GPU here); the library's
    CUDA IPC calls are exercised by the GPU test with two processes."""
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import sparse_moe_layer_beam_b200 as bm

    imported, released = [], []

    def export(ws):
        return f"ws-of-{rank}-at-{ws.data_ptr()}".encode()

    def import_(blob, nbytes):
        imported.append((blob, nbytes))
        return 10_000 + int(blob.decode().split("-")[2])

    def release(blob, p):
        released.append((blob, p))

    ep = bm.ep_cfg(world, rank, 64, 1024)
    ws = _FakeWs(4096 * (rank + 1), 777)
    peers = bm.EpPeers(ep, ws, bm.torch_gather(), export, import_, release)
    ptrs = list(peers.ptrs)
    peers.close()
    bad = None
    try:  # a gather that returns the blobs out of rank order is refused
        rotate = lambda b: (lambda v: v[1:] + v[:1])(bm.torch_gather()(b))  # noqa: E731
        bm.EpPeers(ep, ws, rotate, export, import_, release)
    except ValueError as e:
        bad = str(e)
    out.put((rank, ptrs, [b.decode() for b, _ in imported], [p for _, p in released], bad))
    dist.barrier()
    dist.destroy_process_group()


def test_expert_parallel_peer_exchange_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 32500 + os.getpid() % 1000
    world = 3
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ptrs, imported, released, bad in res:
        assert ptrs[rank] == 4096 * (rank + 1)  # the own slot is the local workspace
        others = [r for r in range(world) if r != rank]
        assert [ptrs[r] for r in others] == [10_000 + r for r in others]
        assert imported[:world - 1] == [f"ws-of-{r}-at-{4096 * (r + 1)}" for r in others]
        assert sorted(released) == sorted(10_000 + r for r in others)
        assert bad and "rank order" in bad
