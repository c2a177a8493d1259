"""Expert parallelism across processes: two ranks, each its own process, share
one GPU and reach each other's workspaces through the library's CUDA IPC
calls (beam_moe_ep_export / import / release, exchanged with an all-gather
over a gloo process group), exactly as ranks on different GPUs do over NVLink.
The phases are ordered on the host (device synchronisation, then a gloo
barrier, also after the dispatch): two processes sharing one GPU must not
depend on each other's kernels running at the same time, so every row has
arrived before either experts call starts and its arrival wait returns at
once. Each rank's output must match
the oracle and a single-process forward of the same tokens.

"Welcome Beam" (section "Mixture of Experts") and the vLLM recipe page run
Beam's experts split over GPUs with all-to-all dispatch and combine."""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def _rank(rank, world, port, Ts, out):
    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        torch.cuda.set_device(0)
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
        import sparse_moe_layer_beam_b200 as bm
        import synth
        from tests import _gpu, _inputs

        wl = synth.workload("tiny")
        cfg = _gpu.cfg_of(wl)
        w13, w2, wr = _gpu.device_weights(wl)
        El = wl.E // world
        x_all, _, _, _, _ = _inputs.routed_inputs(wl.with_T(sum(Ts)))
        x = x_all[sum(Ts[:rank]):sum(Ts[:rank + 1])]
        cap = sum(Ts) * min(wl.K, El)
        ep = bm.ep_cfg(world, rank, max(Ts), cap)
        ws = torch.empty(bm.beam_moe_ep_workspace_size(cfg, ep), dtype=torch.uint8,
                         device="cuda")
        peers = bm.EpPeers(ep, ws, bm.torch_gather())
        xd = _gpu.to_dev_bits(x)
        counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
        bm.beam_moe_ep_route(cfg, ep, xd, wr, None, counts, ws)
        gathered = [torch.zeros(wl.E, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, counts.cpu())
        counts_all = torch.stack(gathered).numpy()
        send_base, recv_counts, recv_rows = bm.beam_moe_ep_plan(cfg, ep, counts_all)
        bm.beam_moe_ep_dispatch(cfg, ep, xd, torch.from_numpy(send_base).cuda(), peers.ptrs, ws)
        torch.cuda.synchronize()
        dist.barrier()  # every rank's rows are in their owners' workspaces
        w13_bytes, w2_bytes = 2 * wl.I * wl.H * 2, wl.H * wl.I * 2
        bm.beam_moe_ep_experts(cfg, ep, recv_counts, w13.data_ptr() + rank * El * w13_bytes,
                               w2.data_ptr() + rank * El * w2_bytes, peers.ptrs, ws)
        torch.cuda.synchronize()
        dist.barrier()  # every y row is back at its source
        o = torch.empty((Ts[rank], wl.H), dtype=torch.int16, device="cuda")
        bm.beam_moe_ep_combine(cfg, ep, Ts[rank], o, ws)
        flags = bm.beam_moe_check(ws)
        got = _gpu.bits_of(o)
        single = _gpu.forward(wl.with_T(Ts[rank]), x)["out"]
        dist.barrier()  # nobody stores into a peer any more
        peers.close()
        dist.barrier()  # every mapping of this rank's workspace is closed
        out.put((rank, None, flags, int(recv_rows), got, single))
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        import traceback
        out.put((rank, traceback.format_exc()[-3000:] + repr(e), None, None, None, None))


@pytest.mark.parametrize("Ts", [[100, 37], [900, 600]])  # copy-kernel return; pair epilogue
def test_ep_two_processes_one_gpu_through_ipc(Ts):
    import oracle
    import synth
    from tests import _gpu, _inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 33500 + os.getpid() % 1000 + Ts[0] % 7
    procs = [ctx.Process(target=_rank, args=(r, 2, port, Ts, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=600) for _ in procs), key=lambda v: v[0])
    for p in procs:
        p.join(timeout=120)
    for rank, err, *_ in res:
        assert err is None, f"rank {rank}: {err}"
    assert all(p.exitcode == 0 for p in procs)
    wl = synth.workload("tiny")
    x, _, wr, b, r = _inputs.routed_inputs(wl.with_T(sum(Ts)))
    assert sum(v[3] for v in res) == sum(Ts) * wl.K  # every assignment received once
    got = np.concatenate([v[4] for v in res])
    ref = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], synth.host_w13(wl),
                         synth.host_w2(wl))
    err, rms = _gpu.max_rel_err(got, ref)
    assert err <= _gpu.TOL, (err, rms)
    for rank, _, flags, _, o, single in res:
        assert flags == 0
        err, rms = _gpu.max_rel_err(o, synth.bf16_to_f32(single).astype(np.float64))
        assert err <= _gpu.TOL, (rank, err, rms)
