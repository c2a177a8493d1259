"""Expert parallelism, with `world` ranks emulated on one GPU: every rank has
its own workspace, peer pointers are the other ranks' workspaces, and the
phases run rank after rank in stream order (a device synchronisation stands
for the barrier after the experts; none is needed after the dispatch, whose
arrival counts the gate/up GEMM waits on).
The kernels are the ones a multi-GPU run uses; only the peer stores stay on
one device. Each rank's output must match the oracle and a single-GPU forward
of the same tokens."""
import numpy as np
import pytest
import torch

import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu


def ep_forward(wl, xs, world, bias=None, fill=None, extra_rows=0):
    """The five phases over emulated ranks. fill: a byte every workspace holds
    before the first call (its status word excepted); extra_rows: rows each
    owner is told its last local expert received beyond what was dispatched.
    Returns (outputs, counts_all, plans, status bits of every rank)."""
    cfg = _gpu.cfg_of(wl)
    w13, w2, wr = _gpu.device_weights(wl)
    El, H = wl.E // world, wl.H
    Ts = [x.shape[0] for x in xs]
    cap = sum(Ts) * min(wl.K, El)
    eps = [bm.ep_cfg(world, r, max(Ts), cap) for r in range(world)]
    wss = [torch.empty(bm.beam_moe_ep_workspace_size(cfg, ep), dtype=torch.uint8, device="cuda")
           for ep in eps]
    if fill is not None:
        for ws in wss:
            ws.fill_(fill)
            ws[:256].zero_()  # the status word
    peers = [ws.data_ptr() for ws in wss]
    xd = [_gpu.to_dev_bits(x) if x.shape[0] else torch.empty((0, H), dtype=torch.int16,
                                                              device="cuda") for x in xs]
    b = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    counts = [torch.empty(wl.E, dtype=torch.int32, device="cuda") for _ in range(world)]
    for r in range(world):
        bm.beam_moe_ep_route(cfg, eps[r], xd[r], wr, b, counts[r], wss[r])
    counts_all = np.stack([c.cpu().numpy() for c in counts])  # the all-gather
    plans = [bm.beam_moe_ep_plan(cfg, eps[r], counts_all) for r in range(world)]
    for r in range(world):
        bm.beam_moe_ep_dispatch(cfg, eps[r], xd[r], torch.from_numpy(plans[r][0]).cuda(), peers,
                                wss[r])
    w13_bytes, w2_bytes = 2 * wl.I * wl.H * 2, wl.H * wl.I * 2  # one expert's weights
    for r in range(world):
        recv = plans[r][1].copy()
        recv[-1] += extra_rows
        bm.beam_moe_ep_experts(cfg, eps[r], recv, w13.data_ptr() + r * El * w13_bytes,
                               w2.data_ptr() + r * El * w2_bytes, peers, wss[r])
    torch.cuda.synchronize()  # barrier: every y row is back at its source
    outs = []
    for r in range(world):
        out = torch.empty((Ts[r], H), dtype=torch.int16, device="cuda")
        bm.beam_moe_ep_combine(cfg, eps[r], Ts[r], out, wss[r])
        outs.append(_gpu.bits_of(out))
    return outs, counts_all, plans, [bm.beam_moe_check(ws) for ws in wss]


def _check(wl, world, Ts, n_sample=None, fill=None, extra_rows=0, want_flags=0):
    T = sum(Ts)
    x, _, wr, b, r = _inputs.routed_inputs(wl.with_T(T))
    xs = np.split(x, np.cumsum(Ts)[:-1])
    outs, counts_all, plans, flags = ep_forward(wl, xs, world, b, fill, extra_rows)
    assert flags == [want_flags] * world
    assert sum(p[2] for p in plans) == T * wl.K  # every assignment received once
    got = np.concatenate(outs)
    tokens = np.arange(T) if n_sample is None else synth.sample_tokens(T, n_sample)
    ref = _gpu.oracle_outputs(wl.with_T(T), x, tokens, r)
    err, rms = _gpu.max_rel_err(got[tokens], ref)
    assert err <= _gpu.TOL, (err, rms)
    for xr, o in zip(xs, outs):  # the same tokens through one GPU's forward
        if xr.shape[0]:
            single = _gpu.forward(wl.with_T(xr.shape[0]), xr, bias=b)["out"]
            err, rms = _gpu.max_rel_err(o, synth.bf16_to_f32(single).astype(np.float64))
            assert err <= _gpu.TOL, (err, rms)


@pytest.mark.parametrize("world,Ts", [(1, [77]), (2, [100, 37]), (4, [64, 1, 129, 0])])
def test_ep_tiny(world, Ts):
    _check(synth.workload("tiny"), world, Ts)


@pytest.mark.parametrize("world,Ts", [(2, [900, 600]), (4, [700, 5, 500, 300])])
def test_ep_tiny_many_rows(world, Ts):
    """Hundreds of rows per local expert: the down GEMM runs on CTA pairs and
    its epilogue stores every y row straight into the source rank's
    workspace (no separate return pass)."""
    _check(synth.workload("tiny"), world, Ts)


def test_ep_decode_full_size_eight_ranks():  # 32 experts per rank, 64 tokens each
    """Every output row of all eight ranks against the oracle."""
    _check(synth.workload("decode"), 8, [64] * 8)


@pytest.mark.parametrize("Ts", [[900, 600], [100, 37]])
def test_ep_return_address_out_of_range_is_dropped_and_flagged(Ts):
    """Each owner is told its last local expert received 16 rows more than any
    rank dispatched. Those rows never arrive: the gate/up GEMM's bounded wait
    for them runs out (status bit 0x1000) and it goes on. Their return
    addresses keep the workspace's 0xFF fill, which names no rank, so the
    experts phase computes those rows but stores none of them, and sets
    status bit 0x400. Both return paths are covered:
    the pair down GEMM's own stores ([900, 600]) and the copy after the 1-CTA
    GEMM ([100, 37]). Every access stays inside the workspaces, and the real
    rows' outputs still match the oracle."""
    _check(synth.workload("tiny"), 2, Ts, fill=0xFF, extra_rows=16, want_flags=0x1400)


def test_ep_dispatch_outside_the_receive_buffer_is_dropped_and_flagged():
    """Rank 0 dispatches with a send_base that is not its plan: every row
    shifted past the owners' receive capacity (as counts from another step
    could place them), then every row at a negative place. No row is stored:
    the peer's workspace is unchanged byte for byte, rank 0's own workspace
    changes only in its status word and its combine positions, and status
    bit 0x800 is set."""
    wl = synth.workload("tiny")
    world, Ts = 2, [100, 37]
    cfg = _gpu.cfg_of(wl)
    _, _, wr = _gpu.device_weights(wl)
    x, _, _, b, _ = _inputs.routed_inputs(wl.with_T(sum(Ts)))
    xs = np.split(x, np.cumsum(Ts)[:-1])
    cap = sum(Ts) * wl.K
    eps = [bm.ep_cfg(world, r, max(Ts), cap) for r in range(world)]
    wss = [torch.empty(bm.beam_moe_ep_workspace_size(cfg, ep), dtype=torch.uint8, device="cuda")
           for ep in eps]
    for ws in wss:
        ws.fill_(0x5A)
        ws[:256].zero_()
    peers = [ws.data_ptr() for ws in wss]
    xd = [_gpu.to_dev_bits(v) for v in xs]
    counts = [torch.empty(wl.E, dtype=torch.int32, device="cuda") for _ in range(world)]
    for r in range(world):
        bm.beam_moe_ep_route(cfg, eps[r], xd[r], wr, None, counts[r], wss[r])
    counts_all = np.stack([c.cpu().numpy() for c in counts])
    send_base = bm.beam_moe_ep_plan(cfg, eps[0], counts_all)[0]
    for bad in (send_base + cap, np.full_like(send_base, -(1 << 20))):
        before = [ws.cpu().numpy().copy() for ws in wss]
        bm.beam_moe_ep_dispatch(cfg, eps[0], xd[0], torch.from_numpy(bad.astype(np.int32)).cuda(),
                                peers, wss[0])
        assert bm.beam_moe_check(wss[0]) == 0x800
        after = [ws.cpu().numpy() for ws in wss]
        assert np.array_equal(after[1], before[1])
        changed = np.count_nonzero(after[0][256:] != before[0][256:])
        assert changed <= Ts[0] * wl.K * 4  # the combine positions (-1 for every slot)
