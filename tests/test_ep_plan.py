"""Expert parallelism on the host: beam_moe_ep_plan (where every rank's rows
land in every owner's receive buffer) and the EP entry points' argument checks,
which run before any CUDA call (no GPU needed)."""
import ctypes

import numpy as np
import pytest

import sparse_moe_layer_beam_b200 as bm

OK, INVALID, UNSUPPORTED, ALIGN, WS_SMALL = 0, 1, 2, 3, 4


def _plans(cfg, world, counts_all, cap):
    t_max = int(counts_all.sum(axis=1).max()) // cfg.top_k + 1
    return [bm.beam_moe_ep_plan(cfg, bm.ep_cfg(world, r, t_max, cap), counts_all)
            for r in range(world)]


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_plan_tiles_every_receive_buffer(world):
    cfg = bm.beam_cfg()
    E, El = cfg.n_experts, cfg.n_experts // world
    rng = np.random.default_rng(world)
    counts_all = rng.integers(0, 40, size=(world, E)).astype(np.int32)
    counts_all[0, :5] = 0  # empty (source, expert) pairs
    plans = _plans(cfg, world, counts_all, cap=10**6)
    for o in range(world):
        send = np.stack([plans[s][0] for s in range(world)])  # [source][E]
        _, recv_counts, recv_rows = plans[o]
        assert np.array_equal(recv_counts, counts_all[:, o * El:(o + 1) * El].sum(axis=0))
        assert recv_rows == recv_counts.sum()
        covered = np.zeros(recv_rows, dtype=np.int32)
        row = 0
        for j in range(El):  # expert-major, then source-major, no gaps
            e = o * El + j
            for s in range(world):
                assert send[s, e] == row
                covered[row:row + counts_all[s, e]] += 1
                row += counts_all[s, e]
        assert row == recv_rows and np.all(covered == 1)


def test_plan_refuses_overflow_on_every_rank():
    cfg = bm.beam_cfg()
    world = 4
    counts_all = np.full((world, cfg.n_experts), 3, dtype=np.int32)
    need = world * 3 * (cfg.n_experts // world)  # rows each owner receives
    L = bm.lib()
    for cap, want in ((need, OK), (need - 1, WS_SMALL)):
        for r in range(world):
            ep = bm.ep_cfg(world, r, 1000, cap)
            sb = np.zeros(cfg.n_experts, np.int32)
            rc = np.zeros(cfg.n_experts // world, np.int32)
            n = ctypes.c_int64(0)
            got = L.beam_moe_ep_plan(ctypes.byref(cfg), ctypes.byref(ep), counts_all.ctypes.data,
                                     sb.ctypes.data, rc.ctypes.data, ctypes.byref(n))
            assert got == want


def test_plan_rejects_bad_counts():
    cfg = bm.beam_cfg()
    L = bm.lib()
    ep = bm.ep_cfg(2, 0, 10, 10**6)
    sb = np.zeros(cfg.n_experts, np.int32)
    rc = np.zeros(cfg.n_experts // 2, np.int32)
    n = ctypes.c_int64(0)
    neg = np.zeros((2, cfg.n_experts), np.int32)
    neg[1, 7] = -1
    too_many = np.zeros((2, cfg.n_experts), np.int32)
    too_many[0, :81] = 1  # 81 > t_max * K = 80 assignments
    for bad in (neg, too_many):
        assert L.beam_moe_ep_plan(ctypes.byref(cfg), ctypes.byref(ep), bad.ctypes.data,
                                  sb.ctypes.data, rc.ctypes.data, ctypes.byref(n)) == INVALID


def test_ep_configuration_and_workspace():
    cfg = bm.beam_cfg()
    size = lambda ep: bm.beam_moe_ep_workspace_size(cfg, ep)
    a = size(bm.ep_cfg(8, 0, 64, 4096))
    assert size(bm.ep_cfg(8, 3, 64, 4096)) == a  # same layout on every rank
    assert size(bm.ep_cfg(8, 0, 64, 8192)) > a and size(bm.ep_cfg(8, 0, 128, 4096)) > a
    H, I, K = cfg.hidden, cfg.inter, cfg.top_k
    # receive rows (fp32 after the down GEMM), h, and the returned y rows at least
    assert a >= 4096 * H * 4 + 4096 * I * 2 + 64 * K * H * 4
    L = bm.lib()
    n = ctypes.c_size_t(0)
    for ep, want in ((bm.ep_cfg(3, 0, 64, 4096), UNSUPPORTED),  # 3 does not divide 256
                     (bm.ep_cfg(9, 0, 64, 4096), INVALID), (bm.ep_cfg(2, 2, 64, 4096), INVALID),
                     (bm.ep_cfg(2, -1, 64, 4096), INVALID), (bm.ep_cfg(2, 0, -1, 4096), INVALID)):
        assert L.beam_moe_ep_workspace_size(ctypes.byref(cfg), ctypes.byref(ep),
                                            ctypes.byref(n)) == want


def test_ep_calls_reject_before_any_cuda_call():
    cfg = bm.beam_cfg()
    ep = bm.ep_cfg(2, 0, 64, 1024)
    need = bm.beam_moe_ep_workspace_size(cfg, ep)
    L = bm.lib()
    a = 1 << 20  # fake but aligned addresses: never dereferenced on these paths
    c, g = ctypes.byref(cfg), ctypes.byref(ep)
    peers = (ctypes.c_void_p * 2)(a, a + (1 << 30))
    assert L.beam_moe_ep_route(c, g, 65, a, a, None, a, a, need, None) == INVALID  # T > t_max
    assert L.beam_moe_ep_route(c, g, 64, a, a, None, a, a, need - 1, None) == WS_SMALL
    assert L.beam_moe_ep_route(c, g, 64, a, a, None, a, a + 8, need, None) == ALIGN
    assert L.beam_moe_ep_route(c, g, 64, a, a, None, None, a, need, None) == INVALID
    assert L.beam_moe_ep_dispatch(c, g, 64, a, a, None, a, need, None) == INVALID
    bad_peers = (ctypes.c_void_p * 2)(a + (1 << 30), a)  # peer_ws[rank] is not ws
    assert L.beam_moe_ep_dispatch(c, g, 64, a, a, bad_peers, a, need, None) == INVALID
    rc = np.full(128, 9, np.int32)  # 1152 rows > recv_cap
    assert L.beam_moe_ep_experts(c, g, rc.ctypes.data, a, a, peers, a, need, None) == WS_SMALL
    rc[:] = 0
    assert L.beam_moe_ep_experts(c, g, rc.ctypes.data, a, a, peers, a, need, None) == OK  # no rows
    assert L.beam_moe_ep_combine(c, g, 64, None, a, need, None) == INVALID
    assert L.beam_moe_ep_combine(c, g, 0, None, a, need, None) == OK
