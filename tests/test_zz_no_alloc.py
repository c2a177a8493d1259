"""beam_moe_route_noalloc: routing for callers that cannot allocate device
memory (a serving process whose pool already holds the GPU's memory, or a
runtime that forbids allocations after start-up). Its scratch is a fixed array
inside the library, so these tests check that it gives the same routes as the
workspace-based beam_moe_route on two calls in a row with different inputs
(the array keeps the previous call's contents), and that it refuses sizes
beyond its limits before launching anything.

Kept in a file that pytest collects last, so a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu


def _route_with_workspace(cfg, x, wr, T, E, K):
    ids = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, T, bm.OP_ROUTE), dtype=torch.uint8,
                     device="cuda")
    bm.beam_moe_route(cfg, x, wr, None, ids, w, counts, ws)
    return ids.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()


def _route_noalloc(cfg, x, wr, T, E, K):
    ids = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -7.0, dtype=torch.float32, device="cuda")
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    st = bm.lib().beam_moe_route_noalloc(ctypes.byref(cfg), T, x.data_ptr(), wr.data_ptr(),
                                         None, ids.data_ptr(), w.data_ptr(), counts.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 0, bm.lib().beam_moe_status_string(st)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()


def test_noalloc_route_matches_workspace_route_twice_in_a_row():
    wl = synth.workload("decode")
    cfg = _gpu.cfg_of(wl)
    _, _, wr = _gpu.device_weights(wl)
    x300, _, _, _, r300 = _inputs.routed_inputs(wl.with_T(300))
    rev = np.arange(299, 235, -1)  # second call: 64 other tokens, in reverse order
    cases = ((x300, r300), (x300[rev], {k: v[rev] for k, v in r300.items()}))
    for x_bits, r in cases:  # consecutive calls with different sizes and tokens
        T = x_bits.shape[0]
        x = _gpu.to_dev_bits(x_bits)
        ref_ids, ref_w, ref_counts = _route_with_workspace(cfg, x, wr, T, wl.E, wl.K)
        got_ids, got_w, got_counts = _route_noalloc(cfg, x, wr, T, wl.E, wl.K)
        gi, gw = _gpu.sorted_routes(got_ids, got_w)
        ri, rw = _gpu.sorted_routes(ref_ids, ref_w)
        assert np.array_equal(gi, ri)
        assert np.array_equal(got_counts, ref_counts)
        assert np.allclose(gw, rw, rtol=1e-5, atol=1e-6)
        _gpu.check_routes({"ids": got_ids, "w": got_w, "counts": got_counts}, r, wl.E)


def test_noalloc_route_refuses_sizes_beyond_its_limits():
    wl = synth.workload("decode")
    cfg = _gpu.cfg_of(wl)
    a = 1 << 20  # never dereferenced: the size check comes first
    L = bm.lib()
    assert L.beam_moe_route_noalloc(ctypes.byref(cfg), 2049, a, a, None, a, a, None,
                                    None) == 4
    big = _gpu.cfg_of(wl)
    big.n_experts, big.n_group = 512, 16
    assert L.beam_moe_route_noalloc(ctypes.byref(big), 64, a, a, None, a, a, None, None) == 4
