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


def _route_with_workspace(cfg, x, wr, T, E, K, bias=None):
    ids = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, T, bm.OP_ROUTE), dtype=torch.uint8,
                     device="cuda")
    bm.beam_moe_route(cfg, x, wr, bias, ids, w, counts, ws)
    return ids.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()


def _noalloc_call(cfg, x, wr, bias, ids, w, counts):
    st = bm.lib().beam_moe_route_noalloc(ctypes.byref(cfg), x.shape[0], x.data_ptr(),
                                         wr.data_ptr(), None if bias is None else bias.data_ptr(),
                                         ids.data_ptr(), w.data_ptr(), counts.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 0, bm.lib().beam_moe_status_string(st)


def _route_noalloc(cfg, x, wr, T, E, K, bias=None):
    ids = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -7.0, dtype=torch.float32, device="cuda")
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    _noalloc_call(cfg, x, wr, bias, ids, w, counts)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()


def _compare(cfg, wl, x_bits, r, bias=None):
    T = x_bits.shape[0]
    x = _gpu.to_dev_bits(x_bits)
    _, _, wr = _gpu.device_weights(wl)
    b = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    ref_ids, ref_w, ref_counts = _route_with_workspace(cfg, x, wr, T, wl.E, wl.K, b)
    got_ids, got_w, got_counts = _route_noalloc(cfg, x, wr, T, wl.E, wl.K, b)
    gi, gw = _gpu.sorted_routes(got_ids, got_w)
    ri, rw = _gpu.sorted_routes(ref_ids, ref_w)
    assert np.array_equal(gi, ri)
    assert np.array_equal(got_counts, ref_counts)
    assert np.allclose(gw, rw, rtol=1e-5, atol=1e-6)
    _gpu.check_routes({"ids": got_ids, "w": got_w, "counts": got_counts}, r, wl.E)


def test_noalloc_route_matches_workspace_route_twice_in_a_row():
    wl = synth.workload("decode")
    cfg = _gpu.cfg_of(wl)
    x300, _, _, _, r300 = _inputs.routed_inputs(wl.with_T(300))
    rev = np.arange(299, 235, -1)  # second call: 64 other tokens, in reverse order
    cases = ((x300, r300), (x300[rev], {k: v[rev] for k, v in r300.items()}))
    for x_bits, r in cases:  # consecutive calls with different sizes and tokens
        _compare(cfg, wl, x_bits, r)


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


def test_noalloc_route_at_its_token_limit_and_with_a_bias():
    """2048 tokens (the limit: the router's H split shrinks until the partial
    logits fit the fixed array), then the skewed workload's +3.0 logit bias on
    16 experts, back to back on the shared array."""
    wl = synth.workload("decode")
    cfg = _gpu.cfg_of(wl)
    x, _, _, _, r = _inputs.routed_inputs(wl.with_T(2048))
    _compare(cfg, wl, x, r)
    sk = synth.workload("skewed").with_T(700)
    x, _, _, b, r = _inputs.routed_inputs(sk)
    assert b is not None
    _compare(_gpu.cfg_of(sk), sk, x, r, bias=b)


def test_noalloc_route_allocates_no_device_memory():
    """After a first call (which looks up the array's address), further calls
    leave the device's free memory and torch's allocation unchanged."""
    wl = synth.workload("decode")
    cfg = _gpu.cfg_of(wl)
    _, _, wr = _gpu.device_weights(wl)
    x = _gpu.to_dev_bits(synth.host_x(wl.with_T(1024)))
    ids = torch.empty((1024, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((1024, wl.K), dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    _noalloc_call(cfg, x, wr, None, ids, w, counts)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        _noalloc_call(cfg, x, wr, None, ids, w, counts)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == alloc0
