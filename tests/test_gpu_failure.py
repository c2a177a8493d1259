"""Failure detection on the device without a fault: a bounded wait that nothing
completes gives up after its limit, the kernel records a status bit and
returns, beam_moe_check reports it, and the same context then runs a forward."""
import ctypes

import pytest
import torch

import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu

DEVICE_TIMEOUT = 6


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    bm.beam_moe_selftest_wait(ws, 20)
    flags = ctypes.c_uint32(0)
    st = bm.lib().beam_moe_check(ws.data_ptr(), 256, None, ctypes.byref(flags))
    assert st == DEVICE_TIMEOUT and flags.value == 0x200
    assert bm.beam_moe_check(ws) == 0  # the check cleared the word
    wl = synth.workload("tiny")
    x, _, _, _, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
