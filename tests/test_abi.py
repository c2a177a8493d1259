"""The C ABI on the host: the library loads without a GPU, exports every symbol
include/*.h declares, sizes workspaces, and rejects bad arguments before any
CUDA call (these tests run on a machine with no GPU)."""
import ctypes
import glob
import os
import re

import pytest

import sparse_moe_layer_beam_b200 as bm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, ALIGN, WS_SMALL = 0, 1, 2, 3, 4


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"\b(beam_moe_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert {"beam_moe_route", "beam_moe_forward", "beam_moe_workspace_size",
            "beam_moe_status_string"} <= names
    L = ctypes.CDLL(bm.LIB_PATH)
    for n in sorted(names):
        assert hasattr(L, n), n


def test_status_strings():
    for s in range(7):
        assert bm.lib().beam_moe_status_string(s)
    assert bm.lib().beam_moe_status_string(99) == b"unknown status"


def ws_size(cfg, T, op=bm.OP_FORWARD):
    n = ctypes.c_size_t(0)
    st = bm.lib().beam_moe_workspace_size(ctypes.byref(cfg), T, op, ctypes.byref(n))
    return st, n.value


def test_workspace_size_scales_and_covers_intermediates():
    cfg = bm.beam_cfg()
    st, n64 = ws_size(cfg, 64)
    assert st == OK
    st, n4k = ws_size(cfg, 4096)
    A = 4096 * 8
    # permuted rows (A x H) and SwiGLU activations (A x I), bf16
    assert n4k >= A * 5120 * 2 + A * 2560 * 2
    assert n4k > n64
    st, r4k = ws_size(cfg, 4096, bm.OP_ROUTE)
    assert st == OK and r4k < n4k / 4
    assert ws_size(cfg, 0) == (OK, 0)


@pytest.mark.parametrize("field,value,code", [
    ("n_group", 7, INVALID),        # 256 experts do not split into 7 groups
    ("topk_group", 9, INVALID),     # more kept groups than groups
    ("top_k", 129, INVALID),        # more experts than the kept groups hold
    ("renormalize", 2, INVALID),
    ("bias_mode", 3, INVALID),
    ("router_tc", 2, INVALID),
    ("hidden", 5000, UNSUPPORTED),  # not a multiple of 128
    ("inter", 2500, UNSUPPORTED),
    ("n_experts", 1024, UNSUPPORTED),
    ("top_k", 0, INVALID),
])
def test_bad_configuration(field, value, code):
    cfg = bm.beam_cfg()
    setattr(cfg, field, value)
    assert ws_size(cfg, 64)[0] == code


def test_group_layout_limits():
    # 256 experts in 64 groups of 4: a lane would hold experts of two groups
    cfg = bm.beam_cfg(G=64, Gk=8)
    assert ws_size(cfg, 64)[0] == UNSUPPORTED
    assert ws_size(bm.beam_cfg(H=256, I=128, E=16, G=4, Gk=2, K=4), 64)[0] == OK
    assert ws_size(bm.beam_cfg(), -1)[0] == INVALID
    assert ws_size(bm.beam_cfg(), 1 << 28)[0] == UNSUPPORTED


def _fwd(cfg, T, x, wr, w13, w2, out, ws, nbytes):
    return bm.lib().beam_moe_forward(ctypes.byref(cfg), T, x, wr, None, w13, w2, out, None, None,
                                     None, ws, nbytes, None)


def test_forward_rejects_before_any_cuda_call():
    cfg = bm.beam_cfg()
    _, need = ws_size(cfg, 64)
    a = 1 << 20  # fake but aligned addresses: never dereferenced on these paths
    assert _fwd(cfg, 0, None, None, None, None, None, None, 0) == OK  # T = 0 is a no-op
    assert _fwd(cfg, 64, a, a, a, a, a, None, need) == INVALID
    assert _fwd(cfg, 64, a, a, a, a, a, a + 8, need) == ALIGN
    assert _fwd(cfg, 64, a, a, a, a, a, a, need - 1) == WS_SMALL
    assert _fwd(cfg, 64, None, a, a, a, a, a, need) == INVALID
    assert _fwd(cfg, 64, a + 2, a, a, a, a, a, need) == ALIGN
    assert _fwd(cfg, 64, a, a, a, a + 4, a, a, need) == ALIGN


def test_route_and_routed_forward_reject_before_any_cuda_call():
    cfg = bm.beam_cfg()
    _, need = ws_size(cfg, 64, bm.OP_ROUTE)
    a = 1 << 20
    L = bm.lib()
    assert L.beam_moe_route(ctypes.byref(cfg), 64, a, a, None, None, a, None, a, need,
                            None) == INVALID
    assert L.beam_moe_route(ctypes.byref(cfg), 64, a, a, None, a, a, a + 4, a, need,
                            None) == ALIGN
    assert L.beam_moe_route(ctypes.byref(cfg), 64, a, a, None, a, a, None, a, need - 1,
                            None) == WS_SMALL
    _, needf = ws_size(cfg, 64)
    assert L.beam_moe_forward_routed(ctypes.byref(cfg), 64, a, None, a, a, a, a, None, a, needf,
                                     None) == INVALID
    assert L.beam_moe_forward_traced(ctypes.byref(cfg), 64, a, a, None, a, a, a, None, None, None,
                                     a, needf, None, None) == INVALID


def test_trace_and_check_argument_errors():
    L = bm.lib()
    h = ctypes.c_void_p()
    assert L.beam_moe_trace_create(0, ctypes.byref(h)) == INVALID
    assert L.beam_moe_trace_destroy(None) == INVALID
    assert L.beam_moe_check(None, 0, None, None) == INVALID


def test_host_forward_workspace_and_argument_checks():
    cfg = bm.beam_cfg()
    H, C = 5120, bm.HOST_CHUNK
    fwd = lambda T: bm.beam_moe_workspace_size(cfg, T, bm.OP_FORWARD)
    host = lambda T, op=bm.OP_FORWARD_HOST: bm.beam_moe_workspace_size(cfg, T, op)
    # one chunk: the forward's workspace plus one staging buffer each way
    assert host(4096) >= fwd(4096) + 2 * 4096 * H * 2
    # from two chunks on: one chunk's workspace plus two staging buffers each way,
    # independent of T and far below the whole batch's forward workspace
    assert host(7 * C) == host(2 * C) >= fwd(C) + 4 * C * H * 2
    assert host(65536) == host(100000) >= fwd(2 * C) + 8 * C * H * 2  # bf16: 2C-token chunks
    assert host(65536) < fwd(65536) // 2
    assert host(65536, bm.OP_FORWARD_NVFP4_HOST) >= 4 * C * H * 2
    L = bm.lib()
    need = host(64)
    a = 1 << 20  # fake but aligned addresses: never dereferenced on these paths
    f = L.beam_moe_forward_host
    assert f(ctypes.byref(cfg), 0, None, None, None, None, None, None, None, 0, None) == OK
    assert f(ctypes.byref(cfg), 64, None, a, None, a, a, a, a, need, None) == INVALID
    assert f(ctypes.byref(cfg), 64, a, a, None, a, a, None, a, need, None) == INVALID
    assert f(ctypes.byref(cfg), 64, a, a, None, a, a, a, a + 8, need, None) == ALIGN
    assert f(ctypes.byref(cfg), 64, a, a, None, a, a, a, a, need - 1, None) == WS_SMALL
    assert f(ctypes.byref(cfg), 64, a, None, None, a, a, a, a, need, None) == INVALID
    odd = bm.beam_cfg(H=320)  # hidden not a multiple of 256
    ex = bm.BeamMoeNvfp4Experts(a, a, a, a, 1.0, 1.0, 1.0, 1.0)
    assert L.beam_moe_forward_nvfp4_host(ctypes.byref(odd), 64, a, a, None, ctypes.byref(ex), a,
                                         a, need, None) == UNSUPPORTED


def test_selftest_argument_checks():
    L = bm.lib()
    a = 1 << 20
    assert L.beam_moe_selftest_wait(None, 256, 20, None) == INVALID
    assert L.beam_moe_selftest_wait(a, 255, 20, None) == INVALID
    assert L.beam_moe_selftest_wait(a, 256, 0, None) == INVALID
    assert L.beam_moe_selftest_wait(a, 256, 1001, None) == INVALID
    assert L.beam_moe_selftest_wait(a + 4, 256, 20, None) == ALIGN


def test_bench_describes_the_host_chunking_the_library_plans():
    """bench.py's e2e line names how the host-buffer call splits a batch. The
    library's host workspace is one forward's workspace (of the larger of a
    full and the last chunk) plus two staging buffers (upload and download)
    per chunk in flight, so its size pins the chunking the description states."""
    import bench

    def up(v):
        return (v + 1023) // 1024 * 1024

    cfg = bm.beam_cfg()
    for T, nvfp4 in [(64, False), (4096, True), (16384, False), (20000, False),
                     (65536, False), (65536, True)]:
        desc = bench.host_chunking(T, nvfp4)
        size = T if desc == "one chunk" else int(desc.split(" of ")[1].split()[0])
        n = -(-T // size)
        if desc != "one chunk":
            assert desc.startswith(f"{n} chunks")
        fwd_op = bm.OP_FORWARD_NVFP4 if nvfp4 else bm.OP_FORWARD
        host_op = bm.OP_FORWARD_NVFP4_HOST if nvfp4 else bm.OP_FORWARD_HOST
        last = T - (n - 1) * size
        fwd = up(max(ws_size(cfg, size, fwd_op)[1], ws_size(cfg, last, fwd_op)[1]))
        bufs = 1 if n == 1 else 2
        assert ws_size(cfg, T, host_op) == (OK, fwd + 2 * bufs * up(size * cfg.hidden * 2))


def test_workspace_layout_rejects_bad_arguments_before_any_cuda_call():
    cfg = bm.beam_cfg()
    lay = bm.BeamMoeWsLayout()
    L = bm.lib()
    assert L.beam_moe_workspace_layout(ctypes.byref(cfg), 64, bm.OP_FORWARD_NVFP4,
                                       ctypes.byref(lay)) == INVALID
    assert L.beam_moe_workspace_layout(ctypes.byref(cfg), 64, bm.OP_FORWARD, None) == INVALID
    assert L.beam_moe_workspace_layout(ctypes.byref(cfg), -1, bm.OP_FORWARD,
                                       ctypes.byref(lay)) == INVALID


def test_forward_stages_rejects_a_bad_stage_before_any_cuda_call():
    cfg = bm.beam_cfg()
    a = 1 << 20  # never dereferenced
    ws_bytes = ws_size(cfg, 64)[1]
    L = bm.lib()
    for stage in (-1, 7):
        assert L.beam_moe_forward_stages(ctypes.byref(cfg), 64, a, a, None, a, a, None, stage,
                                         a, ws_bytes, None) == INVALID
    # the whole forward needs an output
    assert L.beam_moe_forward_stages(ctypes.byref(cfg), 64, a, a, None, a, a, None, 6, a,
                                     ws_bytes, None) == INVALID
