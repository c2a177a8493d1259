"""Beam MoE block forward on B200 (sm_100a): Python binding of libbeam_moe.so.

Argument marshalling only: every step of the block runs in the library's CUDA
kernels. Functions take torch tensors for device buffers (torch provides
device memory and the current stream) and raise BeamMoeError on any non-OK
status. There is no fallback: if the library is missing, the first call
raises ImportError.

The entry points mirror include/beam_moe.h one to one:
beam_moe_workspace_size, beam_moe_route, beam_moe_forward,
beam_moe_forward_routed, beam_moe_forward_traced, beam_moe_check, and the
Trace wrapper of beam_moe_trace_*.
"""
import ctypes
import os

__all__ = ["BeamMoeCfg", "BeamMoeError", "Trace", "OP_ROUTE", "OP_FORWARD", "N_STAGES",
           "STAGE_NAMES", "lib", "beam_cfg", "beam_moe_workspace_size", "beam_moe_route",
           "beam_moe_route_noalloc", "BeamMoeNvfp4Experts", "OP_FORWARD_NVFP4", "nvfp4_experts",
           "beam_moe_forward_nvfp4", "beam_moe_nvfp4_quantize", "OP_FORWARD_HOST",
           "OP_FORWARD_NVFP4_HOST", "HOST_CHUNK", "beam_moe_forward_host",
           "beam_moe_forward_nvfp4_host", "BeamMoeEpCfg", "ep_cfg", "beam_moe_ep_workspace_size",
           "beam_moe_ep_route", "beam_moe_ep_plan", "beam_moe_ep_dispatch", "beam_moe_ep_experts",
           "beam_moe_ep_combine", "beam_moe_selftest_wait",
           "beam_moe_forward", "beam_moe_forward_routed", "beam_moe_forward_traced",
           "beam_moe_forward_stages", "beam_moe_workspace_layout", "BeamMoeWsLayout",
           "BeamMoeEpHandle", "beam_moe_ep_export", "beam_moe_ep_import",
           "beam_moe_ep_release", "EpPeers", "torch_gather",
           "beam_moe_check"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbeam_moe.so")

OP_ROUTE = 0
OP_FORWARD = 1
OP_FORWARD_NVFP4 = 2
OP_FORWARD_HOST = 3
OP_FORWARD_NVFP4_HOST = 4
HOST_CHUNK = 8192
N_STAGES = 7
STAGE_NAMES = ("router_gemm", "router_topk", "scan", "permute", "gateup_gemm", "down_gemm",
               "combine")


class BeamMoeCfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("bias_mode", ctypes.c_int32),
                ("routed_scale", ctypes.c_float), ("router_tc", ctypes.c_int32)]


class BeamMoeWsLayout(ctypes.Structure):
    """Byte offsets of the intermediates inside a forward workspace."""
    _fields_ = [("counts", ctypes.c_int64), ("offsets", ctypes.c_int64), ("ids", ctypes.c_int64),
                ("w", ctypes.c_int64), ("pos", ctypes.c_int64), ("xp", ctypes.c_int64),
                ("h", ctypes.c_int64), ("y", ctypes.c_int64), ("router_splits", ctypes.c_int32),
                ("router_tc", ctypes.c_int32), ("pair_gateup", ctypes.c_int32),
                ("pair_down", ctypes.c_int32), ("light_rows", ctypes.c_int32)]


class BeamMoeNvfp4Experts(ctypes.Structure):
    """NVFP4 expert weights (device pointers) and tensor scales."""
    _fields_ = [("w13_codes", ctypes.c_void_p), ("w13_scales", ctypes.c_void_p),
                ("w2_codes", ctypes.c_void_p), ("w2_scales", ctypes.c_void_p),
                ("w13_scale", ctypes.c_float), ("w2_scale", ctypes.c_float),
                ("x_scale", ctypes.c_float), ("h_scale", ctypes.c_float)]


class BeamMoeEpCfg(ctypes.Structure):
    """Expert parallelism: ranks, this rank, most tokens per rank, receive rows."""
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("t_max", ctypes.c_int64),
                ("recv_cap", ctypes.c_int64)]


class BeamMoeEpHandle(ctypes.Structure):
    """A workspace exported for other processes (CUDA IPC handle and offset)."""
    _fields_ = [("ipc", ctypes.c_uint8 * 64), ("offset", ctypes.c_int64),
                ("bytes", ctypes.c_int64), ("device", ctypes.c_int32), ("pid", ctypes.c_int32)]


class BeamMoeError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {lib().beam_moe_status_string(status).decode()} ({status})")


_lib = None
_P = ctypes.c_void_p
_CFG = ctypes.POINTER(BeamMoeCfg)
_EP = ctypes.POINTER(BeamMoeEpCfg)
_PP = ctypes.POINTER(ctypes.c_void_p)
_SIGS = {
    "beam_moe_workspace_size": [_CFG, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)],
    "beam_moe_route": [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "beam_moe_route_noalloc": [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P],
    "beam_moe_forward": [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                         ctypes.c_size_t, _P],
    "beam_moe_forward_stages": [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, ctypes.c_int32,
                                _P, ctypes.c_size_t, _P],
    "beam_moe_workspace_layout": [_CFG, ctypes.c_int64, ctypes.c_int,
                                  ctypes.POINTER(BeamMoeWsLayout)],
    "beam_moe_forward_routed": [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P,
                                ctypes.c_size_t, _P],
    "beam_moe_forward_traced": [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                ctypes.c_size_t, _P, _P],
    "beam_moe_forward_nvfp4": [_CFG, ctypes.c_int64, _P, _P, _P,
                               ctypes.POINTER(BeamMoeNvfp4Experts), _P, _P, _P, _P, _P,
                               ctypes.c_size_t, _P],
    "beam_moe_forward_nvfp4_traced": [_CFG, ctypes.c_int64, _P, _P, _P,
                                      ctypes.POINTER(BeamMoeNvfp4Experts), _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P, _P],
    "beam_moe_forward_host": [_CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                              _P],
    "beam_moe_forward_nvfp4_host": [_CFG, ctypes.c_int64, _P, _P, _P,
                                    ctypes.POINTER(BeamMoeNvfp4Experts), _P, _P, ctypes.c_size_t,
                                    _P],
    "beam_moe_nvfp4_quantize": [ctypes.c_int64, ctypes.c_int64, _P, ctypes.c_float, _P, _P, _P],
    "beam_moe_ep_workspace_size": [_CFG, _EP, ctypes.POINTER(ctypes.c_size_t)],
    "beam_moe_ep_route": [_CFG, _EP, ctypes.c_int64, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "beam_moe_ep_plan": [_CFG, _EP, _P, _P, _P, ctypes.POINTER(ctypes.c_int64)],
    "beam_moe_ep_dispatch": [_CFG, _EP, ctypes.c_int64, _P, _P, _PP, _P, ctypes.c_size_t, _P],
    "beam_moe_ep_experts": [_CFG, _EP, _P, _P, _P, _PP, _P, ctypes.c_size_t, _P],
    "beam_moe_ep_combine": [_CFG, _EP, ctypes.c_int64, _P, _P, ctypes.c_size_t, _P],
    "beam_moe_ep_export": [_P, ctypes.c_size_t, ctypes.POINTER(BeamMoeEpHandle)],
    "beam_moe_ep_import": [ctypes.POINTER(BeamMoeEpHandle), ctypes.c_size_t,
                           ctypes.POINTER(ctypes.c_void_p)],
    "beam_moe_ep_release": [ctypes.POINTER(BeamMoeEpHandle), _P],
    "beam_moe_trace_create": [ctypes.c_int32, ctypes.POINTER(_P)],
    "beam_moe_trace_destroy": [_P],
    "beam_moe_trace_reset": [_P],
    "beam_moe_trace_read": [_P, _P, ctypes.POINTER(ctypes.c_int32)],
    "beam_moe_check": [_P, ctypes.c_size_t, _P, ctypes.POINTER(ctypes.c_uint32)],
    "beam_moe_selftest_wait": [_P, ctypes.c_size_t, ctypes.c_int32, _P],
    "beam_moe_status_string": [ctypes.c_int],
}


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libbeam_moe.so not built at {LIB_PATH}; run "
                              "`python -m sparse_moe_layer_beam_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_char_p if name == "beam_moe_status_string" else ctypes.c_int
        _lib = L
    return _lib


def beam_cfg(H=5120, I=2560, E=256, G=8, Gk=4, K=8, renormalize=True, bias_mode=0, scale=2.5,
             router_tc=False):
    """Configuration struct; the defaults are the Beam block. router_tc opts in
    to the router GEMM on tensor cores (exact three-way bf16 split of the FP32
    weights); the default is FP32 FMAs on CUDA cores."""
    return BeamMoeCfg(H, I, E, G, Gk, K, 1 if renormalize else 0, bias_mode, scale,
                      1 if router_tc else 0)


def _check(status, where):
    if status != 0:
        raise BeamMoeError(status, where)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def beam_moe_workspace_size(cfg, T, op=OP_FORWARD):
    n = ctypes.c_size_t(0)
    _check(lib().beam_moe_workspace_size(ctypes.byref(cfg), T, op, ctypes.byref(n)),
           "beam_moe_workspace_size")
    return n.value


def beam_moe_route(cfg, x, w_router, bias, topk_ids, topk_w, expert_counts, ws, stream=None):
    T = x.shape[0] if x is not None else 0
    _check(lib().beam_moe_route(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router), _ptr(bias),
                                _ptr(topk_ids), _ptr(topk_w), _ptr(expert_counts), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "beam_moe_route")


def beam_moe_route_noalloc(cfg, x, w_router, bias, topk_ids, topk_w, expert_counts=None,
                           stream=None):
    """Routing with the library's fixed scratch instead of a workspace, for
    callers that cannot allocate device memory (at most 2048 tokens and 256
    experts; concurrent calls on one device race)."""
    T = x.shape[0]
    _check(lib().beam_moe_route_noalloc(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router),
                                        _ptr(bias), _ptr(topk_ids), _ptr(topk_w),
                                        _ptr(expert_counts), _stream(stream)),
           "beam_moe_route_noalloc")


def beam_moe_forward(cfg, x, w_router, bias, w13, w2, out, ws, topk_ids=None, topk_w=None,
                     expert_counts=None, stream=None):
    T = x.shape[0]
    _check(lib().beam_moe_forward(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router), _ptr(bias),
                                  _ptr(w13), _ptr(w2), _ptr(out), _ptr(topk_ids), _ptr(topk_w),
                                  _ptr(expert_counts), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "beam_moe_forward")


def beam_moe_forward_traced(cfg, x, w_router, bias, w13, w2, out, ws, trace, topk_ids=None,
                            topk_w=None, expert_counts=None, stream=None):
    T = x.shape[0]
    _check(lib().beam_moe_forward_traced(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router),
                                         _ptr(bias), _ptr(w13), _ptr(w2), _ptr(out),
                                         _ptr(topk_ids), _ptr(topk_w), _ptr(expert_counts),
                                         _ptr(ws), ws.numel() * ws.element_size(),
                                         _stream(stream), trace.handle),
           "beam_moe_forward_traced")


def beam_moe_forward_stages(cfg, x, w_router, bias, w13, w2, out, last_stage, ws, stream=None):
    """The forward's stages 0..last_stage (0 router GEMM ... 6 combine), leaving
    the intermediates in ws (see beam_moe_workspace_layout)."""
    T = x.shape[0]
    _check(lib().beam_moe_forward_stages(ctypes.byref(cfg), T, _ptr(x), _ptr(w_router),
                                         _ptr(bias), _ptr(w13), _ptr(w2), _ptr(out), last_stage,
                                         _ptr(ws), ws.numel() * ws.element_size(),
                                         _stream(stream)), "beam_moe_forward_stages")


def beam_moe_workspace_layout(cfg, T, op=OP_FORWARD):
    """BeamMoeWsLayout of a workspace for T tokens on the current device."""
    out = BeamMoeWsLayout()
    _check(lib().beam_moe_workspace_layout(ctypes.byref(cfg), T, op, ctypes.byref(out)),
           "beam_moe_workspace_layout")
    return out


def beam_moe_forward_routed(cfg, x, topk_ids, topk_w, w13, w2, out, ws, expert_counts=None,
                            stream=None):
    T = x.shape[0]
    _check(lib().beam_moe_forward_routed(ctypes.byref(cfg), T, _ptr(x), _ptr(topk_ids),
                                         _ptr(topk_w), _ptr(w13), _ptr(w2), _ptr(out),
                                         _ptr(expert_counts), _ptr(ws),
                                         ws.numel() * ws.element_size(), _stream(stream)),
           "beam_moe_forward_routed")


def nvfp4_experts(w13_codes, w13_scales, w2_codes, w2_scales, w13_scale, w2_scale, x_scale,
                  h_scale):
    return BeamMoeNvfp4Experts(_ptr(w13_codes), _ptr(w13_scales), _ptr(w2_codes),
                               _ptr(w2_scales), w13_scale, w2_scale, x_scale, h_scale)


def beam_moe_forward_host(cfg, x_host, w_router, bias, w13, w2, out_host, ws, stream=None):
    """Forward on host buffers (x_host, out_host: CPU tensors, pinned for overlap)."""
    T = x_host.shape[0]
    _check(lib().beam_moe_forward_host(ctypes.byref(cfg), T, _ptr(x_host), _ptr(w_router),
                                       _ptr(bias), _ptr(w13), _ptr(w2), _ptr(out_host), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)),
           "beam_moe_forward_host")


def beam_moe_forward_nvfp4_host(cfg, x_host, w_router, bias, experts, out_host, ws, stream=None):
    T = x_host.shape[0]
    _check(lib().beam_moe_forward_nvfp4_host(ctypes.byref(cfg), T, _ptr(x_host), _ptr(w_router),
                                             _ptr(bias), ctypes.byref(experts), _ptr(out_host),
                                             _ptr(ws), ws.numel() * ws.element_size(),
                                             _stream(stream)),
           "beam_moe_forward_nvfp4_host")


def beam_moe_forward_nvfp4(cfg, x, w_router, bias, experts, out, ws, topk_ids=None, topk_w=None,
                           expert_counts=None, stream=None, trace=None):
    T = x.shape[0]
    args = (ctypes.byref(cfg), T, _ptr(x), _ptr(w_router), _ptr(bias), ctypes.byref(experts),
            _ptr(out), _ptr(topk_ids), _ptr(topk_w), _ptr(expert_counts), _ptr(ws),
            ws.numel() * ws.element_size(), _stream(stream))
    if trace is None:
        _check(lib().beam_moe_forward_nvfp4(*args), "beam_moe_forward_nvfp4")
    else:
        _check(lib().beam_moe_forward_nvfp4_traced(*args, trace.handle),
               "beam_moe_forward_nvfp4_traced")


def beam_moe_nvfp4_quantize(v, g, codes, scales, stream=None):
    rows, K = v.shape
    _check(lib().beam_moe_nvfp4_quantize(rows, K, _ptr(v), g, _ptr(codes), _ptr(scales),
                                         _stream(stream)), "beam_moe_nvfp4_quantize")


def beam_moe_check(ws, stream=None):
    """Synchronizes the stream, returns the device status bits (0 = clean) and
    clears them. Raises BeamMoeError on a CUDA error."""
    flags = ctypes.c_uint32(0)
    st = lib().beam_moe_check(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream),
                              ctypes.byref(flags))
    if st not in (0, 6):
        raise BeamMoeError(st, "beam_moe_check")
    return flags.value


def beam_moe_selftest_wait(ws, limit_ms, stream=None):
    """Runs the device self-check of a bounded wait that runs out."""
    _check(lib().beam_moe_selftest_wait(_ptr(ws), ws.numel() * ws.element_size(), limit_ms,
                                        _stream(stream)), "beam_moe_selftest_wait")


class Trace:
    """Per-stage CUDA-event timing of traced forward calls."""

    def __init__(self, capacity):
        h = _P()
        _check(lib().beam_moe_trace_create(capacity, ctypes.byref(h)), "beam_moe_trace_create")
        self.handle = h
        self.capacity = capacity

    def reset(self):
        _check(lib().beam_moe_trace_reset(self.handle), "beam_moe_trace_reset")

    def read(self):
        """List (one entry per traced call) of per-stage milliseconds."""
        n = ctypes.c_int32(0)
        buf = (ctypes.c_float * (self.capacity * N_STAGES))()
        _check(lib().beam_moe_trace_read(self.handle, buf, ctypes.byref(n)), "beam_moe_trace_read")
        return [list(buf[i * N_STAGES:(i + 1) * N_STAGES]) for i in range(n.value)]

    def close(self):
        if self.handle:
            lib().beam_moe_trace_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------ expert parallelism

def ep_cfg(world, rank, t_max, recv_cap):
    return BeamMoeEpCfg(world, rank, t_max, recv_cap)


def _addr(v):
    return v if isinstance(v, int) or v is None else v.data_ptr()


def _peers(peer_ws):
    return (ctypes.c_void_p * len(peer_ws))(*[_addr(p) for p in peer_ws])


def beam_moe_ep_workspace_size(cfg, ep):
    n = ctypes.c_size_t(0)
    _check(lib().beam_moe_ep_workspace_size(ctypes.byref(cfg), ctypes.byref(ep), ctypes.byref(n)),
           "beam_moe_ep_workspace_size")
    return n.value


def beam_moe_ep_route(cfg, ep, x, w_router, bias, counts, ws, stream=None):
    _check(lib().beam_moe_ep_route(ctypes.byref(cfg), ctypes.byref(ep), x.shape[0], _ptr(x),
                                   _ptr(w_router), _ptr(bias), _ptr(counts), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)),
           "beam_moe_ep_route")


def beam_moe_ep_plan(cfg, ep, counts_all):
    """counts_all: int32 array [world][E] (host). Returns (send_base [E],
    recv_counts [E/world], recv_rows)."""
    import numpy as np
    counts_all = np.ascontiguousarray(counts_all, dtype=np.int32)
    send_base = np.zeros(cfg.n_experts, dtype=np.int32)
    recv_counts = np.zeros(cfg.n_experts // ep.world, dtype=np.int32)
    rows = ctypes.c_int64(0)
    _check(lib().beam_moe_ep_plan(ctypes.byref(cfg), ctypes.byref(ep), counts_all.ctypes.data,
                                  send_base.ctypes.data, recv_counts.ctypes.data,
                                  ctypes.byref(rows)), "beam_moe_ep_plan")
    return send_base, recv_counts, rows.value


def beam_moe_ep_dispatch(cfg, ep, x, send_base, peer_ws, ws, stream=None):
    _check(lib().beam_moe_ep_dispatch(ctypes.byref(cfg), ctypes.byref(ep), x.shape[0], _ptr(x),
                                      _ptr(send_base), _peers(peer_ws), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)),
           "beam_moe_ep_dispatch")


def beam_moe_ep_experts(cfg, ep, recv_counts, w13, w2, peer_ws, ws, stream=None):
    """recv_counts: int32 array [E/world] (host); w13, w2: this rank's experts
    (tensors or device addresses)."""
    import numpy as np
    rc = np.ascontiguousarray(recv_counts, dtype=np.int32)
    _check(lib().beam_moe_ep_experts(ctypes.byref(cfg), ctypes.byref(ep), rc.ctypes.data,
                                     _addr(w13), _addr(w2), _peers(peer_ws), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)),
           "beam_moe_ep_experts")


def beam_moe_ep_combine(cfg, ep, T, out, ws, stream=None):
    _check(lib().beam_moe_ep_combine(ctypes.byref(cfg), ctypes.byref(ep), T, _ptr(out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)),
           "beam_moe_ep_combine")


def beam_moe_ep_export(ws):
    """This rank's workspace as bytes another process can import."""
    h = BeamMoeEpHandle()
    _check(lib().beam_moe_ep_export(_ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(h)),
           "beam_moe_ep_export")
    return bytes(h)


def beam_moe_ep_import(blob, ws_bytes):
    """Device address of another process's exported workspace."""
    h = BeamMoeEpHandle.from_buffer_copy(blob)
    p = ctypes.c_void_p(0)
    _check(lib().beam_moe_ep_import(ctypes.byref(h), ws_bytes, ctypes.byref(p)),
           "beam_moe_ep_import")
    return p.value


def beam_moe_ep_release(blob, peer_ws):
    h = BeamMoeEpHandle.from_buffer_copy(blob)
    _check(lib().beam_moe_ep_release(ctypes.byref(h), peer_ws), "beam_moe_ep_release")


class EpPeers:
    """Every rank's workspace as an address this process can store to.

    gather(blob) must return the list of every rank's blob in rank order (an
    all-gather, e.g. torch.distributed.all_gather_object); export / import_ /
    release default to the library's CUDA IPC calls. This rank's own slot is
    its local workspace; every other slot is imported, and close() releases
    them (call it on every rank, after a barrier, before any rank frees its
    workspace)."""

    def __init__(self, ep, ws, gather, export=None, import_=None, release=None):
        self._release = release or beam_moe_ep_release
        mine = (export or beam_moe_ep_export)(ws)
        blobs = gather(mine)
        if len(blobs) != ep.world or blobs[ep.rank] != mine:
            raise ValueError("gather must return every rank's blob in rank order")
        nbytes = ws.numel() * ws.element_size()
        self.ptrs, self._opened = [], []
        try:
            for r, blob in enumerate(blobs):
                if r == ep.rank:
                    self.ptrs.append(ws.data_ptr())
                else:
                    p = (import_ or beam_moe_ep_import)(blob, nbytes)
                    self._opened.append((blob, p))
                    self.ptrs.append(p)
        except Exception:
            self.close()
            raise

    def close(self):
        while self._opened:
            blob, p = self._opened.pop()
            self._release(blob, p)


def torch_gather(group=None):
    """An all-gather of Python objects over a torch.distributed group."""
    import torch.distributed as dist

    def gather(obj):
        out = [None] * dist.get_world_size(group)
        dist.all_gather_object(out, obj, group=group)
        return out
    return gather
