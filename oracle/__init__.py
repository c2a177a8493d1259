"""fp64 CPU oracle of the Beam MoE block forward (ctypes binding).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product package. The arithmetic
lives in beam_moe_oracle.c; this file only marshals numpy arrays.
"""
import ctypes
import os

import numpy as np

from . import _build


class OracleCfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("bias_mode", ctypes.c_int32),
                ("routed_scale", ctypes.c_double)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        P = ctypes.c_void_p
        L.oracle_route.restype = ctypes.c_int
        L.oracle_route.argtypes = [ctypes.POINTER(OracleCfg), ctypes.c_int64, P, P, P, P, P, P,
                                   P, P, P]
        L.oracle_swiglu_expert.restype = ctypes.c_int
        L.oracle_swiglu_expert.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, P, P]
        L.oracle_experts.restype = ctypes.c_int
        L.oracle_experts.argtypes = [ctypes.POINTER(OracleCfg), ctypes.c_int64, P, P, P, P, P, P]
        L.oracle_hidden.restype = ctypes.c_int
        L.oracle_hidden.argtypes = [ctypes.POINTER(OracleCfg), ctypes.c_int64, P, P, P, P]
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_nvfp4_quantize.restype = ctypes.c_int
        L.oracle_nvfp4_quantize.argtypes = [P, ctypes.c_int64, ctypes.c_float, P, P]
        L.oracle_nvfp4_value.restype = ctypes.c_double
        L.oracle_nvfp4_value.argtypes = [P, P, ctypes.c_int64, ctypes.c_double]
        L.oracle_experts_nvfp4.restype = ctypes.c_int
        L.oracle_experts_nvfp4.argtypes = [ctypes.POINTER(OracleCfg), ctypes.c_int64, P, P, P, P,
                                           P, P, P, ctypes.c_double, ctypes.c_double,
                                           ctypes.c_float, ctypes.c_float, P]
        _lib = L
    return _lib


def cfg_of(H, I, E, G, Gk, K, renormalize=True, scale=2.5, bias_mode=0):
    return OracleCfg(H, I, E, G, Gk, K, 1 if renormalize else 0, bias_mode, scale)


def cfg_for(wl, bias_mode=0, renormalize=None):
    return cfg_of(wl.H, wl.I, wl.E, wl.G, wl.Gk, wl.K,
                  wl.renormalize if renormalize is None else renormalize, wl.scale, bias_mode)


def _ptr(a):
    return None if a is None else a.ctypes.data


def route(cfg, x_bits, w_router, bias=None, want_all_s=False):
    """Route every row of x (bf16 bits [T, H]). Returns a dict of numpy arrays:
    ids [T,K] int32, weights [T,K], scores [T,K], kept [T,Gk] int32,
    margins [T,2] and, if asked, all_s [T,E]."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    wr = np.ascontiguousarray(w_router, dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    T = x.shape[0]
    K, Gk, E = cfg.top_k, cfg.topk_group, cfg.n_experts
    assert x.shape[1] == cfg.hidden and wr.shape == (E, cfg.hidden)
    r = {"ids": np.zeros((T, K), np.int32), "weights": np.zeros((T, K)),
         "scores": np.zeros((T, K)), "kept": np.zeros((T, Gk), np.int32),
         "margins": np.zeros((T, 2))}
    all_s = np.zeros((T, E)) if want_all_s else None
    rc = lib().oracle_route(ctypes.byref(cfg), T, _ptr(x), _ptr(wr), _ptr(b), _ptr(r["ids"]),
                            _ptr(r["weights"]), _ptr(r["scores"]), _ptr(r["kept"]),
                            _ptr(r["margins"]), _ptr(all_s))
    if rc != 0:
        raise ValueError(f"oracle_route failed ({rc})")
    if want_all_s:
        r["all_s"] = all_s
    return r


def swiglu_expert(x, w13_bits, w2_bits):
    """One SwiGLU expert on one fp64 token vector."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    w13 = np.ascontiguousarray(w13_bits, dtype=np.uint16)
    w2 = np.ascontiguousarray(w2_bits, dtype=np.uint16)
    H = x.shape[0]
    I = w13.shape[0] // 2
    assert w13.shape == (2 * I, H) and w2.shape == (H, I)
    y = np.zeros(H)
    rc = lib().oracle_swiglu_expert(H, I, _ptr(x), _ptr(w13), _ptr(w2), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_swiglu_expert failed ({rc})")
    return y


def experts(cfg, x_bits, ids, weights, w13_of, w2_of):
    """out [T, H] fp64 for routed tokens. w13_of / w2_of map an expert id to
    its bf16-bit weight array (a dict, a list, or a stacked array)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(weights, dtype=np.float64)
    T = x.shape[0]
    E = cfg.n_experts
    keep = []
    p13 = (ctypes.c_void_p * E)()
    p2 = (ctypes.c_void_p * E)()
    for e in np.unique(ids):
        a = np.ascontiguousarray(w13_of[int(e)], dtype=np.uint16)
        b = np.ascontiguousarray(w2_of[int(e)], dtype=np.uint16)
        assert a.shape == (2 * cfg.inter, cfg.hidden) and b.shape == (cfg.hidden, cfg.inter)
        keep += [a, b]
        p13[int(e)] = a.ctypes.data
        p2[int(e)] = b.ctypes.data
    out = np.zeros((T, cfg.hidden))
    rc = lib().oracle_experts(ctypes.byref(cfg), T, _ptr(x), _ptr(ids), _ptr(w), p13, p2,
                              _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_experts failed ({rc})")
    return out


def hidden(cfg, x_bits, ids, w13_of):
    """a [T, K, I] fp64: silu(Wg x_t) * (Wu x_t) of every routed (token, expert)
    pair, the gate/up step's output before the down projection."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T = x.shape[0]
    E = cfg.n_experts
    keep = []
    p13 = (ctypes.c_void_p * E)()
    for e in np.unique(ids):
        a = np.ascontiguousarray(w13_of[int(e)], dtype=np.uint16)
        assert a.shape == (2 * cfg.inter, cfg.hidden)
        keep.append(a)
        p13[int(e)] = a.ctypes.data
    out = np.zeros((T, cfg.top_k, cfg.inter))
    rc = lib().oracle_hidden(ctypes.byref(cfg), T, _ptr(x), _ptr(ids), p13, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_hidden failed ({rc})")
    return out


def forward(cfg, x_bits, w_router, bias, w13_of, w2_of):
    """Route, then run the experts: returns (route dict, out [T, H] fp64)."""
    r = route(cfg, x_bits, w_router, bias)
    return r, experts(cfg, x_bits, r["ids"], r["weights"], w13_of, w2_of)


# ------------------------------------------------------------------- NVFP4

def e4m3_encode(values):
    return np.array([lib().oracle_e4m3_encode(float(v)) for v in np.ravel(values)],
                    dtype=np.uint8).reshape(np.shape(values))


def e4m3_value(bytes_):
    return np.array([lib().oracle_e4m3_value(int(b)) for b in np.ravel(bytes_)]).reshape(
        np.shape(bytes_))


def e2m1_encode(values):
    return np.array([lib().oracle_e2m1_encode(float(v)) for v in np.ravel(values)],
                    dtype=np.uint8).reshape(np.shape(values))


def e2m1_value(codes):
    return np.array([lib().oracle_e2m1_value(int(c)) for c in np.ravel(codes)]).reshape(
        np.shape(codes))


def nvfp4_quantize(values, g):
    """Rows of fp32 values [R, K] -> (codes uint8 [R, K/2], scales uint8 [R, K/16])."""
    v = np.ascontiguousarray(np.atleast_2d(values), dtype=np.float32)
    R, K = v.shape
    codes = np.zeros((R, K // 2), np.uint8)
    sf = np.zeros((R, K // 16), np.uint8)
    for r in range(R):
        rc = lib().oracle_nvfp4_quantize(v[r].ctypes.data, K, g, codes[r].ctypes.data,
                                         sf[r].ctypes.data)
        if rc != 0:
            raise ValueError(f"oracle_nvfp4_quantize failed ({rc})")
    return codes, sf


def nvfp4_values(codes, sf, g):
    """One row (codes [K/2], scales [K/16]) -> fp64 values [K] through the C
    decoder the expert path uses (element by element)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    return np.array([lib().oracle_nvfp4_value(codes.ctypes.data, sf.ctypes.data, i, g)
                     for i in range(2 * codes.size)])


_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def nvfp4_dequant(codes, sf, g):
    """(codes [R, K/2], scales [R, K/16]) -> fp64 values [R, K] (table lookups only)."""
    codes = np.atleast_2d(codes)
    sf = np.atleast_2d(sf)
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[0], -1)
    v = _E2M1[nib & 7] * np.where(nib & 8, -1.0, 1.0)
    s = e4m3_table()[sf]
    return v * np.repeat(s, 16, axis=1) * g


_E4M3 = None


def e4m3_table():
    global _E4M3
    if _E4M3 is None:
        _E4M3 = np.array([lib().oracle_e4m3_value(b) for b in range(256)])
    return _E4M3


def experts_nvfp4(cfg, x_bits, ids, weights, w13_of, w2_of, g_w13, g_w2, g_x, g_h):
    """out [T, H] fp64 of the NVFP4 expert path; w13_of / w2_of map an expert id
    to its (codes, scales) pair with row-major scales."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(weights, dtype=np.float64)
    T = x.shape[0]
    E = cfg.n_experts
    keep = []
    P4 = [(ctypes.c_void_p * E)() for _ in range(4)]
    for e in np.unique(ids):
        arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (*w13_of[int(e)], *w2_of[int(e)])]
        keep += arrs
        for j in range(4):
            P4[j][int(e)] = arrs[j].ctypes.data
    out = np.zeros((T, cfg.hidden))
    rc = lib().oracle_experts_nvfp4(ctypes.byref(cfg), T, _ptr(x), _ptr(ids), _ptr(w), P4[0], P4[1],
                                    P4[2], P4[3], g_w13, g_w2, g_x, g_h, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_experts_nvfp4 failed ({rc})")
    return out
