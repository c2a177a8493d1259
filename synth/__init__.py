"""Seeded synthetic inputs for the Beam MoE block (no MoE arithmetic here).

The workloads follow the shapes of the Beam MoE block described in the Hugging
Face launch post "Welcome Beam" (section "Mixture of Experts"): hidden 5120,
256 SwiGLU experts of intermediate 2560, 8 groups of 32, top-4 groups, top-8
experts, routed scale 2.5. Value recipes (std, not variance):

* activations bf16 N(0, 1); the clustered workload uses 8 fp32 centres
  N(0, 1) plus N(0, 0.3) noise per row, row t taking centre t mod 8;
* expert weights bf16 N(0, 0.02);
* router weights fp32 N(0, 1/sqrt(H));
* the skewed workload adds +3.0 to the router logits of 16 experts picked by
  the generator; every other workload has no router bias.

Host arrays are numpy; device buffers are filled in place through raw
pointers, with bytes identical to the host arrays for the same arguments.
"""
import ctypes
import dataclasses
import math
import os

import numpy as np

from . import _build

SEED = 0

STREAM_X = 1
STREAM_WROUTER = 2
STREAM_W13 = 3
STREAM_W2 = 4
STREAM_CENTRES = 5
STREAM_BIASPICK = 6
STREAM_SAMPLE = 7


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    G: int
    Gk: int
    K: int
    scale: float = 2.5
    renormalize: bool = True
    sigma_x: float = 1.0
    sigma_w: float = 0.02
    n_hot: int = 0
    hot_bias: float = 0.0
    n_centres: int = 0

    @property
    def sigma_r(self):
        return float(np.float32(1.0 / math.sqrt(self.H)))

    @property
    def has_bias(self):
        return self.n_hot > 0

    @property
    def w13_elems(self):
        return self.E * 2 * self.I * self.H

    @property
    def w2_elems(self):
        return self.E * self.H * self.I

    def with_T(self, T):
        return dataclasses.replace(self, T=T)


def _beam(name, T, **kw):
    return Workload(name=name, T=T, H=5120, I=2560, E=256, G=8, Gk=4, K=8, **kw)


WORKLOADS = {
    "tiny": Workload(name="tiny", T=64, H=256, I=128, E=16, G=4, Gk=2, K=4),
    "decode": _beam("decode", 64),
    "prefill": _beam("prefill", 4096),
    "skewed": _beam("skewed", 16384, n_hot=16, hot_bias=3.0),
    "long": _beam("long", 65536, n_centres=8, sigma_x=0.3),
}


def workload(name):
    return WORKLOADS[name]


_host = None
_cuda = None


def _u64(v):
    return ctypes.c_uint64(v & 0xFFFFFFFFFFFFFFFF)


def host_lib():
    global _host
    if _host is None:
        lib = ctypes.CDLL(_build.build_host())
        lib.synth_stream_key.restype = ctypes.c_uint64
        lib.synth_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_draw_u64.restype = ctypes.c_uint64
        lib.synth_draw_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_host_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                               ctypes.c_uint64, ctypes.c_float, ctypes.c_float]
        lib.synth_host_normal_f32.argtypes = lib.synth_host_normal_bf16.argtypes
        lib.synth_host_x_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32,
                                          ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int64]
        lib.synth_host_nvfp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                         ctypes.c_int64, ctypes.c_int64, ctypes.c_uint64]
        lib.synth_host_pick.restype = ctypes.c_int
        lib.synth_host_pick.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p]
        _host = lib
    return _host


def cuda_lib():
    """Device fill kernels; fails loudly if the library cannot be built or loaded."""
    global _cuda
    if _cuda is None:
        lib = ctypes.CDLL(_build.build_cuda())
        lib.synth_dev_normal_bf16.restype = ctypes.c_int
        lib.synth_dev_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                              ctypes.c_uint64, ctypes.c_float, ctypes.c_float,
                                              ctypes.c_void_p]
        lib.synth_dev_normal_f32.restype = ctypes.c_int
        lib.synth_dev_normal_f32.argtypes = lib.synth_dev_normal_bf16.argtypes
        lib.synth_dev_x.restype = ctypes.c_int
        lib.synth_dev_x.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                    ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32,
                                    ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_dev_nvfp4.restype = ctypes.c_int
        lib.synth_dev_nvfp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p]
        _cuda = lib
    return _cuda


def key(stream, seed=SEED):
    return host_lib().synth_stream_key(_u64(seed), _u64(stream))


# ---------------------------------------------------------------- host side

def host_normal_bf16(n, stream, idx0=0, mu=0.0, sigma=1.0, seed=SEED):
    out = np.empty(n, dtype=np.uint16)
    host_lib().synth_host_normal_bf16(out.ctypes.data, n, _u64(key(stream, seed)), _u64(idx0),
                                      mu, sigma)
    return out


def host_normal_f32(n, stream, idx0=0, mu=0.0, sigma=1.0, seed=SEED):
    out = np.empty(n, dtype=np.float32)
    host_lib().synth_host_normal_f32(out.ctypes.data, n, _u64(key(stream, seed)), _u64(idx0),
                                     mu, sigma)
    return out


def host_x(wl, attempts=None, rows=None, out=None, seed=SEED):
    """Activations, bf16 bits [T, H]. `attempts` (int32 [T]) selects the
    re-draw of each row; `rows` limits the rows written into `out`."""
    if out is None:
        out = np.zeros((wl.T, wl.H), dtype=np.uint16)
    att = None if attempts is None else np.ascontiguousarray(attempts, dtype=np.int32)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    host_lib().synth_host_x_rows(out.ctypes.data, wl.T, wl.H, _u64(key(STREAM_X, seed)),
                                 _u64(key(STREAM_CENTRES, seed)), wl.n_centres, wl.sigma_x,
                                 None if att is None else att.ctypes.data,
                                 None if rr is None else rr.ctypes.data,
                                 0 if rr is None else len(rr))
    return out


def host_router(wl, seed=SEED):
    """Router weights fp32 [E, H]."""
    return host_normal_f32(wl.E * wl.H, STREAM_WROUTER, sigma=wl.sigma_r, seed=seed).reshape(
        wl.E, wl.H)


def pick(stream, n, k, seed=SEED):
    out = np.zeros(max(k, 1), dtype=np.int64)
    rc = host_lib().synth_host_pick(_u64(key(stream, seed)), n, k, out.ctypes.data)
    if rc != 0:
        raise ValueError(f"synth pick failed ({rc}) for n={n} k={k}")
    return out[:k]


def hot_experts(wl, seed=SEED):
    return pick(STREAM_BIASPICK, wl.E, wl.n_hot, seed)


def host_bias(wl, seed=SEED):
    """Per-expert router bias fp32 [E], or None when the workload has none."""
    if not wl.has_bias:
        return None
    b = np.zeros(wl.E, dtype=np.float32)
    b[hot_experts(wl, seed)] = np.float32(wl.hot_bias)
    return b


def sample_tokens(T, n, seed=SEED):
    return pick(STREAM_SAMPLE, T, min(n, T), seed)


def host_expert_w13(wl, e, seed=SEED):
    """Gate/up weights of expert e, bf16 bits [2I, H] (rows 0..I-1 gate)."""
    n = 2 * wl.I * wl.H
    return host_normal_bf16(n, STREAM_W13, idx0=e * n, sigma=wl.sigma_w, seed=seed).reshape(
        2 * wl.I, wl.H)


def host_expert_w2(wl, e, seed=SEED):
    """Down weights of expert e, bf16 bits [H, I]."""
    n = wl.H * wl.I
    return host_normal_bf16(n, STREAM_W2, idx0=e * n, sigma=wl.sigma_w, seed=seed).reshape(
        wl.H, wl.I)


def host_w13(wl, seed=SEED):
    return host_normal_bf16(wl.w13_elems, STREAM_W13, sigma=wl.sigma_w, seed=seed).reshape(
        wl.E, 2 * wl.I, wl.H)


def host_w2(wl, seed=SEED):
    return host_normal_bf16(wl.w2_elems, STREAM_W2, sigma=wl.sigma_w, seed=seed).reshape(
        wl.E, wl.H, wl.I)


# -------------------------------------------------------------- device side

def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"synth device fill {what} failed with CUDA error {rc}")


def dev_normal_bf16(ptr, n, stream_id, stream, idx0=0, mu=0.0, sigma=1.0, seed=SEED):
    _check(cuda_lib().synth_dev_normal_bf16(ptr, n, _u64(key(stream_id, seed)), _u64(idx0), mu,
                                            sigma, stream), "bf16")


def dev_normal_f32(ptr, n, stream_id, stream, idx0=0, mu=0.0, sigma=1.0, seed=SEED):
    _check(cuda_lib().synth_dev_normal_f32(ptr, n, _u64(key(stream_id, seed)), _u64(idx0), mu,
                                           sigma, stream), "f32")


def dev_x(wl, ptr, stream, attempts_ptr=None, seed=SEED):
    _check(cuda_lib().synth_dev_x(ptr, wl.T, wl.H, _u64(key(STREAM_X, seed)),
                                  _u64(key(STREAM_CENTRES, seed)), wl.n_centres, wl.sigma_x,
                                  attempts_ptr, stream), "x")


def dev_router(wl, ptr, stream, seed=SEED):
    dev_normal_f32(ptr, wl.E * wl.H, STREAM_WROUTER, stream, sigma=wl.sigma_r, seed=seed)


def dev_w13(wl, ptr, stream, seed=SEED):
    dev_normal_bf16(ptr, wl.w13_elems, STREAM_W13, stream, sigma=wl.sigma_w, seed=seed)


def dev_w2(wl, ptr, stream, seed=SEED):
    dev_normal_bf16(ptr, wl.w2_elems, STREAM_W2, stream, sigma=wl.sigma_w, seed=seed)


# ------------------------------------------------------------------- NVFP4

# Per-tensor FP32 scales of the synthetic NVFP4 experts (weights) and the
# static activation scales used when the forward quantises x and h.
NVFP4_WEIGHT_SCALE = 2.0 ** -7
NVFP4_ACT_SCALE = 2.0 ** -6


def host_nvfp4_rows(stream, r0, n, K, seed=SEED):
    """(codes uint8 [n, K/2], scales uint8 [n, K/16]) of rows r0 .. r0+n-1."""
    codes = np.empty((n, K // 2), dtype=np.uint8)
    sf = np.empty((n, K // 16), dtype=np.uint8)
    host_lib().synth_host_nvfp4(codes.ctypes.data, sf.ctypes.data, r0, n, K,
                                _u64(key(stream, seed)))
    return codes, sf


def host_expert_w13_nvfp4(wl, e, seed=SEED):
    """NVFP4 gate/up weights of expert e: codes [2I, H/2], scales [2I, H/16]."""
    return host_nvfp4_rows(STREAM_W13, e * 2 * wl.I, 2 * wl.I, wl.H, seed)


def host_expert_w2_nvfp4(wl, e, seed=SEED):
    """NVFP4 down weights of expert e: codes [H, I/2], scales [H, I/16]."""
    return host_nvfp4_rows(STREAM_W2, e * wl.H, wl.H, wl.I, seed)


def dev_nvfp4(stream_id, codes_ptr, sf_ptr, rows, K, stream, seed=SEED):
    """Device NVFP4 matrix [rows][K]: codes and scales in the MMA scale layout."""
    _check(cuda_lib().synth_dev_nvfp4(codes_ptr, sf_ptr, rows, K, _u64(key(stream_id, seed)),
                                      stream), "nvfp4")


def dev_w13_nvfp4(wl, codes_ptr, sf_ptr, stream, seed=SEED):
    dev_nvfp4(STREAM_W13, codes_ptr, sf_ptr, wl.E * 2 * wl.I, wl.H, stream, seed)


def dev_w2_nvfp4(wl, codes_ptr, sf_ptr, stream, seed=SEED):
    dev_nvfp4(STREAM_W2, codes_ptr, sf_ptr, wl.E * wl.H, wl.I, stream, seed)


def sf_offset(r, b, K):
    """Byte offset of (row, 16-block) in the block-scaled MMA scale layout."""
    r = np.asarray(r, dtype=np.int64)
    b = np.asarray(b, dtype=np.int64)
    rr = r % 128
    return ((r // 128) * (K // 64) + b // 4) * 512 + (rr % 32) * 16 + (rr // 32) * 4 + (b % 4)


def bf16_to_f32(bits):
    """bf16 bits (uint16 array) -> float32 array, exact."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
