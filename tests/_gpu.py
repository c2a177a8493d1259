"""GPU-side helpers for parity tests and the smoke check: device buffers filled
by the synthetic generator, a forward call through the C ABI, and the oracle
comparison on sampled tokens. Expected values come only from oracle/."""
import collections
import concurrent.futures
import os

import numpy as np
import psutil
import torch

import oracle
import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _inputs

TOL = 2e-2  # max |err| <= TOL * RMS(oracle output): bf16 weights/activations, fp32 accumulation

_weights = {}


def cfg_of(wl, renormalize=None, bias_mode=0):
    return bm.beam_cfg(wl.H, wl.I, wl.E, wl.G, wl.Gk, wl.K,
                       wl.renormalize if renormalize is None else renormalize, bias_mode, wl.scale)


def stream():
    return torch.cuda.current_stream().cuda_stream


def device_weights(wl):
    """(w13, w2, w_router) on the device, filled on the GPU with the host
    generator's bytes; cached per block shape (all Beam workloads share them)."""
    key = (wl.H, wl.I, wl.E)
    if key not in _weights:
        _weights.clear()
        torch.cuda.empty_cache()
        w13 = torch.empty(wl.w13_elems, dtype=torch.int16, device="cuda")
        w2 = torch.empty(wl.w2_elems, dtype=torch.int16, device="cuda")
        synth.dev_w13(wl, w13.data_ptr(), stream())
        synth.dev_w2(wl, w2.data_ptr(), stream())
        wr = torch.from_numpy(synth.host_router(wl)).cuda()
        torch.cuda.synchronize()
        _weights[key] = (w13, w2, wr)
    return _weights[key]


_weights4 = {}


def device_weights_nvfp4(wl):
    """NVFP4 experts on the device (codes, scales in the MMA layout) and the
    router, cached per block shape."""
    key = (wl.H, wl.I, wl.E)
    if key not in _weights4:
        _weights4.clear()
        torch.cuda.empty_cache()
        c13 = torch.empty(wl.E * 2 * wl.I * wl.H // 2, dtype=torch.uint8, device="cuda")
        s13 = torch.empty(wl.E * 2 * wl.I * wl.H // 16, dtype=torch.uint8, device="cuda")
        c2 = torch.empty(wl.E * wl.H * wl.I // 2, dtype=torch.uint8, device="cuda")
        s2 = torch.empty(wl.E * wl.H * wl.I // 16, dtype=torch.uint8, device="cuda")
        synth.dev_w13_nvfp4(wl, c13.data_ptr(), s13.data_ptr(), stream())
        synth.dev_w2_nvfp4(wl, c2.data_ptr(), s2.data_ptr(), stream())
        wr = torch.from_numpy(synth.host_router(wl)).cuda()
        torch.cuda.synchronize()
        _weights4[key] = (c13, s13, c2, s2, wr)
    return _weights4[key]


def nvfp4_experts(c13, s13, c2, s2):
    g_w, g_a = synth.NVFP4_WEIGHT_SCALE, synth.NVFP4_ACT_SCALE
    return bm.nvfp4_experts(c13, s13, c2, s2, g_w, g_w, g_a, g_a)


def forward_nvfp4(wl, x_bits, bias=None):
    cfg = cfg_of(wl)
    c13, s13, c2, s2, wr = device_weights_nvfp4(wl)
    T = x_bits.shape[0]
    x = to_dev_bits(x_bits)
    b = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    out = torch.empty((T, wl.H), dtype=torch.int16, device="cuda")
    ids = torch.empty((T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.K), dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, T, bm.OP_FORWARD_NVFP4), dtype=torch.uint8,
                     device="cuda")
    bm.beam_moe_forward_nvfp4(cfg, x, wr, b, nvfp4_experts(c13, s13, c2, s2), out, ws, ids, w,
                              counts)
    flags = bm.beam_moe_check(ws)
    return {"out": bits_of(out), "ids": ids.cpu().numpy(), "w": w.cpu().numpy(),
            "counts": counts.cpu().numpy(), "flags": flags}


class HostExperts:
    """Host copies of expert weights from the host generator, generated on a
    thread pool (the generator's C calls release the GIL) and kept, least
    recently used first out, within a byte budget of half the free memory."""

    def __init__(self):
        self.cache = collections.OrderedDict()  # (kind, H, I, E, e) -> (w13, w2)
        self.bytes = 0

    @staticmethod
    def _make(kind, wl, e):
        if kind == "bf16":
            return synth.host_expert_w13(wl, e), synth.host_expert_w2(wl, e)
        return synth.host_expert_w13_nvfp4(wl, e), synth.host_expert_w2_nvfp4(wl, e)

    @staticmethod
    def _nbytes(v):
        return sum(a.nbytes for part in v for a in (part if isinstance(part, tuple) else (part,)))

    def get(self, wl, experts, kind="bf16"):
        """({e: w13}, {e: w2}) for the listed experts."""
        want = sorted(set(int(e) for e in np.ravel(experts)))
        keys = {e: (kind, wl.H, wl.I, wl.E, e) for e in want}
        missing = [e for e in want if keys[e] not in self.cache]
        if missing:
            workers = max(1, min(16, os.cpu_count() or 1))
            with concurrent.futures.ThreadPoolExecutor(workers) as pool:
                made = list(pool.map(lambda e: self._make(kind, wl, e), missing))
            for e, v in zip(missing, made):
                self.cache[keys[e]] = v
                self.bytes += self._nbytes(v)
        for e in want:
            self.cache.move_to_end(keys[e])
        budget = psutil.virtual_memory().available // 2 + self.bytes
        wanted = set(keys.values())
        while self.bytes > budget:
            k = next((k for k in self.cache if k not in wanted), None)
            if k is None:
                break
            self.bytes -= self._nbytes(self.cache.pop(k))
        w13 = {e: self.cache[keys[e]][0] for e in want}
        w2 = {e: self.cache[keys[e]][1] for e in want}
        return w13, w2


HOST_EXPERTS = HostExperts()


def _batches(tokens, ids, batch):
    """Token batches in the order of their first expert, so that consecutive
    batches share experts (fewer host weights generated per batch)."""
    tokens = np.asarray(tokens)
    order = tokens[np.argsort(ids[tokens, 0], kind="stable")]
    for i in range(0, len(order), batch):
        yield order[i:i + batch]


def oracle_outputs_nvfp4(wl, x_bits, tokens, r_oracle, batch=64):
    """Oracle output rows (NVFP4 expert path) for the listed tokens, in that order."""
    cfg = oracle.cfg_for(wl)
    g_w, g_a = synth.NVFP4_WEIGHT_SCALE, synth.NVFP4_ACT_SCALE
    out = {}
    for tt in _batches(tokens, r_oracle["ids"], batch):
        ids = r_oracle["ids"][tt]
        w13, w2 = HOST_EXPERTS.get(wl, ids, "nvfp4")
        rows = oracle.experts_nvfp4(cfg, x_bits[tt], ids, r_oracle["weights"][tt], w13, w2,
                                    g_w, g_w, g_a, g_a)
        out.update(zip(tt.tolist(), rows))
    return np.stack([out[int(t)] for t in tokens])


def block_cover_tokens(ids, E, block, extra=0, seed=synth.SEED):
    """Tokens whose rows cover, for every expert with rows, the first and last
    rows of its first and last token blocks (rows of an expert are its tokens
    in ascending order, cut into blocks of `block`), plus the first row of the
    second half of its first block (where the second CTA of a pair starts);
    then `extra` more tokens drawn at random. Sorted, without repeats."""
    T, K = ids.shape
    flat_e = ids.ravel()
    flat_t = np.repeat(np.arange(T), K)
    order = np.lexsort((flat_t, flat_e))
    e_sorted, t_sorted = flat_e[order], flat_t[order]
    starts = np.searchsorted(e_sorted, np.arange(E + 1))
    pick = set()
    for e in range(E):
        c = starts[e + 1] - starts[e]
        if c == 0:
            continue
        nb = (c + block - 1) // block
        first_end = min(c, block)
        for r in (0, first_end - 1, first_end // 2, (nb - 1) * block, c - 1):
            pick.add(int(t_sorted[starts[e] + r]))
    rng = np.random.default_rng(seed + 17)
    rest = np.setdiff1d(np.arange(T), np.fromiter(pick, int, len(pick)))
    if extra and rest.size:
        pick.update(rng.choice(rest, size=min(extra, rest.size), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def to_dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def bits_of(t):
    return t.cpu().numpy().view(np.uint16)


def forward(wl, x_bits, bias=None, renormalize=None, bias_mode=0, weights=None):
    """Runs beam_moe_forward; returns dict of host arrays and the device flags."""
    cfg = cfg_of(wl, renormalize, bias_mode)
    w13, w2, wr = weights if weights is not None else device_weights(wl)
    T = x_bits.shape[0]
    x = to_dev_bits(x_bits)
    b = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    out = torch.empty((T, wl.H), dtype=torch.int16, device="cuda")
    ids = torch.empty((T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.K), dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(bm.beam_moe_workspace_size(cfg, T), 256), dtype=torch.uint8,
                     device="cuda")
    bm.beam_moe_forward(cfg, x, wr, b, w13, w2, out, ws, ids, w, counts)
    flags = bm.beam_moe_check(ws)
    return {"out": bits_of(out), "ids": ids.cpu().numpy(), "w": w.cpu().numpy(),
            "counts": counts.cpu().numpy(), "flags": flags}


def sorted_routes(ids, w):
    order = np.argsort(ids, axis=1, kind="stable")
    return np.take_along_axis(ids, order, 1), np.take_along_axis(w, order, 1)


def check_routes(r_gpu, r_oracle, E):
    """Bit-exact expert sets per token and counts; weights to 1e-5 relative: the
    fp32 router logit is a sequential sum over H = 5120 products, whose rounding
    error reaches a few 1e-6, times the sigmoid slope (<= 1/4), relative to
    weights of about 0.3."""
    gi, gw = sorted_routes(r_gpu["ids"], r_gpu["w"])
    oi, ow = sorted_routes(r_oracle["ids"], r_oracle["weights"])
    assert np.array_equal(gi, oi), np.nonzero(np.any(gi != oi, axis=1))[0][:10]
    assert np.array_equal(r_gpu["counts"], np.bincount(oi.ravel(), minlength=E))
    assert np.allclose(gw, ow, rtol=1e-5, atol=1e-6)


def oracle_outputs(wl, x_bits, tokens, r_oracle, batch=64):
    """Oracle output rows for the listed tokens, in that order, generating only
    their experts on the host."""
    cfg = oracle.cfg_for(wl)
    out = {}
    for tt in _batches(tokens, r_oracle["ids"], batch):
        ids = r_oracle["ids"][tt]
        w13, w2 = HOST_EXPERTS.get(wl, ids)
        rows = oracle.experts(cfg, x_bits[tt], ids, r_oracle["weights"][tt], w13, w2)
        out.update(zip(tt.tolist(), rows))
    return np.stack([out[int(t)] for t in tokens])


def oracle_hidden(wl, x_bits, tokens, r_oracle):
    """The oracle's silu(Wg x) * (Wu x) [len(tokens), K, I] for the listed tokens."""
    cfg = oracle.cfg_for(wl)
    ids = r_oracle["ids"][np.asarray(tokens)]
    w13, _ = HOST_EXPERTS.get(wl, ids)
    return oracle.hidden(cfg, x_bits[np.asarray(tokens)], ids, w13)


# NVFP4 outputs. The block's tolerance of 2e-2 x RMS is stated for BF16 weights
# and activations; for NVFP4 it is derived from the arithmetic:
# - each element may differ by half a bf16 step of the output (its one
#   rounding; NVFP4 outputs have heavier tails, RMS about 1.75 and elements up
#   to about 20 at Beam's shapes, where half a step reaches 1/16) plus
#   TOL_NVFP4_ELEM x RMS: where the GPU's FP32 sums and the oracle's fp64 sums
#   put an element of h on either side of an E2M1 decision boundary, its code
#   differs by one step (up to twice the block scale, about amax / 3), which
#   moves out[j] by w_k W2[j, i] times that: up to about 0.035 = 0.02 x RMS at
#   Beam's shapes (w_k about 0.3, |W2| <= 0.088 for the synthetic experts,
#   block amax about 4), a few times per thousand rows;
# - the RMS of the error over all compared elements may exceed that of the
#   output's own bf16 rounding by at most TOL_NVFP4_RMS x RMS, which isolated
#   flips cannot reach but any systematic error (a scale, a code table, a
#   dropped term) would.
TOL_NVFP4_ELEM = 3e-2
TOL_NVFP4_RMS = 1e-3


def nvfp4_errors(out_bits, ref):
    """(max over elements of (|err| - half a bf16 step at the output) / RMS,
    (RMS of the error - RMS of rounding ref to bf16) / RMS, RMS)."""
    got = synth.bf16_to_f32(out_bits).astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    _, e = np.frexp(np.maximum(np.abs(ref), np.abs(got)))
    half_step = np.ldexp(1.0, e - 9)  # bf16 keeps 8 significant bits
    excess = ((np.abs(got - ref) - half_step) / rms).max()
    m, ex = np.frexp(ref)
    rounded = np.ldexp(np.round(m * 256.0), ex - 8)  # ref to bf16, ties to even
    rms_err = np.sqrt(np.mean((got - ref) ** 2))
    rms_round = np.sqrt(np.mean((rounded - ref) ** 2))
    return excess, (rms_err - rms_round) / rms, rms


def check_nvfp4(out_bits, ref):
    excess, rms_excess, rms = nvfp4_errors(out_bits, ref)
    assert excess <= TOL_NVFP4_ELEM, (excess, rms)
    assert rms_excess <= TOL_NVFP4_RMS, (rms_excess, rms)


def combine_bits(y, pos, w):
    """bf16 bits of out[t] = sum_k w[t, k] y[pos[t, k]]: a chain of FP32 fused
    multiply-adds in ascending k (pos < 0 skipped) from 0, rounded once to
    bf16 (nearest, ties to even). Each step forms the exact product plus the
    running sum in extended precision and rounds it to FP32 once."""
    T, K = pos.shape
    acc = np.zeros((T, y.shape[1]), np.float32)
    for k in range(K):
        p = pos[:, k]
        ok = p >= 0
        prod = w[ok, k].astype(np.longdouble)[:, None] * y[p[ok]].astype(np.longdouble)
        acc[ok] = (prod + acc[ok].astype(np.longdouble)).astype(np.float32)
    u = acc.view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def max_rel_err(out_bits, ref):
    got = synth.bf16_to_f32(out_bits).astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    return np.abs(got - ref).max() / rms, rms
