"""Pins of the oracle's NVFP4 arithmetic (4-bit E2M1 values, FP8 E4M3 scale per
16 elements, FP32 tensor scale; the format the "Welcome Beam" post names for
Blackwell in section "Mixture of Experts"): E4M3 against torch's
float8_e4m3fn conversion, E2M1 against brute-force nearest-grid search, the
quantiser's error bounds and exact round trips, the packing order, and the
expert path against numpy matmuls on dequantised values."""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
import synth
from tests import _inputs

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e4m3_matches_torch_float8():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 20000)),
        [2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -6, 0.0155, 1.0, 1.0625, 1.0625 + 1e-6,
         1.1875, 240.0, 247.99, 248.0, 256.0, 447.0, 448.0],
    ]).astype(np.float32)
    ours = oracle.e4m3_value(oracle.e4m3_encode(v))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    # decode table: every finite byte round-trips through torch's decoder
    b = np.arange(0, 0x7F, dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_value(b),
                          torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy())
    assert oracle.e4m3_encode(np.float32(1e6)) == 0x7E  # saturates at 448


def test_e2m1_is_nearest_grid_value_with_ties_to_even():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(-7, 7, 20000),
                        [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.75, -5.0, 6.0, 6.5, 100.0]])
    v = v.astype(np.float32)
    got = oracle.e2m1_value(oracle.e2m1_encode(v))
    a = np.minimum(np.abs(v.astype(np.float64)), 6.0)
    d = np.abs(a[:, None] - GRID[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = np.where(np.isclose(d, best, rtol=0, atol=0), np.arange(8)[None, :], 99)
    even = np.where(cand % 2 == 0, cand, 99).min(axis=1)  # a tie goes to the even code
    code = np.where((cand < 99).sum(axis=1) > 1, even, cand.min(axis=1))
    assert np.array_equal(np.abs(got), GRID[code])
    assert np.all(np.sign(got[got != 0]) == np.sign(v[got != 0]))


def test_quantiser_error_bounds_and_round_trip():
    rng = np.random.default_rng(2)
    g = np.float32(2.0 ** -6)
    v = (rng.standard_normal((64, 256)) * rng.uniform(0.01, 5, (64, 1))).astype(np.float32)
    codes, sf = oracle.nvfp4_quantize(v, g)
    deq = oracle.nvfp4_dequant(codes, sf, float(g))
    s = oracle.e4m3_table()[sf].repeat(16, axis=1) * float(g)
    # every value lands on the nearest point of its block's grid: error <= half a step
    step = np.where(np.abs(v) / s < 2, 0.5, np.where(np.abs(v) / s < 4, 1.0, 2.0)) * s
    assert np.all(np.abs(deq - v) <= step / 2 + 1e-12)
    # the block maximum maps close to 6 (the scale is amax / 6, rounded to E4M3)
    amax = np.abs(v).reshape(64, 16, 16).max(axis=2)
    assert np.all(np.abs(amax / (oracle.e4m3_table()[sf] * float(g)) - 6.0) < 6.0 * 0.07)
    # values already on the grid come back exactly
    codes2, sf2 = oracle.nvfp4_quantize(deq.astype(np.float32), g)
    assert np.array_equal(oracle.nvfp4_dequant(codes2, sf2, float(g)), deq)
    # zero block: zero scale and zero codes
    z = np.zeros((1, 32), np.float32)
    c0, s0 = oracle.nvfp4_quantize(z, g)
    assert not c0.any() and not s0.any()


def test_packing_order_low_nibble_first():
    v = np.zeros((1, 16), np.float32)
    v[0, 0], v[0, 1], v[0, 15] = 6.0, -3.0, 1.0
    codes, sf = oracle.nvfp4_quantize(v, np.float32(1.0))
    assert oracle.e4m3_value(sf)[0, 0] == 1.0
    assert codes[0, 0] == (7 | (0xD << 4)) and codes[0, 7] == (2 << 4)


def test_decoder_reads_the_packing_order():
    """The C decoder the expert path uses reads element 2i from the low nibble
    and 2i+1 from the high one, with the block's scale: it returns the packed
    grid values in order. (A decoder that swapped the nibbles would leave every
    dot product of the expert path unchanged, since it would permute both
    operands alike, so it is pinned here on its own.)"""
    v = np.zeros((1, 32), np.float32)
    v[0, 0], v[0, 1], v[0, 2], v[0, 15] = 6.0, -3.0, 0.5, 1.0
    v[0, 16], v[0, 17] = -3.0, 12.0  # second block: scale 2, values on its grid
    codes, sf = oracle.nvfp4_quantize(v, np.float32(1.0))
    dec = oracle.nvfp4_values(codes[0], sf[0], 1.0)
    assert np.array_equal(dec, v[0].astype(np.float64))
    assert np.array_equal(dec, oracle.nvfp4_dequant(codes, sf, 1.0)[0])


def _swiglu_nvfp4_numpy(x_bits, c13, s13, c2, s2, gw, gx, gh):
    """Numpy float64 matmuls on dequantised values; activations quantised with
    the oracle's (separately pinned) quantiser."""
    xf = synth.bf16_to_f32(x_bits)
    xc, xs = oracle.nvfp4_quantize(xf, np.float32(gx))
    xd = oracle.nvfp4_dequant(xc, xs, gx)
    w13 = oracle.nvfp4_dequant(c13, s13, gw)
    I = w13.shape[0] // 2
    g = xd @ w13[:I].T
    u = xd @ w13[I:].T
    a = (g * expit(g) * u).astype(np.float32)
    ac, as_ = oracle.nvfp4_quantize(a, np.float32(gh))
    return oracle.nvfp4_dequant(ac, as_, gh) @ oracle.nvfp4_dequant(c2, s2, gw).T


def test_nvfp4_identical_experts_closed_form():
    wl = synth.workload("tiny").with_T(24)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    cfg = oracle.cfg_for(wl)
    gw, ga = synth.NVFP4_WEIGHT_SCALE, synth.NVFP4_ACT_SCALE
    c13, s13 = synth.host_expert_w13_nvfp4(wl, 0)
    c2, s2 = synth.host_expert_w2_nvfp4(wl, 0)
    out = oracle.experts_nvfp4(cfg, x, r["ids"], r["weights"], [(c13, s13)] * wl.E,
                               [(c2, s2)] * wl.E, gw, gw, ga, ga)
    f = _swiglu_nvfp4_numpy(x, c13, s13, c2, s2, gw, ga, ga)
    assert np.allclose(out, 2.5 * f, rtol=1e-9, atol=1e-12)


def test_nvfp4_expert_index_and_weights():
    """Distinct experts: out = sum_k w_k f_{e_k}(x), each f from numpy."""
    wl = synth.workload("tiny").with_T(12)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    gw, ga = synth.NVFP4_WEIGHT_SCALE, synth.NVFP4_ACT_SCALE
    w13 = {e: synth.host_expert_w13_nvfp4(wl, e) for e in range(wl.E)}
    w2 = {e: synth.host_expert_w2_nvfp4(wl, e) for e in range(wl.E)}
    out = oracle.experts_nvfp4(oracle.cfg_for(wl), x, r["ids"], r["weights"], w13, w2, gw, gw,
                               ga, ga)
    for t in range(wl.T):
        ref = sum(r["weights"][t, k] * _swiglu_nvfp4_numpy(x[t:t + 1], *w13[int(e)],
                                                            *w2[int(e)], gw, ga, ga)[0]
                  for k, e in enumerate(r["ids"][t]))
        assert np.allclose(out[t], ref, rtol=1e-9, atol=1e-12)


def test_synthetic_nvfp4_weights_resemble_bf16_experts():
    wl = synth.workload("decode")
    c, s = synth.host_expert_w13_nvfp4(wl, 7)
    w = oracle.nvfp4_dequant(c[:64], s[:64], synth.NVFP4_WEIGHT_SCALE)
    assert abs(w.std() - 0.02) < 0.004 and abs(w.mean()) < 1e-3
    assert set(np.unique(s)) <= set(range(0x38, 0x40))
