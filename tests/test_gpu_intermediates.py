"""Intermediates of the CUDA forward against their definitions and the oracle.

"Welcome Beam", section "Mixture of Experts": each token runs through its 8
chosen SwiGLU experts; section "Residual Stream": the SwiGLU product is FP32.
The forward is run stage by stage through the C ABI (beam_moe_forward_stages)
and the workspace is read at the offsets beam_moe_workspace_layout reports:

- counts and offsets equal the bincount and exclusive scan of the routes;
- pos is the stable grouping by expert: the rows of expert e start at
  offsets[e] and hold its tokens in ascending order (the only permutation the
  library documents), so pos is a bijection onto the A = T K rows;
- the permuted rows are x[t] byte for byte at pos[t, k];
- h at pos[t, k] is the oracle's fp64 silu(Wg x) * (Wu x) after one rounding
  to bf16: within half a bf16 step plus the FP32 accumulation slack stated in
  `_h_slack`, and equal to the correctly rounded value on all but a small
  fraction of elements (those whose exact value lies within that slack of a
  rounding midpoint);
- out is the k-ordered FP32 sum of the y rows the workspace holds, bit for
  bit, after either down GEMM (one CTA per tile or CTA pairs).
"""
import numpy as np
import pytest
import torch
from scipy.special import expit

import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu

# Elements of h allowed to differ from the correctly rounded bf16 value of the
# oracle's fp64 value. FP32 accumulation moves a value across a rounding
# midpoint with probability about 2 |delta| / ulp, about 1e-3 here; a SiLU
# evaluated with a 2^-11 relative error (a hardware tanh) flips about 10 %.
MAX_MISROUNDED = 0.01


def _bf16_round(a):
    """Nearest bf16 value of fp64 values, ties to even, and the bf16 spacing there."""
    m, e = np.frexp(a)
    ulp = np.ldexp(1.0, e - 8)
    return np.ldexp(np.round(m * 256.0), e - 8), ulp


def _run_stages(wl, x_bits, last, bias=None):
    cfg = _gpu.cfg_of(wl)
    w13, w2, wr = _gpu.device_weights(wl)
    T = x_bits.shape[0]
    x = _gpu.to_dev_bits(x_bits)
    b = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    bm.beam_moe_forward_stages(cfg, x, wr, b, w13, w2, None, last, ws)
    assert bm.beam_moe_check(ws) == 0
    return ws, bm.beam_moe_workspace_layout(cfg, T)


def _read(ws, off, dtype, shape):
    n = int(np.prod(shape)) * np.dtype(dtype).itemsize
    return ws[off:off + n].cpu().numpy().view(dtype).reshape(shape)


def _expected_pos(ids, E):
    """Row of (t, k) under the stable grouping: offsets[e] + rank of t among
    the tokens routed to e."""
    T, K = ids.shape
    counts = np.bincount(ids.ravel(), minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    flat = ids.ravel()
    order = np.lexsort((np.repeat(np.arange(T), K), flat))  # by expert, then token
    pos = np.empty(T * K, np.int64)
    pos[order] = np.arange(T * K)
    return pos.reshape(T, K), counts, offsets


def _check_dispatch(wl, x, r, ws, lay):
    T, K, E, H = wl.T, wl.K, wl.E, wl.H
    ids = _read(ws, lay.ids, np.int32, (T, K))
    gi, _ = _gpu.sorted_routes(ids, ids.astype(np.float32))
    oi, _ = _gpu.sorted_routes(r["ids"], r["weights"])
    assert np.array_equal(gi, oi)  # same expert sets as the oracle
    want_pos, counts, offsets = _expected_pos(ids, E)
    assert np.array_equal(_read(ws, lay.counts, np.int32, (E,)), counts)
    assert np.array_equal(_read(ws, lay.offsets, np.int32, (E + 1,)), offsets)
    pos = _read(ws, lay.pos, np.int32, (T, K))
    assert np.array_equal(pos, want_pos)
    return ids, pos


def _check_permuted_rows(wl, x, pos, ws, lay):
    xp = _read(ws, lay.xp, np.uint16, (wl.T * wl.K, wl.H))
    for k in range(wl.K):
        assert np.array_equal(xp[pos[:, k]], x), k


def _h_slack(wl, x, ids, tokens, w13):
    """Absolute slack of each h element beyond its bf16 rounding: the FP32
    accumulations of g and u over H exact bf16 products are allowed
    8 * 2^-24 * sum_h |x_h w_h| each (eight FP32 roundings of the whole
    magnitude: several times what the tensor core's per-16 partial sums
    accumulate, far below the worst-case bound H * 2^-24 * sum, which would be
    looser than the rounding under test), carried into h through
    |d h / d g| = |silu'(g) u| and |d h / d u| = |silu(g)|, plus 2^-20 |h|
    for evaluating the sigmoid in FP32."""
    xf = synth.bf16_to_f32(x[tokens]).astype(np.float64)
    I = wl.I
    slack = np.zeros((len(tokens), wl.K, I))
    for e in np.unique(ids[tokens]):
        sel = np.argwhere(ids[tokens] == e)
        w = synth.bf16_to_f32(w13[int(e)]).astype(np.float64)
        xe = xf[sel[:, 0]]
        g, u = xe @ w[:I].T, xe @ w[I:].T
        sg, su = np.abs(xe) @ np.abs(w[:I]).T, np.abs(xe) @ np.abs(w[I:]).T
        sig = expit(g)
        dsilu = sig * (1.0 + g * (1.0 - sig))
        dg, du = 8 * 2.0 ** -24 * sg, 8 * 2.0 ** -24 * su
        h = g * sig * u
        slack[sel[:, 0], sel[:, 1]] = (np.abs(dsilu * u) * dg + np.abs(g * sig) * du
                                       + 2.0 ** -20 * np.abs(h))
    return slack


def _check_h(wl, x, r, ids, pos, ws, lay, tokens):
    h_all = _read(ws, lay.h, np.uint16, (wl.T * wl.K, wl.I))
    a = _gpu.oracle_hidden(wl, x, tokens, r)  # [n, K, I], the oracle's slot order
    w13, _ = _gpu.HOST_EXPERTS.get(wl, r["ids"][tokens])
    slack = _h_slack(wl, x, r["ids"], tokens, w13)
    # the GPU lists a token's experts in its own order: match slots by expert
    rows = np.empty((len(tokens), wl.K), np.int64)
    for i, t in enumerate(tokens):
        for k in range(wl.K):
            rows[i, k] = pos[t, np.nonzero(ids[t] == r["ids"][t, k])[0][0]]
    h = synth.bf16_to_f32(h_all[rows]).astype(np.float64)
    nearest, ulp = _bf16_round(a)
    excess = np.abs(h - a) - 0.5 * ulp - slack
    misrounded = np.mean(h != nearest)
    print(f"{wl.name} T={wl.T}: h elements {h.size}, misrounded {misrounded:.2e}, "
          f"max |h - a| / ulp {np.max(np.abs(h - a) / ulp):.4f}, max excess {excess.max():.3e}")
    assert excess.max() <= 0.0, np.unravel_index(np.argmax(excess), excess.shape)
    assert misrounded <= MAX_MISROUNDED


@pytest.mark.parametrize("T", [300, 1500, 3001])  # 1-CTA tiles; CTA pairs (>= 64 rows per expert)
def test_tiny_intermediates(T):
    wl = synth.workload("tiny").with_T(T)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    ws, lay = _run_stages(wl, x, 3)
    ids, pos = _check_dispatch(wl, x, r, ws, lay)
    _check_permuted_rows(wl, x, pos, ws, lay)
    ws, lay = _run_stages(wl, x, 4)
    assert lay.pair_gateup == (1 if T >= 1500 else 0)
    _check_h(wl, x, r, ids, pos, ws, lay, np.arange(T))


def test_decode_intermediates():
    """Beam's shape at 64 tokens: every permuted row and every h element."""
    wl = synth.workload("decode")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    ws, lay = _run_stages(wl, x, 3)
    ids, pos = _check_dispatch(wl, x, r, ws, lay)
    _check_permuted_rows(wl, x, pos, ws, lay)
    ws, lay = _run_stages(wl, x, 4)
    _check_h(wl, x, r, ids, pos, ws, lay, np.arange(wl.T))


def test_prefill_intermediates():
    """Beam's shape at 4096 tokens (gate/up on CTA pairs): every permuted row;
    h on the tokens covering every expert's first and last token blocks."""
    wl = synth.workload("prefill")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    ws, lay = _run_stages(wl, x, 3)
    ids, pos = _check_dispatch(wl, x, r, ws, lay)
    _check_permuted_rows(wl, x, pos, ws, lay)
    del ws
    ws, lay = _run_stages(wl, x, 4)
    assert lay.pair_gateup == 1
    _check_h(wl, x, r, ids, pos, ws, lay, _gpu.block_cover_tokens(r["ids"], wl.E, 256))


def test_all_stages_equal_the_forward():
    """beam_moe_forward_stages through the combine is beam_moe_forward, bit for bit."""
    wl = synth.workload("tiny").with_T(200)
    x = synth.host_x(wl)
    g = _gpu.forward(wl, x)
    cfg = _gpu.cfg_of(wl)
    w13, w2, wr = _gpu.device_weights(wl)
    out = torch.empty((wl.T, wl.H), dtype=torch.int16, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T), dtype=torch.uint8, device="cuda")
    bm.beam_moe_forward_stages(cfg, _gpu.to_dev_bits(x), wr, None, w13, w2, out, 6, ws)
    assert bm.beam_moe_check(ws) == 0
    assert np.array_equal(_gpu.bits_of(out), g["out"])


@pytest.mark.parametrize("name,T", [("tiny", 200), ("tiny", 1500), ("prefill", None)])
def test_combine_is_the_k_ordered_fp32_sum(name, T):
    """T = 200: y from the one-CTA down GEMM; 1500 and prefill (Beam's shape):
    y from the down GEMM on CTA pairs."""
    wl = synth.workload(name) if T is None else synth.workload(name).with_T(T)
    x = synth.host_x(wl)
    cfg = _gpu.cfg_of(wl)
    w13, w2, wr = _gpu.device_weights(wl)
    out = torch.empty((wl.T, wl.H), dtype=torch.int16, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T), dtype=torch.uint8, device="cuda")
    bm.beam_moe_forward_stages(cfg, _gpu.to_dev_bits(x), wr, None, w13, w2, out, 6, ws)
    assert bm.beam_moe_check(ws) == 0
    lay = bm.beam_moe_workspace_layout(cfg, wl.T)
    assert lay.pair_down == (0 if wl.T == 200 else 1)
    A = wl.T * wl.K
    pos = _read(ws, lay.pos, np.int32, (wl.T, wl.K))
    w = _read(ws, lay.w, np.float32, (wl.T, wl.K))
    y = _read(ws, lay.y, np.float32, (A, wl.H))
    assert np.array_equal(_gpu.bits_of(out), _gpu.combine_bits(y, pos, w))


def test_light_experts_on_one_cta_tiles():
    """With CTA pairs on (225 rows per expert on average), experts with at
    most 64 rows run on the one-CTA kernels after the pair kernels: a
    selection bias on three experts leaves four experts with 43 to 57 rows,
    nine with about 180 to 215 and the three biased ones with over 550 (more
    than their 256 weight rows: token-block-outer order). Every h element
    against the oracle, the combine chain bit for bit, every output row
    against the oracle."""
    import dataclasses
    wl = dataclasses.replace(synth.workload("tiny").with_T(900), n_hot=3, hot_bias=3.0)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    counts = np.bincount(r["ids"].ravel(), minlength=wl.E)
    ws, lay = _run_stages(wl, x, 4, bias=b)
    assert lay.pair_gateup == 1 and lay.light_rows == 64
    assert (counts <= 64).sum() >= 4 and (counts > 256).sum() >= 3
    ids, pos = _check_dispatch(wl, x, r, ws, lay)
    _check_h(wl, x, r, ids, pos, ws, lay, np.arange(wl.T))
    del ws
    cfg = _gpu.cfg_of(wl)
    w13, w2, wrd = _gpu.device_weights(wl)
    out = torch.empty((wl.T, wl.H), dtype=torch.int16, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T), dtype=torch.uint8, device="cuda")
    bd = torch.from_numpy(np.asarray(b, np.float32)).cuda()
    bm.beam_moe_forward_stages(cfg, _gpu.to_dev_bits(x), wrd, bd, w13, w2, out, 6, ws)
    assert bm.beam_moe_check(ws) == 0
    A = wl.T * wl.K
    y = _read(ws, lay.y, np.float32, (A, wl.H))
    w = _read(ws, lay.w, np.float32, (wl.T, wl.K))
    got = _gpu.bits_of(out)
    assert np.array_equal(got, _gpu.combine_bits(y, pos, w))
    ref = _gpu.oracle_outputs(wl, x, np.arange(wl.T), r)
    err, _ = _gpu.max_rel_err(got, ref)
    assert err <= _gpu.TOL
