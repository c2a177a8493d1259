"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Routing must match bit-exactly: the same expert set for every token and the
same per-expert counts (inputs are re-drawn until every oracle top-k margin
exceeds 1e-4, so fp32 and fp64 routing must agree). Outputs must match within
max |err| <= 2e-2 x RMS of the oracle output (bf16 weights and activations,
fp32 accumulation, bf16 h, fp32 y, bf16 out). Full-size workloads are compared on all
routes and on output rows that cover every touched expert's first and last token
blocks (decode: every row).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu


def _full_case(name, tokens=None, min_rows=0):
    """Routing on every token; outputs on `tokens`, by default the tokens that
    cover the first and last rows of every touched expert's first and last
    256-row token block (the grouped GEMMs' token tiles, in both tile orders),
    topped up at random to at least `min_rows` rows."""
    wl = synth.workload(name)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x, bias=b)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    if tokens is None:
        tokens = _gpu.block_cover_tokens(r["ids"], wl.E, 256)
        if len(tokens) < min_rows:
            tokens = _gpu.block_cover_tokens(r["ids"], wl.E, 256, extra=min_rows - len(tokens))
    ref = _gpu.oracle_outputs(wl, x, tokens, r)
    err, rms = _gpu.max_rel_err(g["out"][tokens], ref)
    assert err <= _gpu.TOL, (name, err, rms)
    return wl, x, r, g, tokens


def test_device_generator_matches_host():
    wl = synth.workload("decode")
    n = 1 << 20
    d = torch.empty(n, dtype=torch.int16, device="cuda")
    synth.dev_normal_bf16(d.data_ptr(), n, synth.STREAM_W13, _gpu.stream(), idx0=7 * n,
                          sigma=wl.sigma_w)
    host = synth.host_normal_bf16(n, synth.STREAM_W13, idx0=7 * n, sigma=wl.sigma_w)
    assert np.array_equal(_gpu.bits_of(d), host)
    f = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.dev_normal_f32(f.data_ptr(), n, synth.STREAM_WROUTER, _gpu.stream(), sigma=wl.sigma_r)
    assert np.array_equal(f.cpu().numpy(), synth.host_normal_f32(n, synth.STREAM_WROUTER,
                                                                   sigma=wl.sigma_r))
    lg = synth.workload("long").with_T(40)
    xd = torch.empty((40, lg.H), dtype=torch.int16, device="cuda")
    att = torch.arange(40, dtype=torch.int32, device="cuda") % 3
    synth.dev_x(lg, xd.data_ptr(), _gpu.stream(), att.data_ptr())
    assert np.array_equal(_gpu.bits_of(xd), synth.host_x(lg, att.cpu().numpy()))


def test_tiny_forward_matches_oracle_everywhere():
    wl = synth.workload("tiny")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    cfg = oracle.cfg_for(wl)
    ref = oracle.experts(cfg, x, r["ids"], r["weights"], synth.host_w13(wl), synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(g["out"], ref)
    assert err <= _gpu.TOL, err


@pytest.mark.parametrize("T", [1, 7, 129, 300])
def test_tiny_ragged_token_counts(T):
    """Ragged T: partial chunks (128 tokens), partial router tiles (64), single token."""
    wl = synth.workload("tiny").with_T(T)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    ref = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], synth.host_w13(wl),
                         synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(g["out"], ref)
    assert err <= _gpu.TOL, err


@pytest.mark.parametrize("T", [600, 1024, 1500, 2100, 3001])
def test_tiny_many_rows_per_expert(T):
    """More than 100 rows per expert on average: the grouped GEMMs run on CTA
    pairs (cta_group::2) with ragged token blocks, each CTA loading its half
    of a block's rows as a box of 64 or 128 rows; at T = 2100 and 3001
    experts have more rows than weight rows and run token block by token
    block."""
    wl = synth.workload("tiny").with_T(T)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    ref = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], synth.host_w13(wl),
                         synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(g["out"], ref)
    assert err <= _gpu.TOL, err


def test_tie_case_is_bit_exact():
    """Zero router weights: every score is exactly 0.5; groups 0..Gk-1 and
    experts 0..K-1 are chosen, each with weight S/K."""
    for name in ("tiny", "decode"):
        wl = synth.workload(name).with_T(70)
        w13, w2, _ = _gpu.device_weights(wl)
        wr0 = torch.zeros((wl.E, wl.H), dtype=torch.float32, device="cuda")
        g = _gpu.forward(wl, synth.host_x(wl), weights=(w13, w2, wr0))
        assert np.array_equal(g["ids"], np.tile(np.arange(wl.K), (wl.T, 1)))
        assert np.all(g["w"] == np.float32(wl.scale / wl.K))
        assert np.array_equal(g["counts"][:wl.K], np.full(wl.K, wl.T))


def test_renormalize_off_and_selection_only_bias():
    wl = synth.workload("tiny")
    x, _, wr, _, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x, renormalize=False)
    r0 = oracle.route(oracle.cfg_for(wl, renormalize=False), x, wr)
    _gpu.check_routes(g, r0, wl.E)
    bias = np.zeros(wl.E, np.float32)
    bias[[1, 2, 9]] = [0.3, 0.2, -0.25]
    for mode in (0, 1):
        ocfg = oracle.cfg_for(wl, bias_mode=mode)
        rb = oracle.route(ocfg, x, wr, bias)
        ok = rb["margins"].min(1) >= _inputs.MARGIN  # compare tokens with a clear margin
        g = _gpu.forward(wl, x, bias=bias, bias_mode=mode)
        sub = {k: v[ok] for k, v in g.items() if k in ("ids", "w")}
        gi, gw = _gpu.sorted_routes(sub["ids"], sub["w"])
        oi, ow = _gpu.sorted_routes(rb["ids"][ok], rb["weights"][ok])
        assert ok.mean() > 0.8
        assert np.array_equal(gi, oi)
        assert np.allclose(gw, ow, rtol=1e-5, atol=1e-6)


def test_forward_is_deterministic():
    wl = synth.workload("tiny").with_T(200)
    x = synth.host_x(wl)
    a = _gpu.forward(wl, x)
    b = _gpu.forward(wl, x)
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["w"], b["w"])


def test_routed_forward_matches_oracle():
    """Caller-supplied routes (routing replay): the oracle's own ids and weights."""
    wl = synth.workload("tiny").with_T(150)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    cfg = _gpu.cfg_of(wl)
    w13, w2, _ = _gpu.device_weights(wl)
    xd = _gpu.to_dev_bits(x)
    ids = torch.from_numpy(r["ids"]).cuda()
    w = torch.from_numpy(r["weights"].astype(np.float32)).cuda()
    out = torch.empty((wl.T, wl.H), dtype=torch.int16, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T), dtype=torch.uint8, device="cuda")
    bm.beam_moe_forward_routed(cfg, xd, ids, w, w13, w2, out, ws, counts)
    assert bm.beam_moe_check(ws) == 0
    ref = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], synth.host_w13(wl),
                         synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(_gpu.bits_of(out), ref)
    assert err <= _gpu.TOL
    assert np.array_equal(counts.cpu().numpy(), np.bincount(r["ids"].ravel(), minlength=wl.E))
    # an out-of-range id is dropped and flagged, never dereferenced
    ids[3, 1] = wl.E + 5
    bm.beam_moe_forward_routed(cfg, xd, ids, w, w13, w2, out, ws, counts)
    assert bm.beam_moe_check(ws) & 0x100


def test_routed_forward_on_cta_pairs_with_dropped_and_repeated_ids():
    """Routing replay with both grouped GEMMs on CTA pairs: an out-of-range id
    drops its assignment (flag 0x100), a token with no valid id gets a zero
    row, and a repeated id (outside the call's contract of distinct ids) adds
    the expert's output once per slot, as the oracle's sum does."""
    wl = synth.workload("tiny").with_T(600)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    cfg = _gpu.cfg_of(wl)
    assert bm.beam_moe_workspace_layout(cfg, wl.T).pair_down == 1
    w13, w2, _ = _gpu.device_weights(wl)
    ids = r["ids"].astype(np.int32).copy()
    w = r["weights"].astype(np.float32).copy()
    ids[3, 1] = wl.E + 5
    ids[5, :] = -1
    ids[7, 2] = ids[7, 0]
    ids[9, :] = ids[9, 0]
    out = torch.empty((wl.T, wl.H), dtype=torch.int16, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T), dtype=torch.uint8, device="cuda")
    bm.beam_moe_forward_routed(cfg, _gpu.to_dev_bits(x), torch.from_numpy(ids).cuda(),
                               torch.from_numpy(w).cuda(), w13, w2, out, ws, None)
    assert bm.beam_moe_check(ws) & 0x100
    got = _gpu.bits_of(out)
    assert not got[5].any()  # no valid id: a zero row
    bad = (ids < 0) | (ids >= wl.E)
    ref = oracle.experts(oracle.cfg_for(wl), x, np.where(bad, 0, ids), np.where(bad, 0.0, w),
                         synth.host_w13(wl), synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(got, ref)
    assert err <= _gpu.TOL


def test_routed_forward_light_expert_bounds():
    """Routing replay with 900 tokens (CTA pairs on): experts with exactly 64
    rows (the largest that runs on one-CTA tiles), 65 (the smallest on pairs),
    1 and 0 rows, the others about 290; every output row against the oracle,
    the counts bit-exact."""
    wl = synth.workload("tiny").with_T(900)
    x, _, _, _, _ = _inputs.routed_inputs(wl)
    T, K, E = wl.T, wl.K, wl.E
    rng = np.random.default_rng(7)
    ids = np.empty((T, K), np.int32)
    heavy = np.arange(4, E)
    for t in range(T):
        first = 0 if t < 64 else 1 if t < 129 else 2 if t == 129 else None
        rest = rng.choice(heavy, size=K if first is None else K - 1, replace=False)
        ids[t] = rest if first is None else np.concatenate([[first], rest])
    w = rng.uniform(0.05, 0.6, size=(T, K)).astype(np.float32)
    counts_want = np.bincount(ids.ravel(), minlength=E)
    assert list(counts_want[:4]) == [64, 65, 1, 0]
    cfg = _gpu.cfg_of(wl)
    lay = bm.beam_moe_workspace_layout(cfg, T)
    assert lay.pair_gateup == 1 and lay.light_rows == 64
    w13, w2, _ = _gpu.device_weights(wl)
    out = torch.empty((T, wl.H), dtype=torch.int16, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    bm.beam_moe_forward_routed(cfg, _gpu.to_dev_bits(x), torch.from_numpy(ids).cuda(),
                               torch.from_numpy(w).cuda(), w13, w2, out, ws, counts)
    assert bm.beam_moe_check(ws) == 0
    assert np.array_equal(counts.cpu().numpy(), counts_want)
    ref = oracle.experts(oracle.cfg_for(wl), x, ids, w, synth.host_w13(wl), synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(_gpu.bits_of(out), ref)
    assert err <= _gpu.TOL


@pytest.mark.parametrize("T", [300, 2000])  # one-CTA tiles of 32 tokens; CTA pairs
def test_widest_configuration(T):
    """The most experts and the largest top-k the library takes: 512 experts
    in 8 groups of 64, top-4 groups, top-32 (16 experts per lane in the top-k
    warp, 32 slots per token in the permute and the combine). Routes bit-exact,
    every output row against the oracle."""
    wl = synth.Workload(name="wide", T=T, H=256, I=128, E=512, G=8, Gk=4, K=32)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    lay = bm.beam_moe_workspace_layout(_gpu.cfg_of(wl), T)
    assert lay.pair_gateup == (1 if T == 2000 else 0)
    ref = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], synth.host_w13(wl),
                         synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(g["out"], ref)
    assert err <= _gpu.TOL, err


@pytest.mark.parametrize("E,G,Gk,K,H,T", [(4, 2, 1, 2, 128, 100),    # 2 groups of 2, keep 1
                                           (16, 1, 1, 4, 256, 200),   # one group: no group step
                                           (16, 4, 2, 1, 256, 150)])  # top-1: weight = scale
def test_smallest_configurations(E, G, Gk, K, H, T):
    """Degenerate routing shapes: the fewest experts per group the top-k warp
    takes, a single group (the group selection keeps everything), and top-1
    routing (renormalised, every weight is exactly the scale). Routes
    bit-exact, every output row against the oracle."""
    wl = synth.Workload(name="small", T=T, H=H, I=128, E=E, G=G, Gk=Gk, K=K)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward(wl, x)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    if K == 1:
        assert np.all(g["w"] == np.float32(wl.scale))
    ref = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], synth.host_w13(wl),
                         synth.host_w2(wl))
    err, _ = _gpu.max_rel_err(g["out"], ref)
    assert err <= _gpu.TOL, err


def test_route_only_entry_point():
    wl = synth.workload("decode").with_T(300)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    cfg = _gpu.cfg_of(wl)
    _, _, wrd = _gpu.device_weights(wl)
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T, bm.OP_ROUTE), dtype=torch.uint8,
                     device="cuda")
    bm.beam_moe_route(cfg, _gpu.to_dev_bits(x), wrd, None, ids, w, counts, ws)
    assert bm.beam_moe_check(ws) == 0
    g = {"ids": ids.cpu().numpy(), "w": w.cpu().numpy(), "counts": counts.cpu().numpy()}
    _gpu.check_routes(g, r, wl.E)
    # listed by descending score: the oracle's order where consecutive scores differ clearly
    s = np.take_along_axis(r["scores"], np.argsort(-r["scores"], 1), 1)
    clear = np.all(np.abs(np.diff(s, axis=1)) > 1e-5, axis=1)
    assert np.array_equal(g["ids"][clear], r["ids"][clear])


def test_decode_full_size():
    """Every one of the 64 output rows."""
    _full_case("decode", tokens=np.arange(64))


def test_prefill_full_size():
    *_, tokens = _full_case("prefill", min_rows=512)
    assert len(tokens) >= 512


def test_skewed_full_size():
    wl, x, r, g, tokens = _full_case("skewed")
    hot = synth.hot_experts(wl)
    assert g["counts"][hot].sum() > 0.5 * wl.T * wl.K  # the 16 hot experts take most rows
    # experts with more rows than weight rows run token block by token block,
    # the others weight block by weight block: both orders are compared
    assert g["counts"].max() > 2 * wl.I and np.any((g["counts"] > 0) & (g["counts"] <= 2 * wl.I))


def test_long_full_size():
    _full_case("long")
