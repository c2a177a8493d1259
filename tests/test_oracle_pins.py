"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Source of the method: Hugging Face launch post "Welcome Beam", section
"Mixture of Experts" (sigmoid scores over 256 experts, 8 groups of 32, keep
the 4 groups with the best sum of their two top scores, top 8 experts inside
them, SwiGLU experts of intermediate 2560, normalized weights, scale 2.5, no
shared expert). None of these checks re-types the oracle's code: they use
brute-force enumeration, closed forms that reduce to a dense SwiGLU MLP
computed with numpy matmuls, exact special cases, invariants and the page's
printed constants.
"""
import itertools
import math
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle
import synth
from tests import _inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "beam_block_constants.txt")


def golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = [s.strip() for s in line.split("=")]
                vals[k] = float(v)
    return vals


def f64(bits):
    return synth.bf16_to_f32(bits).astype(np.float64)


def dense_swiglu(x, w13_bits, w2_bits):
    """Textbook dense SwiGLU MLP with numpy float64 matmuls: Wd (silu(Wg x) * Wu x)."""
    w13 = f64(w13_bits)
    I = w13.shape[0] // 2
    g = x @ w13[:I].T
    u = x @ w13[I:].T
    return (g * expit(g) * u) @ f64(w2_bits).T


# ------------------------------------------------------------- page constants

def test_golden_constants_match_workloads():
    g = golden()
    wl = synth.workload("decode")
    assert wl.H == g["hidden_size"] and wl.I == g["expert_intermediate"]
    assert wl.E == g["n_experts"] and wl.G == g["n_group"]
    assert wl.E // wl.G == g["experts_per_group"]
    assert wl.Gk == g["topk_group"] and wl.K == g["top_k"] and wl.scale == g["routed_scale"]
    assert g["dense_layers"] + g["moe_layers"] == g["num_layers"]


def test_golden_parameter_counts_are_consistent():
    g = golden()
    per_expert = 3 * g["hidden_size"] * g["expert_intermediate"]  # gate, up, down
    assert per_expert == 39_321_600
    assert abs(per_expert - g["params_per_expert_about"]) < 0.5e6  # "about 39M"
    experts_total = per_expert * g["n_experts"] * g["moe_layers"]
    # 501B is rounded to the nearest billion: the share must fall inside that envelope
    lo, hi = experts_total / (g["total_params"] + 0.5e9), experts_total / (g["total_params"] - 0.5e9)
    assert lo * 100 <= g["expert_share_percent"] + 0.05 and g["expert_share_percent"] - 0.05 <= hi * 100
    # active: top-8 experts of every MoE layer plus the replicated 8B part, about 23B
    active = g["top_k"] * per_expert * g["moe_layers"] + g["replicated_params"]
    assert abs(active - g["active_params"]) < 0.6e9


# ------------------------------------------------------------------ routing

def test_scores_are_sigmoid_of_router_logits():
    wl = synth.workload("tiny")
    x = synth.host_x(wl)
    wr = synth.host_router(wl)
    r = oracle.route(oracle.cfg_for(wl), x, wr, want_all_s=True)
    ref = expit(f64(x) @ wr.astype(np.float64).T)
    assert np.allclose(r["all_s"], ref, rtol=0, atol=1e-13)


def _brute_force_route(s, G, Gk, K):
    """Best group subset by total group score, then best expert subset by total score."""
    E = s.shape[0]
    per = E // G
    gscore = np.array([np.sort(s[g * per:(g + 1) * per])[-2:].sum() for g in range(G)])
    best_groups = max(itertools.combinations(range(G), Gk), key=lambda c: gscore[list(c)].sum())
    eligible = [e for g in best_groups for e in range(g * per, (g + 1) * per)]
    best = max(itertools.combinations(eligible, K), key=lambda c: s[list(c)].sum())
    return set(best_groups), set(best), gscore


@pytest.mark.parametrize("shape", ["tiny", "micro"])
def test_brute_force_routes(shape):
    if shape == "tiny":
        wl = synth.workload("tiny")
    else:  # 8 experts in 4 groups of 2, keep 2 groups, top 2: every route enumerated
        wl = synth.Workload(name="micro", T=128, H=64, I=32, E=8, G=4, Gk=2, K=2)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    s_all = expit(f64(x) @ wr.astype(np.float64).T)
    for t in range(wl.T):
        groups, chosen, gscore = _brute_force_route(s_all[t], wl.G, wl.Gk, wl.K)
        assert set(r["kept"][t].tolist()) == groups, t
        assert set(r["ids"][t].tolist()) == chosen, t
        # kept groups carry the sum of their top-2 scores, as ranked
        assert np.all(np.diff(gscore[r["kept"][t]]) <= 0)


def test_invariants_at_beam_shape():
    wl = synth.workload("decode")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    s_all = expit(f64(x) @ wr.astype(np.float64).T)
    per = wl.E // wl.G
    for t in range(wl.T):
        ids, kept = r["ids"][t], r["kept"][t]
        assert len(set(ids.tolist())) == wl.K  # 8 distinct experts
        assert len(set(kept.tolist())) == wl.Gk  # exactly 4 kept groups
        assert set((ids // per).tolist()) <= set(kept.tolist())  # drawn from kept groups
        gscore = np.sort(s_all[t].reshape(wl.G, per), axis=1)[:, -2:].sum(axis=1)
        others = np.setdiff1d(np.arange(wl.G), kept)
        assert gscore[kept].min() > gscore[others].max()
        eligible = np.concatenate([np.arange(g * per, (g + 1) * per) for g in kept])
        rest = np.setdiff1d(eligible, ids)
        assert s_all[t, ids].min() > s_all[t, rest].max()
        assert np.all(np.diff(s_all[t, ids]) <= 0)  # listed by descending score
        assert np.allclose(r["scores"][t], s_all[t, ids], atol=1e-13)
    assert r["margins"].min() >= _inputs.MARGIN


def _margins_numpy(s, choice, G, Gk, K):
    """(group margin, expert margin) of one token from the scores alone: rank
    the groups by the sum of their two best choice scores, keep Gk, take the K
    best choice scores among the kept groups' experts; each margin is the last
    kept candidate's value minus the best rejected one's (inf if none)."""
    E = s.shape[0]
    per = E // G
    gscore = np.sort(choice.reshape(G, per), axis=1)[:, -2:].sum(axis=1)
    order = sorted(range(G), key=lambda g: (-gscore[g], g))
    kept, rest = order[:Gk], order[Gk:]
    mg = gscore[kept].min() - gscore[rest].max() if rest else math.inf
    eligible = np.concatenate([np.arange(g * per, (g + 1) * per) for g in kept])
    ranked = sorted(eligible.tolist(), key=lambda e: (-choice[e], e))
    me = choice[ranked[K - 1]] - choice[ranked[K]] if len(ranked) > K else math.inf
    return mg, me


@pytest.mark.parametrize("name,bias_mode", [("tiny", 0), ("tiny", 1), ("decode", 0)])
def test_margins_match_an_independent_recomputation(name, bias_mode):
    """The margins the parity inputs are re-drawn on, recomputed from sigmoid
    scores of numpy logits, with the group and expert ranking written out
    here: a margin taken from the wrong side, over the wrong experts or from
    the wrong kept group would let near-tie tokens into the parity tests."""
    wl = synth.workload(name).with_T(48)
    x = synth.host_x(wl)
    wr = synth.host_router(wl)
    bias = np.linspace(-0.2, 0.2, wl.E).astype(np.float32)
    r = oracle.route(oracle.cfg_for(wl, bias_mode=bias_mode), x, wr, bias)
    lg = f64(x) @ wr.astype(np.float64).T
    for t in range(wl.T):
        if bias_mode == 0:
            s = expit(lg[t] + bias)
            c = s
        else:
            s = expit(lg[t])
            c = s + bias.astype(np.float64)
        mg, me = _margins_numpy(s, c, wl.G, wl.Gk, wl.K)
        assert r["margins"][t, 0] == pytest.approx(mg, rel=1e-9, abs=1e-12), t
        assert r["margins"][t, 1] == pytest.approx(me, rel=1e-9, abs=1e-12), t
    assert r["margins"].min() >= 0.0


def test_tie_case_selects_lowest_indices():
    for name in ("tiny", "decode"):
        wl = synth.workload(name).with_T(4)
        x = synth.host_x(wl)
        wr = np.zeros((wl.E, wl.H), np.float32)
        r = oracle.route(oracle.cfg_for(wl), x, wr, np.zeros(wl.E, np.float32))
        assert np.array_equal(r["kept"], np.tile(np.arange(wl.Gk), (4, 1)))
        assert np.array_equal(r["ids"], np.tile(np.arange(wl.K), (4, 1)))
        assert np.all(r["weights"] == wl.scale / wl.K)
        assert np.all(r["scores"] == 0.5)


def test_weights_sum_to_scale_when_renormalized():
    wl = synth.workload("tiny")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    assert np.allclose(r["weights"].sum(axis=1), 2.5, rtol=1e-12)
    r0 = oracle.route(oracle.cfg_for(wl, renormalize=False), x, wr, b)
    assert np.array_equal(r0["ids"], r["ids"])
    assert np.allclose(r0["weights"], 2.5 * r["scores"], rtol=1e-14)


def test_bias_on_logits_and_selection_only_bias():
    """A large bias on two experts of one group lifts that group's top-2 sum above
    every other group's, so both experts are chosen, 13 (bias 40) before 12 (20).
    A bias on one expert alone need not help: its group can still lose on the
    sum of its top two scores, which is what group-limited routing means."""
    wl = synth.workload("tiny")
    x = synth.host_x(wl)
    wr = synth.host_router(wl)
    bias = np.zeros(wl.E, np.float32)
    bias[13], bias[12] = 40.0, 20.0
    lg = f64(x) @ wr.astype(np.float64).T
    r0 = oracle.route(oracle.cfg_for(wl, bias_mode=0), x, wr, bias)
    assert np.all(r0["ids"][:, 0] == 13) and np.all(r0["ids"][:, 1] == 12)
    assert np.all(r0["kept"][:, 0] == 3)
    assert np.allclose(r0["scores"][:, 0], expit(lg[:, 13] + 40.0), atol=1e-15)
    r1 = oracle.route(oracle.cfg_for(wl, bias_mode=1), x, wr, bias)
    assert np.all(r1["ids"][:, 0] == 13) and np.all(r1["ids"][:, 1] == 12)
    s = expit(lg)  # selection-only: the weights come from the unbiased scores
    sel = np.take_along_axis(s, r1["ids"].astype(np.int64), 1)
    assert np.allclose(r1["weights"], 2.5 * sel / sel.sum(1, keepdims=True), rtol=1e-12)
    one = np.zeros(wl.E, np.float32)
    one[13] = 40.0
    r2 = oracle.route(oracle.cfg_for(wl), x, wr, one, want_all_s=True)
    gs = np.sort(r2["all_s"].reshape(wl.T, wl.G, -1), axis=2)[:, :, -2:].sum(2)
    dropped = ~np.any(r2["ids"] == 13, axis=1)
    assert np.all(np.sort(gs[dropped], 1)[:, -wl.Gk] > gs[dropped, 3])


# ------------------------------------------------------------ expert math

def test_single_expert_is_dense_swiglu():
    wl = synth.workload("tiny")
    x = f64(synth.host_x(wl))[:4]
    w13, w2 = synth.host_expert_w13(wl, 5), synth.host_expert_w2(wl, 5)
    ref = dense_swiglu(x, w13, w2)
    for t in range(4):
        assert np.allclose(oracle.swiglu_expert(x[t], w13, w2), ref[t], rtol=1e-11, atol=1e-14)


def test_hidden_is_dense_swiglu_hidden():
    """oracle.hidden gives silu(Wg x) * (Wu x) of each routed (token, slot),
    against numpy matmuls, for the expert each slot names."""
    wl = synth.workload("tiny").with_T(12)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    w13 = synth.host_w13(wl)
    a = oracle.hidden(oracle.cfg_for(wl), x, r["ids"], w13)
    xf = f64(x)
    for t in range(wl.T):
        for k in range(wl.K):
            w = f64(w13[r["ids"][t, k]])
            g, u = w[:wl.I] @ xf[t], w[wl.I:] @ xf[t]
            assert np.allclose(a[t, k], g * expit(g) * u, rtol=1e-11, atol=1e-14), (t, k)


@pytest.mark.parametrize("renormalize", [True, False])
def test_identical_experts_closed_form(renormalize):
    """All experts equal to one dense SwiGLU f: out = S * (sum of weights) * f(x);
    with renormalization that is exactly 2.5 * f(x)."""
    wl = synth.workload("tiny")
    x, _, wr, b, _ = _inputs.routed_inputs(wl)
    cfg = oracle.cfg_for(wl, renormalize=renormalize)
    w13, w2 = synth.host_expert_w13(wl, 0), synth.host_expert_w2(wl, 0)
    r, out = oracle.forward(cfg, x, wr, b, [w13] * wl.E, [w2] * wl.E)
    f = dense_swiglu(f64(x), w13, w2)
    s = expit(f64(x) @ wr.astype(np.float64).T)
    wsum = 2.5 * (np.ones(wl.T) if renormalize else np.take_along_axis(
        s, r["ids"].astype(np.int64), 1).sum(1))
    assert np.allclose(out, wsum[:, None] * f, rtol=1e-10, atol=1e-13)


def test_expert_index_closed_form():
    """Expert e = the same f with its up rows scaled by 2^(e mod 3) and its down
    weights by 2^(e mod 2) (exact in bf16): out = sum_k w_k 2^(..) f(x). A wrong
    expert index, slot or weight fails it."""
    wl = synth.workload("tiny")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g0, d0 = synth.host_expert_w13(wl, 0), synth.host_expert_w2(wl, 0)
    w13s, w2s, mult = [], [], []
    for e in range(wl.E):
        up = f64(g0[wl.I:]) * 2.0 ** (e % 3)
        w13s.append(np.concatenate([g0[:wl.I], synth_bits(up)]))
        w2s.append(synth_bits(f64(d0) * 2.0 ** (e % 2)))
        mult.append(2.0 ** (e % 3 + e % 2))
    out = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], w13s, w2s)
    f = dense_swiglu(f64(x), g0, d0)
    m = (r["weights"] * np.array(mult)[r["ids"]]).sum(1)
    assert np.allclose(out, m[:, None] * f, rtol=1e-10, atol=1e-13)


def synth_bits(v):
    """float64 values exactly representable in bf16 -> bits."""
    f = np.asarray(v, np.float32)
    assert np.array_equal(f.astype(np.float64), v)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_to_f32(bits), f)
    return bits


def test_output_is_linear_in_down_weights():
    wl = synth.workload("tiny")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    w13, w2 = synth.host_w13(wl), synth.host_w2(wl)
    out1 = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], w13, w2)
    w2x2 = synth_bits(f64(w2) * 2.0)
    out2 = oracle.experts(oracle.cfg_for(wl), x, r["ids"], r["weights"], w13, w2x2)
    assert np.array_equal(out2, 2.0 * out1)


def test_no_shared_expert_and_unselected_experts_unused():
    """Changing an expert no token selects leaves the output unchanged (there is
    no shared expert); changing a selected one changes exactly its tokens."""
    wl = synth.workload("tiny")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    w13, w2 = synth.host_w13(wl), synth.host_w2(wl)
    cfg = oracle.cfg_for(wl)
    base = oracle.experts(cfg, x, r["ids"], r["weights"], w13, w2)
    counts = np.bincount(r["ids"].ravel(), minlength=wl.E)
    e = int(np.argmax(counts))
    w2m = w2.copy()
    w2m[e] = synth_bits(f64(w2[e]) * 2.0)
    out = oracle.experts(cfg, x, r["ids"], r["weights"], w13, w2m)
    hit = np.any(r["ids"] == e, axis=1)
    assert np.array_equal(out[~hit], base[~hit])
    assert np.all(np.abs(out[hit] - base[hit]).max(axis=1) > 0)
    unused = np.nonzero(counts == 0)[0]
    if unused.size:
        w13m = w13.copy()
        w13m[unused[0]] = 0
        assert np.array_equal(oracle.experts(cfg, x, r["ids"], r["weights"], w13m, w2), base)


def test_margin_redraw_converges_and_is_deterministic():
    wl = synth.workload("decode")
    x1, a1, _, _, r1 = _inputs.routed_inputs(wl)
    x2, a2, _, _, r2 = _inputs.routed_inputs(wl)
    assert np.array_equal(x1, x2) and np.array_equal(a1, a2)
    assert r1["margins"].min() >= _inputs.MARGIN
    assert math.isfinite(r1["weights"].sum())
