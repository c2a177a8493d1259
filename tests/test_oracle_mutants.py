"""The oracle's pins catch plausible mistakes: each mutant below plants one in
a copy of the C oracle (a dropped term, a flipped sign, a wrong index, a
swapped or transposed operand, a wrong rounding rule), is built with the
oracle's own flags into a temporary directory, and must fail at least one pin
of tests/test_oracle_pins.py or tests/test_oracle_nvfp4.py. All mutants run in
one child process, so none of them is ever loaded into the test process; the
oracle under oracle/ is not touched. Every planted access stays inside the
arrays the unmutated code reads.
"""
import json
import os
import subprocess
import sys

from oracle import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, [(text in beam_moe_oracle.c, replacement), ...]); each text occurs once
MUTANTS = [
    ("sigmoid sign", [("s[e] = 1.0 / (1.0 + exp(-l));", "s[e] = 1.0 / (1.0 + exp(l));")]),
    ("token row ignored", [("const uint16_t* xt = x + t * (int64_t)H;",
                            "const uint16_t* xt = x;")]),
    ("logit bias dropped", [("if (bias && cfg->bias_mode == 0) l += (double)bias[e];", "")]),
    ("selection bias on the weights", [
        ("for (int k = 0; k < K; ++k) sum += s[sel[k]];",
         "for (int k = 0; k < K; ++k) sum += c[sel[k]];"),
        ("double w = cfg->renormalize ? s[sel[k]] / sum : s[sel[k]];",
         "double w = cfg->renormalize ? c[sel[k]] / sum : c[sel[k]];")]),
    ("group score from the top expert only", [
        ("gs[g] = c[b1] + (b2 >= 0 ? c[b2] : 0.0);", "gs[g] = c[b1];")]),
    ("group score from top-1 plus the worst", [
        ("} else if (b2 < 0 || beats(c[e], e, c[b2], b2)) {",
         "} else if (b2 < 0 || beats(c[b2], b2, c[e], e)) {")]),
    ("ties to the higher index", [("return va > vb || (va == vb && ia < ib);",
                                   "return va > vb || (va == vb && ia > ib);")]),
    ("one group too few kept", [("for (int r = 0; r < Gk; ++r) {",
                                 "for (int r = 0; r < Gk - 1; ++r) {"),
                                ("if (kept) kept[t * Gk + r] = best;",
                                 "if (kept) { kept[t * Gk + r] = best; kept[t * Gk + Gk - 1] = best; }")]),
    ("expert's group by modulo", [
        ("if (gkept[e / per] && !taken[e] && (best < 0 || beats(c[e], e, c[best], best)))",
         "if (gkept[e % G] && !taken[e] && (best < 0 || beats(c[e], e, c[best], best)))")]),
    ("no renormalisation", [("double w = cfg->renormalize ? s[sel[k]] / sum : s[sel[k]];",
                             "double w = s[sel[k]];")]),
    ("scale dropped", [("if (weights) weights[t * K + k] = cfg->routed_scale * w;",
                        "if (weights) weights[t * K + k] = w;")]),
    ("gate and up swapped", [("a[i] = g / (1.0 + exp(-g)) * u; /* silu(g) * u */",
                              "a[i] = u / (1.0 + exp(-u)) * g;")]),
    ("silu dropped", [("a[i] = g / (1.0 + exp(-g)) * u; /* silu(g) * u */", "a[i] = g * u;")]),
    ("silu sign", [("a[i] = g / (1.0 + exp(-g)) * u; /* silu(g) * u */",
                    "a[i] = g / (1.0 + exp(g)) * u;")]),
    ("down weights transposed", [
        ("for (int i = 0; i < I; ++i) acc += bf16_to_double(wd[i]) * a[i];",
         "for (int i = 0; i < I; ++i) acc += bf16_to_double(w2[(int64_t)i * H + j]) * a[i];")]),
    ("combine weights dropped", [("for (int h = 0; h < H; ++h) ot[h] += weights[t * K + k] * y[h];",
                                  "for (int h = 0; h < H; ++h) ot[h] += y[h];")]),
    ("E2M1 grid value", [("{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}",
                          "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0}")]),
    ("E2M1 tie to odd", [("if (a <= 0.25) c = 0;", "if (a < 0.25) c = 0;")]),
    ("E4M3 exponent bias", [("double v = E ? ldexp(1.0 + f / 8.0, E - 7) : ldexp(f / 8.0, -6);",
                             "double v = E ? ldexp(1.0 + f / 8.0, E - 8) : ldexp(f / 8.0, -6);")]),
    ("NVFP4 block scale from amax / 4", [("const float sd = amax / (6.0f * g);",
                                          "const float sd = amax / (4.0f * g);")]),
    ("NVFP4 nibble order", [
        ("uint8_t code = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);",
         "uint8_t code = (i & 1) ? (uint8_t)(byte & 15) : (uint8_t)(byte >> 4);")]),
    ("expert margin over every group", [
        ("if (gkept[e / per] && !taken[e] && c[e] > bestu) bestu = c[e];",
         "if (!taken[e] && c[e] > bestu) bestu = c[e];")]),
    ("group margin from the best kept group", [
        ("if (gkept[g] && gs[g] < lastk) lastk = gs[g];",
         "if (gkept[g] && (lastk == INFINITY || gs[g] > lastk)) lastk = gs[g];")]),
    ("hidden activations in the wrong slot", [
        ("swiglu_hidden(H, I, xd, w13[e], a + (t * K + k) * (int64_t)I);",
         "swiglu_hidden(H, I, xd, w13[e], a + t * (int64_t)I);")]),
    ("NVFP4 h not quantised", [
        ("for (int i = 0; i < I; ++i) ad[i] = nvfp4_value(ac, as, i, (double)g_h);",
         "for (int i = 0; i < I; ++i) ad[i] = af[i];")]),
]

# pins run against every mutant, cheapest first; a mutant is caught by the
# first one that fails
PINS = [
    ("test_oracle_pins", "test_tie_case_selects_lowest_indices", ()),
    ("test_oracle_pins", "test_weights_sum_to_scale_when_renormalized", ()),
    ("test_oracle_pins", "test_brute_force_routes", ("micro",)),
    ("test_oracle_pins", "test_brute_force_routes", ("tiny",)),
    ("test_oracle_pins", "test_scores_are_sigmoid_of_router_logits", ()),
    ("test_oracle_pins", "test_bias_on_logits_and_selection_only_bias", ()),
    ("test_oracle_pins", "test_single_expert_is_dense_swiglu", ()),
    ("test_oracle_pins", "test_hidden_is_dense_swiglu_hidden", ()),
    ("test_oracle_pins", "test_margins_match_an_independent_recomputation", ("tiny", 0)),
    ("test_oracle_pins", "test_identical_experts_closed_form", (True,)),
    ("test_oracle_pins", "test_identical_experts_closed_form", (False,)),
    ("test_oracle_pins", "test_expert_index_closed_form", ()),
    ("test_oracle_pins", "test_output_is_linear_in_down_weights", ()),
    ("test_oracle_pins", "test_invariants_at_beam_shape", ()),
    ("test_oracle_nvfp4", "test_e4m3_matches_torch_float8", ()),
    ("test_oracle_nvfp4", "test_e2m1_is_nearest_grid_value_with_ties_to_even", ()),
    ("test_oracle_nvfp4", "test_quantiser_error_bounds_and_round_trip", ()),
    ("test_oracle_nvfp4", "test_packing_order_low_nibble_first", ()),
    ("test_oracle_nvfp4", "test_decoder_reads_the_packing_order", ()),
    ("test_oracle_nvfp4", "test_nvfp4_identical_experts_closed_form", ()),
    ("test_oracle_nvfp4", "test_nvfp4_expert_index_and_weights", ()),
]

CHILD = r"""
import importlib, json, sys
ROOT, PINS, LIBS = json.loads(sys.argv[1])
sys.path.insert(0, ROOT)
import oracle
mods = {m: importlib.import_module("tests." + m) for m in set(p[0] for p in PINS)}
result = {}
for name, lib in LIBS:
    oracle._build.build = lambda force=False, lib=lib: lib
    oracle._lib = None
    caught = None
    for mod, fn, args in PINS:
        try:
            getattr(mods[mod], fn)(*args)
        except Exception as e:
            caught = f"{fn}{tuple(args)}: {type(e).__name__}"
            break
    result[name] = caught
print("RESULT " + json.dumps(result))
"""


def _build_mutant(tmp, idx, subs):
    with open(os.path.join(ROOT, "oracle", "beam_moe_oracle.c")) as f:
        src = f.read()
    for old, new in subs:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    d = os.path.join(tmp, f"m{idx}")
    os.makedirs(d)
    c = os.path.join(d, "beam_moe_oracle.c")
    with open(c, "w") as f:
        f.write(src)
    with open(os.path.join(ROOT, "oracle", "beam_moe_oracle.h")) as f:
        header = f.read()
    with open(os.path.join(d, "beam_moe_oracle.h"), "w") as f:
        f.write(header)
    so = os.path.join(d, "liboracle_mutant.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-ffp-contract=off", c, "-o", so, "-lm"], check=True)
    return so


def test_every_planted_mistake_fails_a_pin(tmp_path):
    _build.build()  # the unmutated oracle passes every pin in its own test files
    libs = [(name, _build_mutant(str(tmp_path), i, subs)) for i, (name, subs) in
            enumerate(MUTANTS)]
    env = dict(os.environ, OMP_NUM_THREADS=os.environ.get("OMP_NUM_THREADS", "4"))
    run = subprocess.run([sys.executable, "-c", CHILD, json.dumps([ROOT, PINS, libs])],
                         capture_output=True, text=True, timeout=900, env=env, cwd=ROOT)
    lines = [l for l in run.stdout.splitlines() if l.startswith("RESULT ")]
    assert run.returncode == 0 and lines, run.stderr[-2000:]
    result = json.loads(lines[-1][len("RESULT "):])
    survivors = [n for n, caught in result.items() if caught is None]
    assert not survivors, f"mutants no pin catches: {survivors}"
    assert set(result) == set(n for n, _ in MUTANTS)
