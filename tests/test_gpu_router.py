"""The FP32 router ("Welcome Beam", section "Residual Stream": the router runs
in FP32; section "Mixture of Experts": sigmoid scores) on both of its GEMM
paths, through the C ABI: the default chain of FP32 FMAs on CUDA cores and the
opt-in tensor-core contraction (router_tc = 1: each FP32 weight split exactly
into three bf16 parts, products exact, sums in the tensor core's FP32
accumulator).

With renormalize = 0 a token's weights are S * s_k, so the sigmoid scores
come back exactly up to the FP32 multiply by S. Each is compared with the
oracle's fp64 score within the error bound of an FP32 sum of H products,
gamma * sum_h |x_h w_h| with gamma = H * 2^-24 (any order of H - 1 additions,
each rounding by at most 2^-24 of a partial sum bounded by that magnitude;
twice that for the tensor core's accumulator, whose additions need not round
to nearest), times the sigmoid's slope s (1 - s) <= 1/4, plus FP32 rounding of
the sigmoid, the bias and the scale. The chosen experts must equal the
oracle's bit for bit (inputs are re-drawn until every margin exceeds 1e-4).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu


def _route(wl, x_bits, bias, router_tc, renormalize):
    cfg = bm.beam_cfg(wl.H, wl.I, wl.E, wl.G, wl.Gk, wl.K, renormalize, 0, wl.scale,
                      router_tc=router_tc)
    _, _, wr = _gpu.device_weights(wl)
    T = x_bits.shape[0]
    ids = torch.empty((T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.K), dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, T, bm.OP_ROUTE), dtype=torch.uint8,
                     device="cuda")
    b = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).cuda()
    bm.beam_moe_route(cfg, _gpu.to_dev_bits(x_bits), wr, b, ids, w, counts, ws)
    assert bm.beam_moe_check(ws) == 0
    lay = bm.beam_moe_workspace_layout(cfg, T, bm.OP_ROUTE)
    assert lay.router_tc == (1 if router_tc else 0)
    return {"ids": ids.cpu().numpy(), "w": w.cpu().numpy(), "counts": counts.cpu().numpy()}


@pytest.mark.parametrize("name,T", [("tiny", 300), ("decode", 64), ("decode", 1000),
                                    ("skewed", 512)])
@pytest.mark.parametrize("router_tc", [False, True])
def test_router_scores_within_the_fp32_bound(name, T, router_tc):
    wl = synth.workload(name).with_T(T)
    x, _, wr, b, _ = _inputs.routed_inputs(wl)
    r = oracle.route(oracle.cfg_for(wl, renormalize=False), x, wr, b)
    ok = r["margins"].min(1) >= _inputs.MARGIN  # margins were checked with renormalize on
    assert ok.mean() > 0.95
    g = _route(wl, x, b, router_tc, renormalize=False)
    gi, gw = _gpu.sorted_routes(g["ids"], g["w"])
    oi, os_ = _gpu.sorted_routes(r["ids"], r["scores"])
    assert np.array_equal(gi[ok], oi[ok])
    xf = synth.bf16_to_f32(x).astype(np.float64)
    mag = np.abs(xf) @ np.abs(wr.astype(np.float64)).T  # [T, E] sum_h |x_h w_h|
    gamma = (2.0 if router_tc else 1.0) * wl.H * 2.0 ** -24
    bound = 0.25 * gamma * np.take_along_axis(mag, oi.astype(np.int64), 1) + 2.0 ** -20
    s_gpu = gw.astype(np.float64) / wl.scale
    err = np.abs(s_gpu - os_)[ok]
    print(f"{name} T={T} tc={router_tc}: max |ds| {err.max():.3e}, "
          f"max |ds| / bound {(err / bound[ok]).max():.3e}")
    assert np.all(err <= bound[ok])


@pytest.mark.parametrize("router_tc", [False, True])
def test_router_paths_choose_the_oracles_experts_at_beam_shape(router_tc):
    """Both GEMM paths give the oracle's expert sets and counts at 4096 tokens,
    with renormalized weights within the parity tests' tolerance."""
    wl = synth.workload("prefill")
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _route(wl, x, b, router_tc, renormalize=True)
    _gpu.check_routes(g, r, wl.E)
