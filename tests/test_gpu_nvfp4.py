"""NVFP4 (W4A4) path against the oracle: the GPU quantiser bit for bit (scales
exactly, values exactly), the device weight fill against the host generator,
and the whole block (routing bit-exact; outputs against the oracle's fp64
evaluation on exactly dequantised values within half a bf16 step of the
output plus 3e-2 x RMS per element, and an RMS error within 1e-3 x RMS of the
output's own bf16 rounding: see _gpu.TOL_NVFP4_ELEM for the derivation)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu

TINY4 = synth.Workload(name="tiny-nvfp4", T=64, H=256, I=256, E=16, G=4, Gk=2, K=4)


def test_gpu_quantizer_matches_oracle_bit_for_bit():
    rng = np.random.default_rng(3)
    rows = [rng.standard_normal(512) * s for s in (1e-4, 0.02, 0.3, 1.0, 7.0, 300.0)]
    ties = np.repeat(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float64), 2)
    rows.append(np.concatenate([ties, -ties, np.zeros(16), ties * 3] * 8)[:512])
    v = np.stack(rows).astype(np.float32)
    for g in (2.0 ** -6, 1.0, 0.37):
        vc = torch.from_numpy(v).cuda()
        codes = torch.empty((v.shape[0], 256), dtype=torch.uint8, device="cuda")
        sf = torch.empty((v.shape[0], 32), dtype=torch.uint8, device="cuda")
        bm.beam_moe_nvfp4_quantize(vc, g, codes, sf)
        torch.cuda.synchronize()
        oc, osf = oracle.nvfp4_quantize(v, np.float32(g))
        assert np.array_equal(sf.cpu().numpy(), osf)
        gv = oracle.nvfp4_dequant(codes.cpu().numpy(), osf, g)
        assert np.array_equal(gv, oracle.nvfp4_dequant(oc, osf, g))


def test_device_nvfp4_weights_match_host():
    wl = TINY4
    c13, s13, c2, s2, _ = _gpu.device_weights_nvfp4(wl)
    hc, hs = synth.host_expert_w13_nvfp4(wl, 5)
    rows = 2 * wl.I
    dc = c13.cpu().numpy().reshape(wl.E * rows, wl.H // 2)[5 * rows:6 * rows]
    assert np.array_equal(dc, hc)
    r, b = np.meshgrid(np.arange(5 * rows, 6 * rows), np.arange(wl.H // 16), indexing="ij")
    ds = s13.cpu().numpy()[synth.sf_offset(r, b, wl.H)]
    assert np.array_equal(ds, hs)


@pytest.mark.parametrize("T", [64, 1, 129, 300, 1024, 4000, 4100])  # from 1024 rows/expert: pairs
def test_nvfp4_forward_tiny(T):
    wl = TINY4.with_T(T)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward_nvfp4(wl, x)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    tokens = np.arange(wl.T) if wl.T <= 256 else synth.sample_tokens(wl.T, 64)
    ref = _gpu.oracle_outputs_nvfp4(wl, x, tokens, r, batch=64)
    _gpu.check_nvfp4(g["out"][tokens], ref)


def _full_case(name, tokens=None):
    """Routing on every token; outputs on `tokens`, by default the tokens that
    cover the first and last rows of every touched expert's first and last
    128-row token tile (the NVFP4 GEMMs' tile; its 256-row pair tiles start on
    every other one)."""
    wl = synth.workload(name)
    x, _, wr, b, r = _inputs.routed_inputs(wl)
    g = _gpu.forward_nvfp4(wl, x, bias=b)
    assert g["flags"] == 0
    _gpu.check_routes(g, r, wl.E)
    if tokens is None:
        tokens = _gpu.block_cover_tokens(r["ids"], wl.E, 128)
    ref = _gpu.oracle_outputs_nvfp4(wl, x, tokens, r)
    _gpu.check_nvfp4(g["out"][tokens], ref)


def test_nvfp4_decode_full_size():
    """Every one of the 64 output rows."""
    _full_case("decode", tokens=np.arange(64))


def test_nvfp4_prefill_full_size():
    _full_case("prefill")


def test_nvfp4_skewed_full_size():  # router bias on the logits of 16 hot experts
    _full_case("skewed")


def test_nvfp4_long_full_size():  # 2048 rows per expert: the down GEMM runs on CTA pairs
    _full_case("long")
