"""beam_moe_forward_host / beam_moe_forward_nvfp4_host: the forward on host
buffers. One chunk must give exactly beam_moe_forward's bytes; a batch of
several chunks must give exactly the bytes of device forwards over the same
chunks (each chunk is routed on its own) and match the oracle on sampled
tokens."""
import numpy as np
import pytest
import torch

import sparse_moe_layer_beam_b200 as bm
import synth
from tests import _gpu, _inputs

pytestmark = pytest.mark.gpu

TINY4 = synth.Workload(name="tiny-nvfp4", T=64, H=256, I=256, E=16, G=4, Gk=2, K=4)


def _host_forward(wl, x_bits, nvfp4=False):
    cfg = _gpu.cfg_of(wl)
    T = x_bits.shape[0]
    x_host = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).pin_memory()
    out_host = torch.empty((T, wl.H), dtype=torch.int16).pin_memory()
    op = bm.OP_FORWARD_NVFP4_HOST if nvfp4 else bm.OP_FORWARD_HOST
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, T, op), dtype=torch.uint8, device="cuda")
    if nvfp4:
        c13, s13, c2, s2, wr = _gpu.device_weights_nvfp4(wl)
        bm.beam_moe_forward_nvfp4_host(cfg, x_host, wr, None,
                                       _gpu.nvfp4_experts(c13, s13, c2, s2), out_host, ws)
    else:
        w13, w2, wr = _gpu.device_weights(wl)
        bm.beam_moe_forward_host(cfg, x_host, wr, None, w13, w2, out_host, ws)
    torch.cuda.synchronize()
    return out_host.numpy().view(np.uint16).copy()


def _device_chunks(wl, x_bits, nvfp4=False):
    fwd = _gpu.forward_nvfp4 if nvfp4 else _gpu.forward
    T, C = x_bits.shape[0], bm.HOST_CHUNK
    chunk = T if T < 2 * C else (2 * C if (not nvfp4 and T >= 8 * C) else C)
    return np.concatenate([fwd(wl, x_bits[t:t + chunk])["out"] for t in range(0, T, chunk)])


@pytest.mark.parametrize("T", [1, 64, 300])
def test_one_chunk_equals_device_forward(T):
    wl = synth.workload("tiny").with_T(T)
    x, _, _, _, _ = _inputs.routed_inputs(wl)
    assert np.array_equal(_host_forward(wl, x), _gpu.forward(wl, x)["out"])


@pytest.mark.parametrize("nvfp4,T", [(False, 2 * bm.HOST_CHUNK + 3616),
                                     (True, 2 * bm.HOST_CHUNK + 3616),
                                     (False, 8 * bm.HOST_CHUNK + 4464)])  # 2C-token chunks
def test_chunked_batch(nvfp4, T):
    wl = (TINY4 if nvfp4 else synth.workload("tiny")).with_T(T)
    x, _, _, _, r = _inputs.routed_inputs(wl)
    got = _host_forward(wl, x, nvfp4)
    assert np.array_equal(got, _device_chunks(wl, x, nvfp4))  # several chunks, the last ragged
    tokens = synth.sample_tokens(wl.T, 48)
    ref = (_gpu.oracle_outputs_nvfp4 if nvfp4 else _gpu.oracle_outputs)(wl, x, tokens, r)
    err, rms = _gpu.max_rel_err(got[tokens], ref)
    assert err <= _gpu.TOL, (err, rms)
