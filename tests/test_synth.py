"""The synthetic generator: determinism, independence of streams, moments,
and the exactness properties the host/device equality relies on."""
import numpy as np

import synth


def test_deterministic_and_seeded():
    a = synth.host_normal_bf16(4096, synth.STREAM_X)
    b = synth.host_normal_bf16(4096, synth.STREAM_X)
    c = synth.host_normal_bf16(4096, synth.STREAM_X, seed=1)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)


def test_streams_and_offsets_are_consistent():
    full = synth.host_normal_f32(1000, synth.STREAM_W2)
    tail = synth.host_normal_f32(400, synth.STREAM_W2, idx0=600)
    assert np.array_equal(full[600:], tail)
    other = synth.host_normal_f32(1000, synth.STREAM_W13)
    assert abs(np.corrcoef(full, other)[0, 1]) < 0.1


def test_normal_moments_and_exactness():
    z = synth.host_normal_f32(1 << 20, 42)
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    # sum of 12 uniforms: kurtosis 3 - 6/(5*12) = 2.9, support +-6
    kurt = ((z - z.mean()) ** 4).mean() / z.var() ** 2
    assert abs(kurt - 2.9) < 0.03
    assert np.abs(z).max() <= 6.0
    # every deviate is a multiple of 2^-17 (exact in fp32)
    assert np.all(np.floor(z.astype(np.float64) * 131072) == z.astype(np.float64) * 131072)


def test_bf16_rounding_is_nearest_even():
    f = synth.host_normal_f32(1 << 16, 9, sigma=0.02)
    bits = synth.host_normal_bf16(1 << 16, 9, sigma=0.02)
    back = synth.bf16_to_f32(bits).astype(np.float64)
    f64 = f.astype(np.float64)
    ulp = np.ldexp(1.0, np.frexp(np.abs(back))[1] - 8)
    assert np.all(np.abs(back - f64) <= ulp / 2 + 1e-30)


def test_workload_shapes_and_distributions():
    for name in ("decode", "prefill", "skewed", "long"):
        wl = synth.workload(name)
        assert (wl.H, wl.I, wl.E, wl.G, wl.Gk, wl.K, wl.scale) == (5120, 2560, 256, 8, 4, 8, 2.5)
    assert [synth.workload(n).T for n in ("decode", "prefill", "skewed", "long")] == [
        64, 4096, 16384, 65536]
    tiny = synth.workload("tiny")
    assert (tiny.T, tiny.H, tiny.I, tiny.E, tiny.G, tiny.Gk, tiny.K) == (64, 256, 128, 16, 4, 2, 4)
    wr = synth.host_router(synth.workload("decode"))
    assert wr.dtype == np.float32 and abs(wr.std() * np.sqrt(5120) - 1.0) < 0.01
    w13 = synth.bf16_to_f32(synth.host_expert_w13(tiny, 3))
    assert abs(w13.std() - 0.02) < 0.001


def test_skewed_bias_and_clustered_rows():
    sk = synth.workload("skewed")
    b = synth.host_bias(sk)
    assert b.shape == (256,) and np.count_nonzero(b) == 16 and set(np.unique(b)) == {0.0, 3.0}
    assert synth.host_bias(synth.workload("prefill")) is None
    lg = synth.workload("long").with_T(32)
    x = synth.bf16_to_f32(synth.host_x(lg)).astype(np.float64)
    # rows t and t+8 share a centre: their difference is pure noise (std 0.3*sqrt(2))
    d = x[8:16] - x[0:8]
    assert abs(d.std() - 0.3 * np.sqrt(2)) < 0.02
    assert abs(x.std() - np.sqrt(1 + 0.09)) < 0.05


def test_row_redraw_changes_only_that_row():
    wl = synth.workload("tiny")
    att = np.zeros(wl.T, np.int32)
    x0 = synth.host_x(wl, att)
    att[5] = 1
    x1 = synth.host_x(wl, att)
    assert not np.array_equal(x0[5], x1[5])
    assert np.array_equal(np.delete(x0, 5, 0), np.delete(x1, 5, 0))
    x2 = synth.host_x(wl, att, rows=[5], out=x0.copy())
    assert np.array_equal(x2, x1)


def test_pick_is_sorted_distinct_and_stable():
    p = synth.sample_tokens(65536, 32)
    assert len(set(p.tolist())) == 32 and np.all(np.diff(p) > 0)
    assert np.array_equal(p, synth.sample_tokens(65536, 32))
