"""Seeded inputs for parity tests: the synthetic generator plus the margin rule.

Every token whose oracle group or expert margin is below MARGIN is re-drawn
(next attempt of its row) until all margins clear it, so that fp32 routing on
the GPU and fp64 routing in the oracle must choose the same experts. Only the
oracle decides margins; nothing here comes from the GPU path.
"""
import numpy as np

import oracle
import synth

MARGIN = 1e-4


def routed_inputs(wl, bias_mode=0, margin=MARGIN, max_rounds=64, seed=synth.SEED):
    """Returns (x bits [T,H], attempts [T], w_router, bias, oracle route dict)."""
    cfg = oracle.cfg_for(wl, bias_mode=bias_mode)
    wr = synth.host_router(wl, seed)
    b = synth.host_bias(wl, seed)
    attempts = np.zeros(wl.T, dtype=np.int32)
    x = synth.host_x(wl, attempts, seed=seed)
    r = oracle.route(cfg, x, wr, b)
    for _ in range(max_rounds):
        bad = np.nonzero(r["margins"].min(axis=1) < margin)[0]
        if bad.size == 0:
            return x, attempts, wr, b, r
        attempts[bad] += 1
        synth.host_x(wl, attempts, rows=bad, out=x, seed=seed)
        rb = oracle.route(cfg, x[bad], wr, b)
        for k in r:
            r[k][bad] = rb[k]
    raise RuntimeError(f"margin re-draw did not converge for {wl.name}")


def expert_tables(wl, experts, seed=synth.SEED):
    """Host weights of the listed experts: ({e: w13}, {e: w2})."""
    w13, w2 = {}, {}
    for e in sorted(set(int(v) for v in np.ravel(experts))):
        w13[e] = synth.host_expert_w13(wl, e, seed)
        w2[e] = synth.host_expert_w2(wl, e, seed)
    return w13, w2
