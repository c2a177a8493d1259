"""Benchmark of the Beam MoE block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|decode|...]
                    [--impl ours|reference] [--no-cpu-baseline]
                    [--format bf16|nvfp4] [--bias-mode 0|1] [--router-tc] [--replay]

A step is one whole block forward (router GEMM, top-k, scan, permute, gate/up
grouped GEMM, down grouped GEMM, combine) over one batch of T synthetic tokens
with Beam's shapes: hidden 5120, 256 SwiGLU experts of intermediate 2560 in 8
groups of 32, top-4 groups, top-8 experts, routed scale 2.5. By default one
run times all four Beam workloads on one set of expert weights: decode
(T = 64), prefill (T = 4096), skewed routing (T = 16384) and the long prefill
chunk (T = 65536, clustered inputs). The long chunk, the largest configuration
that fits one GPU, is the line's headline (`value`, `roofline`, `e2e`,
`cpu_baseline`); the other three sit under `workloads`, each with its own
`roofline`, `e2e` and `clocks`. Weights and inputs are synthetic and seeded
(bf16 experts N(0, 0.02), fp32 router N(0, 1/sqrt(5120)), bf16 activations
N(0, 1)); they are resident in HBM before timing starts. The L2 cache is
flushed (256 MB write) before every timed step, outside the timed interval.
Timing: CUDA events on the launching stream around each step, summed over K
steps, max over ranks.

With N GPUs (torchrun, one process per GPU) every rank holds all experts and
runs its own batch of T tokens: the block is data-parallel over tokens with
no exchange, so scaling is weak and the only collective is the max of the
timings.

--format nvfp4 times the same block with NVFP4 experts and activations (4-bit
E2M1 codes, one E4M3 scale per 16 elements, an fp32 scale per tensor) on the
block-scaled FP4 tensor cores; its tensor peak is 4x the measured bf16 peak.

--impl reference times the fp64 CPU oracle (the reference arm of this
repository) on a bounded sample of the headline workload on the host cores.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

import synth

METRIC = "MoE-block tokens/s; achieved TFLOP/s or HBM GB/s as % of B200 roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES = ("router_gemm", "router_topk", "scan", "permute", "gateup_gemm", "down_gemm", "combine")
# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the gate/up
# kernel, from ncu captures of small cases in the same regime as a workload,
# scaled to a full launch by the unit named: touched experts at decode (the
# weights dominate; about 2 rows per expert in both), assignments for the long
# chunk (2048 rows per expert in both). A record is valid only while the
# sources of the kernel that runs hash to `sha256`; any edit voids it.
GATEUP_TRAFFIC = {
    "decode": {"per": "touched_expert", "bytes": 52568082,
               "sources": ("sparse_moe_layer_beam_b200/csrc/grouped_gemm.cu",
                           "sparse_moe_layer_beam_b200/csrc/grouped_gemm.cuh",
                           "sparse_moe_layer_beam_b200/csrc/sm100.cuh"),
               "sha256": "725f4dd9c7269a71650243ecd4c2c23c391aabfe12ab9e3dcb7a997760ff1606"},
    "long": {"per": "assignment", "bytes": 42326,
             "sources": ("sparse_moe_layer_beam_b200/csrc/grouped_gemm_2sm.cu",
                         "sparse_moe_layer_beam_b200/csrc/grouped_gemm.cuh",
                         "sparse_moe_layer_beam_b200/csrc/sm100.cuh"),
             "sha256": "cebdcde26c340ca125578851fff5f185362925fc332250afcd3d3b44e9d9ac43"},
}


def sources_sha256(paths):
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gateup_traffic(wl, alg):
    """Estimated DRAM bytes of one gate/up launch, or None without a valid record."""
    rec = GATEUP_TRAFFIC.get(wl.name)
    if rec is None or rec["bytes"] is None or sources_sha256(rec["sources"]) != rec["sha256"]:
        return None
    units = alg["touched_experts"] if rec["per"] == "touched_expert" else wl.T * wl.K
    return rec["bytes"] * units


def host_chunking(T, nvfp4):
    """How the host-buffer entry points split T tokens (the rule of
    include/beam_moe.h, BEAM_MOE_HOST_CHUNK): one chunk below two chunks'
    worth, else chunks of BEAM_MOE_HOST_CHUNK, twice that for bf16 batches of
    at least eight."""
    import sparse_moe_layer_beam_b200 as bm  # constants only; the library loads on first call

    c = bm.HOST_CHUNK
    if T < 2 * c:
        return "one chunk"
    size = 2 * c if (not nvfp4 and T >= 8 * c) else c
    n = -(-T // size)
    return f"{n} chunks of {size} tokens, copies overlapped"


def describe(wl):
    extra = ""
    if wl.n_hot:
        extra = f", router bias +{wl.hot_bias} on {wl.n_hot} experts"
    if wl.n_centres:
        extra = f", clustered inputs ({wl.n_centres} centres + N(0,{wl.sigma_x}) noise)"
    return (f"Beam MoE block {wl.name}: T={wl.T}, hidden {wl.H}, {wl.E} SwiGLU experts of "
            f"intermediate {wl.I} in {wl.G} groups of {wl.E // wl.G}, top-{wl.Gk} groups, "
            f"top-{wl.K} experts, scale {wl.scale}{extra}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(wl, counts, fmt="bf16"):
    """Algorithmic work of one forward with these routed counts.

    FLOPs: 6 H I per assignment (tensor cores) + 2 H E per token (FP32 router).
    Bytes: 3 H I x b per touched expert (b = 2 for bf16; 0.5625 for NVFP4: a
    4-bit code plus one E4M3 scale per 16 elements), router weights, x and out.
    gate/up kernel bytes: 2 I H x b per touched expert + its input rows + its
    output rows (bf16 rows, or NVFP4 rows at 0.5625 bytes per element).
    """
    touched = int(np.count_nonzero(counts))
    A = wl.T * wl.K
    b = 2.0 if fmt == "bf16" else 0.5625
    return {
        "touched_experts": touched,
        "expert_flops": 6.0 * wl.H * wl.I * A,
        "router_flops": 2.0 * wl.H * wl.E * wl.T,
        "block_bytes": touched * 3.0 * wl.H * wl.I * b + wl.E * wl.H * 4 + 2 * wl.T * wl.H * 2,
        "gateup_bytes": touched * 2.0 * wl.I * wl.H * b + A * wl.H * b + A * wl.I * b,
        "gateup_flops": 4.0 * wl.H * wl.I * A,
    }


def roofline(alg, gate_ms, ms_step, peaks, peak_kind, nvfp4):
    """The line's `roofline` (the gate/up kernel) and `block` objects.

    gate_ms: the gate/up kernel's mean event time (None when the entry point
    records no per-stage events). The tensor peak is the burst figure for
    steps under 10 ms and the sustained (power-capped) one from 10 ms on; for
    NVFP4 it is 4 x the measured bf16 peak (the nominal dense FP4:BF16 ratio).
    The kernel's bound follows from its algorithmic bytes and flops: whichever
    takes longer at its peak."""
    if nvfp4:
        peaks = dict(peaks, bf16_tflops=4 * peaks["bf16_tflops"],
                     bf16_tflops_sustained=4 * peaks.get("bf16_tflops_sustained",
                                                         peaks["bf16_tflops"]))
    sustained = ms_step >= 10.0 and "bf16_tflops_sustained" in peaks
    tc_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    t_hbm = alg["gateup_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = alg["gateup_flops"] / (tc_peak * 1e12)
    ok = gate_ms is not None and gate_ms == gate_ms and gate_ms > 0
    if t_hbm >= t_tc:
        achieved = alg["gateup_bytes"] / (gate_ms / 1000.0) / 1e9 if ok else None
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = alg["gateup_flops"] / (gate_ms / 1000.0) / 1e12 if ok else None
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                "peak_kind": "sustained" if sustained else "burst"}
    roof["frac"] = None if roof["achieved"] is None else roof["achieved"] / roof["peak"]
    roof["traffic"] = None
    roof["algorithmic_bytes"] = alg["gateup_bytes"]
    roof["kernel"] = "gateup_grouped_gemm_nvfp4" if nvfp4 else "gateup_grouped_gemm"
    if nvfp4:
        roof["peak_note"] = "dense FP4 tensor peak = 4 x measured bf16 (nominal ratio)"
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" \
        else "fallback"
    block_s = ms_step / 1000.0
    block = {"hbm_gbs": alg["block_bytes"] / block_s / 1e9,
             "hbm_frac": alg["block_bytes"] / block_s / 1e9 / peaks["hbm_gbs"],
             "tflops": alg["expert_flops"] / block_s / 1e12,
             "tensor_frac": alg["expert_flops"] / block_s / 1e12 / tc_peak,
             "tensor_frac_of_burst": alg["expert_flops"] / block_s / 1e12 / peaks["bf16_tflops"],
             "tensor_peak_kind": "sustained" if sustained else "burst",
             "touched_experts": alg["touched_experts"]}
    return roof, block


class ClockSampler:
    """nvidia-smi samples of clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------------ reference arm

class OracleSample:
    """The fp64 CPU oracle (routing, experts and combine) on n sampled tokens of
    a workload. The expert weights of the sampled tokens are generated once,
    before any timed call."""

    def __init__(self, wl, n_tokens, seed=synth.SEED):
        import oracle

        self.oracle = oracle
        self.cfg = oracle.cfg_for(wl)
        tokens = synth.sample_tokens(wl.T, n_tokens, seed)
        self.n = len(tokens)
        self.x = synth.host_x(wl, seed=seed)[tokens]
        self.wr = synth.host_router(wl, seed)
        self.b = synth.host_bias(wl, seed)
        ids = oracle.route(self.cfg, self.x, self.wr, self.b)["ids"]
        self.w13 = {int(e): synth.host_expert_w13(wl, int(e), seed) for e in np.unique(ids)}
        self.w2 = {int(e): synth.host_expert_w2(wl, int(e), seed) for e in np.unique(ids)}
        self.threads = min(self.n, int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)))
        self.desc = (f"{self.n} of the {wl.T} tokens (seeded sample): full routing and all "
                     f"{wl.K} experts per token in fp64; expert weights generated before timing")

    def run(self):
        """Returns (tokens/s, seconds) of one timed oracle pass over the sample."""
        t0 = time.perf_counter()
        r = self.oracle.route(self.cfg, self.x, self.wr, self.b)
        self.oracle.experts(self.cfg, self.x, r["ids"], r["weights"], self.w13, self.w2)
        dt = time.perf_counter() - t0
        return self.n / dt, dt


def oracle_sample_size(wl):
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return max(1, min(wl.T, cores, 16))


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sample = OracleSample(wl, oracle_sample_size(wl))
    vals = []
    for i in range(args.warmup + args.steps):
        v, dt = sample.run()
        if i >= args.warmup:
            vals.append((v, dt))
    value = sample.n * len(vals) / sum(dt for _, dt in vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.mean(dt for _, dt in vals),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": describe(wl), "T": wl.T, "sample_tokens_per_step": sample.n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": sample.threads,
                         "kind": "oracle", "sample": sample.desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------------------- ours

def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (the one collective of a run)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def rank_seed(rank):
    """Seed of a rank's token batch; all ranks share the expert weights (seed 0)."""
    return synth.SEED + rank


class Experts:
    """The expert weights every workload of one run shares (seed 0), on the
    device: bf16 W13 / W2, or NVFP4 codes and scales."""

    def __init__(self, wl, fmt, dev, st):
        import torch

        import sparse_moe_layer_beam_b200 as bm

        self.nvfp4 = fmt == "nvfp4"
        if self.nvfp4:
            self.c13 = torch.empty(wl.w13_elems // 2, dtype=torch.uint8, device=dev)
            self.s13 = torch.empty(wl.w13_elems // 16, dtype=torch.uint8, device=dev)
            self.c2 = torch.empty(wl.w2_elems // 2, dtype=torch.uint8, device=dev)
            self.s2 = torch.empty(wl.w2_elems // 16, dtype=torch.uint8, device=dev)
            synth.dev_w13_nvfp4(wl, self.c13.data_ptr(), self.s13.data_ptr(), st)
            synth.dev_w2_nvfp4(wl, self.c2.data_ptr(), self.s2.data_ptr(), st)
            self.experts = bm.nvfp4_experts(self.c13, self.s13, self.c2, self.s2,
                                            synth.NVFP4_WEIGHT_SCALE, synth.NVFP4_WEIGHT_SCALE,
                                            synth.NVFP4_ACT_SCALE, synth.NVFP4_ACT_SCALE)
            self.w13 = self.w2 = None
        else:
            self.w13 = torch.empty(wl.w13_elems, dtype=torch.int16, device=dev)
            self.w2 = torch.empty(wl.w2_elems, dtype=torch.int16, device=dev)
            synth.dev_w13(wl, self.w13.data_ptr(), st)
            synth.dev_w2(wl, self.w2.data_ptr(), st)
            self.experts = None
        self.wr = torch.from_numpy(synth.host_router(wl)).to(dev)


def measure(args, wl, ex, dev, stream, rank, world, local):
    """Times W warm-up and K timed steps of one workload (device events on the
    launching stream, L2 flushed before each step), then the same number of
    end-to-end steps through the host-buffer entry point. Returns the
    workload's part of the JSON line (max over ranks) and the routed counts."""
    import torch
    import torch.distributed as dist

    import sparse_moe_layer_beam_b200 as bm

    st = stream.cuda_stream
    nvfp4 = ex.nvfp4
    cfg = bm.beam_cfg(wl.H, wl.I, wl.E, wl.G, wl.Gk, wl.K, wl.renormalize, args.bias_mode,
                      wl.scale, router_tc=args.router_tc)
    bias = synth.host_bias(wl)
    b = None if bias is None else torch.from_numpy(bias).to(dev)
    x = torch.empty((wl.T, wl.H), dtype=torch.int16, device=dev)
    synth.dev_x(wl, x.data_ptr(), st, seed=rank_seed(rank))
    out = torch.empty((wl.T, wl.H), dtype=torch.int16, device=dev)
    counts = torch.zeros(wl.E, dtype=torch.int32, device=dev)
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T,
                                                bm.OP_FORWARD_NVFP4 if nvfp4 else bm.OP_FORWARD),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    lay = bm.beam_moe_workspace_layout(cfg, wl.T)

    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device=dev)
    wts = torch.empty((wl.T, wl.K), dtype=torch.float32, device=dev)
    if args.replay:  # record the routes once; the timed steps replay them
        bm.beam_moe_forward(cfg, x, ex.wr, b, ex.w13, ex.w2, out, ws, ids, wts, counts, stream=st)

    def step(trace=None):
        if nvfp4:
            bm.beam_moe_forward_nvfp4(cfg, x, ex.wr, b, ex.experts, out, ws, expert_counts=counts,
                                      stream=st, trace=trace)
        elif args.replay:
            bm.beam_moe_forward_routed(cfg, x, ids, wts, ex.w13, ex.w2, out, ws, counts, stream=st)
        elif trace is None:
            bm.beam_moe_forward(cfg, x, ex.wr, b, ex.w13, ex.w2, out, ws, expert_counts=counts,
                                stream=st)
        else:
            bm.beam_moe_forward_traced(cfg, x, ex.wr, b, ex.w13, ex.w2, out, ws, trace,
                                       expert_counts=counts, stream=st)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    flags = bm.beam_moe_check(ws, st)
    if flags:
        raise SystemExit(f"{wl.name}: device status flags {flags:#x} after warm-up")

    trace = None if args.replay else bm.Trace(args.steps)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        step(trace)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = sum(a.elapsed_time(c) for a, c in ev)
    stage_ms = (np.full((args.steps, len(STAGES)), np.nan) if trace is None
                else np.array(trace.read()))  # [steps][stages]
    if trace is not None:
        trace.close()
    flags = bm.beam_moe_check(ws, st)
    if flags:
        raise SystemExit(f"{wl.name}: device status flags {flags:#x} in the timed region")

    # End to end with host buffers: pinned x in, out back. The forward goes
    # through beam_moe_forward_host (chunked, copies overlapped with compute);
    # replayed routes have no host-buffer entry point, so that line copies
    # around beam_moe_forward_routed.
    x_host = x.cpu().pin_memory()
    out_host = torch.empty_like(out, device="cpu").pin_memory()
    ws_h = None
    if not args.replay:
        del ws
        op_h = bm.OP_FORWARD_NVFP4_HOST if nvfp4 else bm.OP_FORWARD_HOST
        ws_h = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T, op_h), dtype=torch.uint8,
                           device=dev)

    def e2e_step():
        if nvfp4:
            bm.beam_moe_forward_nvfp4_host(cfg, x_host, ex.wr, b, ex.experts, out_host, ws_h,
                                           stream=st)
        elif not args.replay:
            bm.beam_moe_forward_host(cfg, x_host, ex.wr, b, ex.w13, ex.w2, out_host, ws_h,
                                     stream=st)
        else:
            x.copy_(x_host, non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)

    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    for i in range(args.warmup + args.steps):
        flush.zero_()
        j = i - args.warmup
        if j >= 0:
            e2e_ev[j][0].record(stream)
        e2e_step()
        if j >= 0:
            e2e_ev[j][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(c) for a, c in e2e_ev)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)
    ms_step = total_ms / args.steps
    tokens = wl.T * world
    value = tokens / (ms_step / 1000.0)
    e2e_value = tokens / (e2e_ms / args.steps / 1000.0)

    routed = counts.cpu().numpy()
    alg = algorithmic(wl, routed, args.format)
    peaks, peak_kind = load_peaks()
    stage_mean = {n: float(stage_ms[:, i].mean()) for i, n in enumerate(STAGES)}
    gate_ms = float(stage_ms[:, 4].mean()) if trace is not None else float("nan")
    roof, block = roofline(alg, None if args.replay else gate_ms, ms_step, peaks, peak_kind,
                           nvfp4)
    # the recorded DRAM traffic belongs to the bf16 gate/up kernel only
    roof["traffic"] = None if nvfp4 else gateup_traffic(wl, alg)
    # router GEMM (plus the weight split on tensor cores), top-k, scan,
    # permute, gate/up, down, combine; replayed routes: the route copy, scan,
    # permute, gate/up, down, combine; the light experts' one-CTA gate/up and
    # down after the CTA-pair ones
    per_step = ((6 if args.replay else (8 if lay.router_tc else 7))
                + (2 if lay.light_rows and not nvfp4 else 0))
    part = {
        "value": value, "ms_per_step": ms_step,
        "config": {"workload": describe(wl) + (" [routes replayed]" if args.replay else "")
                   + (" [NVFP4 experts and activations]" if nvfp4 else "")
                   + (" [selection-only bias]" if args.bias_mode == 1 else "")
                   + (" [router GEMM on tensor cores]" if lay.router_tc else ""),
                   "T": wl.T, "tokens_per_rank": wl.T,
                   "l2": "flushed before every timed step (256 MB write, outside the events)",
                   "router": "tensor cores (exact bf16 split)" if lay.router_tc
                   else "FP32 FMA on CUDA cores",
                   "parallelism": f"replicas x{world} (token data parallel, no exchange)"},
        "roofline": roof,
        "block": block,
        "stages_ms": None if args.replay else stage_mean,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": wl.T * wl.H * 2,
                "d2h_bytes_per_step": wl.T * wl.H * 2,
                "call": ("copies around beam_moe_forward_routed" if args.replay else
                         ("beam_moe_forward_nvfp4_host" if nvfp4 else "beam_moe_forward_host")
                         + f" ({host_chunking(wl.T, nvfp4)})")},
        "gpu_launches": per_step * args.steps,
        "clocks": clk,
    }
    return part


def run_ep(args, wl):
    """Expert parallelism over the N ranks (one per GPU; N = 1 runs the same
    phases on one GPU): each rank holds E / N experts, routes its own T
    tokens, exchanges workspaces once through CUDA IPC, and per step
    all-gathers the counts (NCCL), plans on the host, dispatches by peer
    stores, runs its experts (y rows stored back into their sources) and
    combines. No barrier between dispatch and experts: the gate/up GEMM waits
    for each expert's rows on the arrival counters the dispatch increments;
    one barrier after the experts."""
    import datetime

    import torch
    import torch.distributed as dist

    import sparse_moe_layer_beam_b200 as bm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if wl.E % world:
        raise SystemExit(f"{wl.E} experts do not split over {world} ranks")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    stream = torch.cuda.current_stream()
    st = stream.cuda_stream
    ex = Experts(wl, "bf16", dev, st)
    cfg = bm.beam_cfg(wl.H, wl.I, wl.E, wl.G, wl.Gk, wl.K, wl.renormalize, args.bias_mode,
                      wl.scale, router_tc=args.router_tc)
    El = wl.E // world
    w13 = ex.w13.data_ptr() + rank * El * 2 * wl.I * wl.H * 2
    w2 = ex.w2.data_ptr() + rank * El * wl.H * wl.I * 2
    bias = synth.host_bias(wl)
    b = None if bias is None else torch.from_numpy(bias).to(dev)
    x = torch.empty((wl.T, wl.H), dtype=torch.int16, device=dev)
    synth.dev_x(wl, x.data_ptr(), st, seed=rank_seed(rank))
    out = torch.empty((wl.T, wl.H), dtype=torch.int16, device=dev)
    ep = bm.ep_cfg(world, rank, wl.T, wl.T * world * min(wl.K, El))
    ws = torch.empty(bm.beam_moe_ep_workspace_size(cfg, ep), dtype=torch.uint8, device=dev)
    counts = torch.empty(wl.E, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if world > 1:
        peers = bm.EpPeers(ep, ws, bm.torch_gather())
        gathered = [torch.empty_like(counts) for _ in range(world)]
        ones = torch.ones(1, device=dev)
    else:
        peers = bm.EpPeers(ep, ws, lambda blob: [blob], export=lambda w: b"self")
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.all_reduce(ones)  # stream-ordered: every rank's earlier work is done

    def step():
        bm.beam_moe_ep_route(cfg, ep, x, ex.wr, b, counts, ws, stream=st)
        if world > 1:
            dist.all_gather(gathered, counts)
            counts_all = torch.stack(gathered).cpu().numpy()
        else:
            counts_all = counts.cpu().numpy()[None]
        send_base, recv_counts, _ = bm.beam_moe_ep_plan(cfg, ep, counts_all)
        bm.beam_moe_ep_dispatch(cfg, ep, x, torch.from_numpy(send_base).to(dev, non_blocking=True),
                                peers.ptrs, ws, stream=st)
        bm.beam_moe_ep_experts(cfg, ep, recv_counts, w13, w2, peers.ptrs, ws, stream=st)
        barrier()
        bm.beam_moe_ep_combine(cfg, ep, wl.T, out, ws, stream=st)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    if bm.beam_moe_check(ws, st):
        raise SystemExit("device status flags after warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    flags = bm.beam_moe_check(ws, st)
    if flags:
        raise SystemExit(f"device status flags {flags:#x} in the timed region")
    total_ms = max_over_ranks([sum(a.elapsed_time(c) for a, c in ev)], dev)[0]
    ms_step = total_ms / args.steps
    value = wl.T * world / (ms_step / 1000.0)
    alg = algorithmic(wl, counts.cpu().numpy(), "bf16")
    peaks, peak_kind = load_peaks()
    _, block = roofline(alg, None, ms_step, peaks, peak_kind, False)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(wl) + " [expert parallel]", "T": wl.T,
                   "tokens_per_rank": wl.T, "experts_per_rank": El,
                   "l2": "flushed before every timed step (256 MB write, outside the events)",
                   "parallelism": f"expert parallel x{world}: peer-store dispatch and return "
                                  "through CUDA IPC, NCCL all-gather of counts"},
        "roofline": None, "block": block, "clocks": clk,
        # router GEMM, top-k, scan, dispatch, gate/up, down (+ the return copy
        # when the down GEMM runs on single CTAs, below 64 rows per expert),
        # combine; the tensor-core router adds its weight split
        "gpu_launches": (7 + (1 if wl.T * world * wl.K / wl.E < 64 else 0)
                         + (1 if args.router_tc else 0)) * args.steps,
    }
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    peers.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_route_only(args, wl):
    """Routing alone (beam_moe_route: router GEMM, top-k and the per-expert
    counts) on one GPU, with no expert weights allocated: the router's own
    throughput, against the FP32 ALU peak (2 H E FLOP per token of FMAs)."""
    import torch

    import sparse_moe_layer_beam_b200 as bm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    st = stream.cuda_stream
    cfg = bm.beam_cfg(wl.H, wl.I, wl.E, wl.G, wl.Gk, wl.K, wl.renormalize, args.bias_mode,
                      wl.scale, router_tc=args.router_tc)
    wr = torch.from_numpy(synth.host_router(wl)).to(dev)
    bias = synth.host_bias(wl)
    b = None if bias is None else torch.from_numpy(bias).to(dev)
    x = torch.empty((wl.T, wl.H), dtype=torch.int16, device=dev)
    synth.dev_x(wl, x.data_ptr(), st)
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device=dev)
    w = torch.empty((wl.T, wl.K), dtype=torch.float32, device=dev)
    counts = torch.empty(wl.E, dtype=torch.int32, device=dev)
    ws = torch.empty(bm.beam_moe_workspace_size(cfg, wl.T, bm.OP_ROUTE), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        bm.beam_moe_route(cfg, x, wr, b, ids, w, counts, ws, stream=st)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(0)
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        bm.beam_moe_route(cfg, x, wr, b, ids, w, counts, ws, stream=st)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if bm.beam_moe_check(ws, st):
        raise SystemExit("device status flags in the timed region")
    ms = sum(a.elapsed_time(c) for a, c in ev) / args.steps
    flops = 2.0 * wl.H * wl.E * wl.T
    lay = bm.beam_moe_workspace_layout(cfg, wl.T, bm.OP_ROUTE)
    line = {
        "metric": "router tokens/s (beam_moe_route)", "value": wl.T / (ms / 1000.0),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": describe(wl) + " [routing only]", "T": wl.T,
                   "router": "tensor cores (exact bf16 split)" if lay.router_tc
                   else "FP32 FMA on CUDA cores", "router_splits": lay.router_splits,
                   "l2": "flushed before every timed step (256 MB write, outside the events)"},
        "router_tflops": flops / (ms / 1000.0) / 1e12,
        "gpu_launches": (4 if lay.router_tc else 3) * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


# The default run times every Beam workload; the line's headline is the last
# (the long prefill chunk, the largest configuration that fits one GPU).
DEFAULT_WORKLOADS = ("decode", "prefill", "skewed", "long")


def run_ours(args, wls):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    stream = torch.cuda.current_stream()
    # all ranks hold the same experts (seed 0); each rank routes its own tokens
    ex = Experts(wls[-1], args.format, dev, stream.cuda_stream)
    parts = {}
    for wl in wls:
        parts[wl.name] = measure(args, wl, ex, dev, stream, rank, world, local)
        torch.cuda.empty_cache()
    head_wl = wls[-1]
    head = parts.pop(head_wl.name)
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4" if ex.nvfp4 else "bf16", "data": "synthetic",
    }
    line.update({k: v for k, v in head.items() if k not in ("value", "ms_per_step")})
    if parts:
        line["workloads"] = parts
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(head_wl, oracle_sample_size(head_wl))
        v, dt = sample.run()
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": sample.threads,
                                "kind": "oracle", "sample": sample.desc, "seconds": dt}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all", choices=["all"] + sorted(synth.WORKLOADS),
                    help="all (default): decode, prefill, skewed and long, the last one the "
                         "headline; or one workload")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bias-mode", type=int, default=0, choices=[0, 1],
                    help="0: router bias on the logits; 1: on the choice scores only")
    ap.add_argument("--format", default="bf16", choices=["bf16", "nvfp4"],
                    help="expert weight / activation format of the timed forward")
    ap.add_argument("--router-tc", action="store_true",
                    help="opt in to the router GEMM on tensor cores (exact bf16 split)")
    ap.add_argument("--replay", action="store_true",
                    help="time the expert path with recorded routes (beam_moe_forward_routed)")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the N ranks (one workload, bf16)")
    ap.add_argument("--route-only", action="store_true",
                    help="time beam_moe_route alone on one workload (no expert weights)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (small profiling captures only)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override the expert count, 8 groups kept (small profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.replay and args.format != "bf16":
        raise SystemExit("--replay times the bf16 routed entry point only")
    names = DEFAULT_WORKLOADS if args.workload == "all" else (args.workload,)
    wls = []
    for name in names:
        wl = synth.workload(name)
        if args.tokens is not None:
            wl = wl.with_T(args.tokens)
        if args.experts is not None:
            import dataclasses
            wl = dataclasses.replace(wl, name=f"{wl.name} (E={args.experts})", E=args.experts)
        wls.append(wl)
    if args.impl == "reference":
        return run_reference(args, wls[-1])
    if args.route_only:
        if len(wls) != 1 or args.gpus != 1:
            raise SystemExit("--route-only times one workload on one GPU")
        return run_route_only(args, wls[0])
    if args.ep:
        if len(wls) != 1 or args.format != "bf16" or args.replay:
            raise SystemExit("--ep times one bf16 workload (--workload decode, ...)")
        return run_ep(args, wls[0])
    return run_ours(args, wls)


if __name__ == "__main__":
    sys.exit(main())
