"""Benchmark of the NSA forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload nsa_64k]

A step is one full NSA prefill forward (phi of K and V, compressed attention +
group-summed block scores + top-k, selected-block attention, sliding window +
gated combine) over the T = 65536 synthetic workload (B = 1, 64 query heads in
4 KV groups of 16, d_k = 192, d_v = 128, top-16 of 64-token blocks, window 512).
Inputs are resident in HBM when the timed region starts; L2 is flushed (a
256 MB write) before every timed step, outside its CUDA events.  Rank 0 prints
one JSON line.  With N > 1 every rank runs its own replica (the path does not
shard across GPUs); value = tokens of all ranks / max-over-ranks time.

--impl reference times the CPU oracle (the fp64 restatement of the pages in
oracle/) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import shutil
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "NSA fwd tokens/s @T=64K and % bf16 tensor peak; decode GB/s vs HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0   # the datasheet dense bf16 rate of one B200 (context for the measured peaks)
L, S, BSEL = 32, 16, 64
STAGES = ["phi_k", "phi_v", "cmp_select", "slc_attn", "swa_combine"]


# ----------------------------------------------------------------------------- work counts

def n_cmp(T):
    return 0 if T < L else (T - L) // S + 1


def nsa_flops(T, h_q, h_kv, d_k, d_v, top_k, window, B=1):
    """Algorithmic FLOPs per stage: 2*(q.k pairs)*d_k + 2*(p.v pairs)*d_v over the pairs the
    method evaluates (causal structure exact, no padding, no recomputation), plus phi."""
    t = torch.arange(T, dtype=torch.float64)
    nvis = torch.where(t < L - 1, torch.zeros_like(t), torch.clamp(torch.div(t - L + 1, S, rounding_mode="floor") + 1,
                                                                  max=n_cmp(T)))
    nb = torch.div(t, BSEL, rounding_mode="floor") + 1
    slc = torch.where(nb <= top_k, t + 1, 64.0 * (top_k - 1) + torch.remainder(t, BSEL) + 1)
    win = torch.clamp(t + 1, max=window)
    per_pair = 2.0 * (d_k + d_v) * h_q * B
    nc = n_cmp(T)
    phi_k = 2.0 * B * nc * h_kv * L * d_k * d_k
    phi_v = 2.0 * B * nc * h_kv * L * d_v * d_v
    return {"phi_k": phi_k, "phi_v": phi_v, "cmp_select": float(nvis.sum()) * per_pair,
            "slc_attn": float(slc.sum()) * per_pair, "swa_combine": float(win.sum()) * per_pair}


def moba_flops(T, H, d, block, top_k, B=1):
    """MoBA: 2*(q.k + p.v pairs)*d over the chosen past blocks and the causal own block, plus the
    unscaled q . mean-key scores over every complete past block."""
    t = torch.arange(T, dtype=torch.float64)
    J = torch.div(t, block, rounding_mode="floor")
    pairs = torch.clamp(J, max=top_k) * block + torch.remainder(t, block) + 1
    attn = float(pairs.sum()) * 2.0 * (2 * d) * H * B
    score = float(J.sum()) * 2.0 * d * H * B
    return attn, score


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples nvidia-smi every 25 ms while the timed region runs (read-only queries)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 25

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.reader = None
        self.lines = []

    def __enter__(self):
        if shutil.which("nvidia-smi"):
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", str(self.PERIOD_MS), "-i", str(self.gpu)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.reader:
            self.reader.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle timing

def cpu_workload():
    c = synth.WORKLOADS["nsa_64k"]
    return synth.nsa_inputs(c["B"], c["T"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"], seed=0)


def oracle_rate(x, n_sample, seed, threads):
    """Oracle tokens/s on the 64K workload: phi over the whole sequence, timed, plus the three
    branches on n_sample uniformly drawn query tokens, timed and scaled to all T tokens."""
    import oracle
    c = synth.WORKLOADS["nsa_64k"]
    torch.set_num_threads(threads)
    g = torch.Generator().manual_seed(seed)
    toks = sorted(torch.randint(0, c["T"], (n_sample,), generator=g).tolist())
    t0 = time.perf_counter()
    kc = oracle.compress_cache(x.k, x.w_k, L, S)
    vc = oracle.compress_cache(x.v, x.w_v, L, S)
    t_phi = time.perf_counter() - t0
    G = c["h_q"] // c["h_kv"]
    q, k, v, gates = (oracle.nsa_oracle._f64(a) for a in (x.q, x.k, x.v, x.gates))
    scale = 1.0 / math.sqrt(c["d_k"])
    t0 = time.perf_counter()
    for t in toks:
        for gi in range(c["h_kv"]):
            hs = slice(gi * G, (gi + 1) * G)
            oracle.nsa_token(q[0, t, hs], k[0, :, gi], v[0, :, gi], kc[0, :, gi], vc[0, :, gi], gates[0, t, hs], t,
                             l=L, s=S, b=BSEL, k=c["top_k"], w=c["window"], scale=scale)
    t_tok = time.perf_counter() - t0
    total = t_phi + t_tok * c["T"] / n_sample
    return c["T"] / total, {"t_phi_s": round(t_phi, 3), "t_sample_s": round(t_tok, 3), "n_sample": n_sample}


def run_reference(args, rank):
    if rank != 0:
        return
    threads = os.cpu_count() or 1
    c = synth.WORKLOADS["nsa_64k"]
    n = args.ref_sample
    rates = []
    x = cpu_workload()
    for i in range(args.warmup + args.steps):
        r, info = oracle_rate(x, n, seed=100 + i, threads=threads)
        if i >= args.warmup:
            rates.append(r)
    val = statistics.mean(rates)
    sample = (f"per step: phi over all {c['T']} tokens plus all three branches for {n} uniformly drawn query "
              f"tokens (64 heads), branch time scaled to {c['T']} tokens")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * c["T"] / val,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(c, "nsa_64k"),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(c, name):
    return {"workload": f"{name}: NSA forward B={c['B']} T={c['T']} h_q={c['h_q']} h_kv={c['h_kv']} "
                        f"d_k={c['d_k']} d_v={c['d_v']} l=32 s=16 sel_block=64 top_k={c['top_k']} "
                        f"window={c['window']} bf16",
            "global_batch": c["B"], "seq_len": c["T"], "parallelism": "replicas",
            "l2": "inputs 1.8 GB > 126 MB L2, plus a 256 MB L2 flush before every timed step (outside the events)"}


# ----------------------------------------------------------------------------- GPU arm

# DRAM bytes (read + write) per (token, KV group) item of each forward stage, from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of the T=8192 workload (B=1,
# 64 query heads, 4 KV groups: 32768 items).  These kernels' DRAM traffic is their q,
# accumulator and output rows, so it grows in proportion to the items; K/V and the
# compressed cache stay mostly in L2.  An entry goes back to None whenever its kernel
# changes, until it is captured again.
NCU_DRAM_BYTES_PER_ITEM = {
    "cmp_select": (205.892352e6 + 217.154048e6) / 32768,    # --set full capture of the three kernels
    "slc_attn": (501143552 + 228722944) / 32768,           # dram__bytes capture of the selected branch
    "swa_combine": (494.068480e6 + 118.855680e6) / 32768,   # --set full capture of the three kernels
}

# The selected branch gathers whole 64-token K/V blocks from L2 into shared memory; its
# ceiling is the L2 -> SM gather rate, measured at 67 B per clock per SM by a probe of the
# same access pattern (TMA gathers of random 64-row blocks while K/V fit in L2).
GATHER_B_PER_CLK_SM = 67.0


def run_ours(args, rank, world, local_rank):
    import block_sparse_attention_compress_b200 as nsa
    from block_sparse_attention_compress_b200.torch_ops import NSAForward

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    c = synth.WORKLOADS[args.workload]
    B, T, hq, hkv, dk, dv = c["B"], c["T"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"]
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=rank, device=dev)
    f = NSAForward(B, T, hq, hkv, dk, dv, x.w_k, x.w_v, top_k=c["top_k"], window=c["window"], device=dev)
    out = torch.empty((B, T, hq, dv), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    nstage = len(STAGES) + 1
    ev_sets = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage)] for _ in range(args.steps)]
    for evs in ev_sets:            # torch creates the CUDA event on first record
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    handles = [ctypes_array(ev) for ev in ev_sets]

    def step(i=None):
        if i is None:
            f.cfg.stage_events, f.cfg.n_stage_events = None, 0
        else:
            f.cfg.stage_events, f.cfg.n_stage_events = handles[i][0], nstage
        nsa.nsa_forward(x.q, x.k, x.v, x.gates, f.cfg, out)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(i)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    per_stage = {s: [] for s in STAGES}
    step_ms = []
    for evs in ev_sets:
        step_ms.append(evs[0].elapsed_time(evs[-1]))
        for j, s in enumerate(STAGES):
            per_stage[s].append(evs[j].elapsed_time(evs[j + 1]))
    my_ms = sum(step_ms)
    total_ms = allreduce_max(my_ms, world, dev)
    tokens = world * B * T * args.steps
    value = tokens / (total_ms / 1000.0)

    flops = nsa_flops(T, hq, hkv, dk, dv, c["top_k"], c["window"], B)
    stage_mean = {s: statistics.mean(v) for s, v in per_stage.items()}
    dom = max(stage_mean, key=stage_mean.get)
    peaks, src = load_peaks()
    ach = flops[dom] / (stage_mean[dom] * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]     # burst: each stage is timed by events inside a sub-second step
    total_flops = sum(flops.values())
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; distributions of the workload)",
        "config": workload_config(c, args.workload),
        "tflops_computed": total_flops / (statistics.mean(step_ms) * 1e-3) / 1e12,
        "frac_of_bf16_peak": total_flops / (statistics.mean(step_ms) * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "frac_of_bf16_sustained": total_flops / (statistics.mean(step_ms) * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
        "frac_of_bf16_nominal": total_flops / (statistics.mean(step_ms) * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                     "frac": ach / peak,
                     "traffic": (None if NCU_DRAM_BYTES_PER_ITEM.get(dom) is None
                                 else NCU_DRAM_BYTES_PER_ITEM[dom] * B * T * hkv),
                     "traffic_note": "DRAM bytes per launch, scaled by items from an ncu capture at T=8192",
                     "peak_source": f"{src} bf16_tflops (burst: the kernel is timed by CUDA events inside a "
                                    f"step of tens of milliseconds)"},
        "gather": slc_gather(T, hq, hkv, dk, dv, c["top_k"], stage_mean["slc_attn"], B),
        "stages_ms": {s: round(v, 4) for s, v in stage_mean.items()},
        "stage_tflops": {s: round(flops[s] / (stage_mean[s] * 1e-3) / 1e12, 1) for s in STAGES},
        "gpu_launches": len(STAGES) * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_e2e:
        result["e2e"] = run_e2e(args, f, x, out, dev, world)
    if not args.no_decode:
        del x, f, out, flush
        torch.cuda.empty_cache()
        result["decode"] = run_decode_bench(args, dev, world)
        result["gpu_launches"] += result["decode"]["gpu_launches"]
    if not args.no_moba:
        torch.cuda.empty_cache()
        result["moba"] = run_moba_bench(args, dev, world)
        result["gpu_launches"] += result["moba"]["gpu_launches"]
    if not args.no_varlen:
        torch.cuda.empty_cache()
        result["varlen"] = run_varlen_bench(args, dev, world)
        result["gpu_launches"] += result["varlen"]["gpu_launches"]
    if not args.no_backward:
        torch.cuda.empty_cache()
        result["backward"] = run_backward_bench(args, dev, world)
        result["gpu_launches"] += result["backward"]["gpu_launches"]
    if not args.no_dsa:
        torch.cuda.empty_cache()
        result["dsa"] = run_dsa_bench(args, dev, world)
        result["gpu_launches"] += result["dsa"]["gpu_launches"]
    if not args.no_phi_mlp:
        torch.cuda.empty_cache()
        result["phi_mlp"] = run_phi_mlp_bench(args, dev, world)
        result["gpu_launches"] += result["phi_mlp"]["gpu_launches"]
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        r, info = oracle_rate(cpu_workload(), args.ref_sample, seed=7, threads=os.cpu_count() or 1)
        result["cpu_baseline"] = {"value": r, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
                                  "sample": f"phi over all {T} tokens plus the three branches for "
                                            f"{args.ref_sample} uniformly drawn query tokens, scaled to {T} tokens",
                                  **info}
    if rank == 0:
        print(json.dumps(result), flush=True)


def slc_gather(T, h_q, h_kv, d_k, d_v, top_k, ms, B=1, sms=148):
    """The selected branch against the resource that bounds it: the K/V bytes it moves from L2
    into shared memory (every token u <= t of the chosen blocks, once per (token, group):
    (d_k + d_v) * 2 bytes each), per launch, against the L2 -> SM gather ceiling (the probe's
    bytes per clock per SM x SMs x the sampled SM clock is taken as 1.95 GHz)."""
    t = torch.arange(T, dtype=torch.float64)
    nb = torch.div(t, BSEL, rounding_mode="floor") + 1
    toks = torch.where(nb <= top_k, t + 1, 64.0 * (top_k - 1) + torch.remainder(t, BSEL) + 1)
    nbytes = float(toks.sum()) * B * h_kv * (d_k + d_v) * 2
    ach = nbytes / (ms * 1e-3) / 1e12
    peak = GATHER_B_PER_CLK_SM * sms * 1.95e9 / 1e12
    return {"bound": "l2_gather", "bytes_per_launch": nbytes, "achieved": ach, "peak": peak, "unit": "TB/s",
            "frac": ach / peak, "peak_source": f"probe: {GATHER_B_PER_CLK_SM} B/clk per SM x {sms} SMs x 1.95 GHz"}


def decode_bytes(idx, seqlens, h_q, d_k, d_v, window):
    """Algorithmic HBM bytes of one decode step: for every (sequence, group) the visible
    compressed keys/values, the union of the chosen blocks' tokens and the window's tokens
    (each K/V row once), plus q, gates and out."""
    B, H_kv, k = idx.shape
    row = (d_k + d_v) * 2
    total = 0
    for b in range(B):
        L = int(seqlens[b])
        t = L - 1
        nvis = 0 if L < 32 else (t - 31) // 16 + 1
        for g in range(H_kv):
            toks = set(range(max(0, t - window + 1), t + 1))
            for j in idx[b, g].tolist():
                if j >= 0:
                    toks.update(range(64 * j, min(64 * j + 64, t + 1)))
            total += nvis * row + len(toks) * row
        total += h_q * (d_k * 2 + 3 * 2 + d_v * 2)
    return total


def run_decode_bench(args, dev, world):
    """One decode step per sequence of the 32 x 65536 workload (--decode-batch sequences);
    L2 flushed before each step."""
    import block_sparse_attention_compress_b200 as nsa
    from block_sparse_attention_compress_b200.torch_ops import compress_torch
    c = synth.WORKLOADS["nsa_decode"]
    B, L, hq, hkv, dk, dv = args.decode_batch or c["B"], c["L"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"]
    d = synth.decode_inputs(B, L, hq, hkv, dk, dv, seed=0, device=dev)
    kc, vc = compress_torch(d.k_cache, d.w_k), compress_torch(d.v_cache, d.w_v)
    idx = torch.empty((B, hkv, c["top_k"]), dtype=torch.int32, device=dev)
    out = torch.empty((B, hq, dv), dtype=torch.bfloat16, device=dev)
    cfg = nsa.make_config(batch=B, seqlen=L, h_q=hq, h_kv=hkv, d_k=dk, d_v=dv, top_k=c["top_k"], window=c["window"],
                          w_cmp_k=d.w_k, w_cmp_v=d.w_v, sel_idx_out=idx)
    ws = torch.empty(nsa.nsa_workspace_size(cfg, B), dtype=torch.uint8, device=dev)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    step = lambda: nsa.nsa_decode(d.q, d.k_cache, d.v_cache, kc, vc, d.seqlens, L, d.gates, cfg, out)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    # K steps back to back between two events: the caches (5.4 GB) are far larger than L2, so
    # no step finds the previous one's rows there, and the launches queue behind each other
    # instead of each event also timing the gap before its own launch
    nrep = 4 * args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush.zero_()
    e0.record()
    for _ in range(nrep):
        step()
    e1.record()
    torch.cuda.synchronize()
    mean_ms = allreduce_max(e0.elapsed_time(e1) / nrep, world, dev)
    # the compressed-cache update a decode step makes when its new token completes a block:
    # at L = 65536 every sequence is at a block boundary, one new Kc and Vc row each
    app_ms = []
    for i in range(args.warmup + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        nsa.nsa_compress_append(d.k_cache, d.w_k, d.seqlens, kc)
        nsa.nsa_compress_append(d.v_cache, d.w_v, d.seqlens, vc)
        e1.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            app_ms.append(e0.elapsed_time(e1))
    app_us = allreduce_max(statistics.mean(app_ms), world, dev) * 1e3
    nbytes = decode_bytes(idx.cpu(), d.seqlens.cpu(), hq, dk, dv, c["window"])
    peaks, src = load_peaks()
    gbs = nbytes / (mean_ms * 1e-3) / 1e9
    return {"workload": f"nsa_decode: B={B} sequences x L={L} cache, h_q={hq} h_kv={hkv} d_k={dk} d_v={dv} "
                        f"top_k={c['top_k']} window={c['window']}, one new token each",
            "us_per_step": mean_ms * 1e3, "tokens_per_s": world * B / (mean_ms * 1e-3),
            "bytes_per_step": nbytes, "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
            "frac": gbs / peaks["hbm_gbs"], "frac_of_8tbs": gbs / 8000.0, "bound": "hbm",
            "peak_source": f"{src} hbm_gbs", "gpu_launches": 4 * args.steps + 2 * (args.warmup + args.steps),
            "timing": f"{4 * args.steps} steps back to back between two CUDA events (inputs > L2)",
            "compress_append_us": app_us,
            "compress_append_note": "nsa_compress_append for K and V (one new compressed row per sequence and "
                                    "head, 32 x 4 heads), the update a step makes every 16 tokens",
            "l2": "the caches (5.4 GB K/V, 0.34 GB compressed) exceed the 126 MB L2; one 256 MB flush before "
                  "the timed steps"}


def run_moba_bench(args, dev, world):
    """MoBA forward of the 128K-token, 32-head workload (stage times from the library's events);
    --moba-seqlen takes a shorter sequence of the same shape (for a profiler capture)."""
    import block_sparse_attention_compress_b200 as nsa
    c = synth.WORKLOADS["moba_128k"]
    B, T, H, d = 1, args.moba_seqlen or c["T"], c["h"], c["d"]
    x = synth.moba_inputs(B, T, H, d, seed=0, device=dev)
    out = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=dev)
    cfg = nsa.make_config(mode=nsa.NSA_MODE_MOBA, batch=B, seqlen=T, h_q=H, h_kv=H, d_k=d, d_v=d,
                          sel_block=c["block"], top_k=c["top_k"])
    ws = torch.empty(nsa.nsa_workspace_size(cfg), dtype=torch.uint8, device=dev)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    names = ["block_means", "select", "lists", "past_attn", "own_merge"]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    for es in evs:
        for e in es:
            e.record()
    torch.cuda.synchronize()
    handles = [ctypes_array(es) for es in evs]
    for _ in range(args.warmup):
        flush.zero_()
        cfg.stage_events, cfg.n_stage_events = None, 0
        nsa.nsa_forward(x.q, x.k, x.v, None, cfg, out)
    torch.cuda.synchronize()
    barrier(world)
    for i in range(args.steps):
        flush.zero_()
        cfg.stage_events, cfg.n_stage_events = handles[i][0], len(names) + 1
        nsa.nsa_forward(x.q, x.k, x.v, None, cfg, out)
    torch.cuda.synchronize()
    step_ms = statistics.mean(es[0].elapsed_time(es[-1]) for es in evs)
    stages = {n: statistics.mean(es[j].elapsed_time(es[j + 1]) for es in evs) for j, n in enumerate(names)}
    ms = allreduce_max(step_ms, world, dev)
    attn, score = moba_flops(T, H, d, c["block"], c["top_k"], B)
    peaks, src = load_peaks()
    name = "moba_128k" if T == c["T"] else "moba"
    return {"workload": f"{name}: B=1 T={T} heads={H} d={d} block={c['block']} top_k={c['top_k']} + own block",
            "ms_per_step": ms, "tokens_per_s": world * B * T / (ms * 1e-3),
            "tflops_computed": (attn + score) / (ms * 1e-3) / 1e12,
            "frac_of_bf16_peak": (attn + score) / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "stages_ms": {n: round(v, 4) for n, v in stages.items()},
            "gpu_launches": 6 * args.steps}


def run_varlen_bench(args, dev, world):
    """NSA forward of a packed batch of 8 sequences of different lengths, 65536 tokens in all
    (nsa_forward_varlen; stage times from the library's events)."""
    from block_sparse_attention_compress_b200.torch_ops import NSAForwardVarlen
    c = synth.WORKLOADS["nsa_varlen"]
    lengths = list(c["lengths"])
    hq, hkv, dk, dv = c["h_q"], c["h_kv"], c["d_k"], c["d_v"]
    x, cu = synth.nsa_varlen_inputs(lengths, hq, hkv, dk, dv, seed=0, device=dev)
    total = int(sum(lengths))
    f = NSAForwardVarlen(len(lengths), max(lengths), hq, hkv, dk, dv, x.w_k, x.w_v, top_k=c["top_k"],
                         window=c["window"], device=dev)
    out = torch.empty((total, hq, dv), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    nstage = len(STAGES) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage)] for _ in range(args.steps)]
    for es in evs:
        for e in es:
            e.record()
    torch.cuda.synchronize()
    handles = [ctypes_array(es) for es in evs]
    for _ in range(args.warmup):
        flush.zero_()
        f.cfg.stage_events, f.cfg.n_stage_events = None, 0
        f(x.q, x.k, x.v, x.gates, cu, out)
    torch.cuda.synchronize()
    barrier(world)
    for i in range(args.steps):
        flush.zero_()
        f.cfg.stage_events, f.cfg.n_stage_events = handles[i][0], nstage
        f(x.q, x.k, x.v, x.gates, cu, out)
    torch.cuda.synchronize()
    assert f.device_status() == 0, "a device-side wait timed out"
    step_ms = statistics.mean(es[0].elapsed_time(es[-1]) for es in evs)
    stages = {n: statistics.mean(es[j].elapsed_time(es[j + 1]) for es in evs) for j, n in enumerate(STAGES)}
    ms = allreduce_max(step_ms, world, dev)
    flops = 0.0
    for L in lengths:
        flops += sum(nsa_flops(L, hq, hkv, dk, dv, c["top_k"], c["window"], 1).values())
    peaks, _ = load_peaks()
    return {"workload": f"nsa_varlen: 8 packed sequences of lengths {lengths} ({total} tokens), h_q={hq} "
                        f"h_kv={hkv} d_k={dk} d_v={dv} top_k={c['top_k']} window={c['window']}",
            "ms_per_step": ms, "tokens_per_s": world * total / (ms * 1e-3),
            "tflops_computed": flops / (ms * 1e-3) / 1e12,
            "frac_of_bf16_peak": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "stages_ms": {n: round(v, 4) for n, v in stages.items()},
            "gpu_launches": (len(STAGES) + 1) * args.steps}   # + the check of cu_seqlens (one warp)


def run_phi_mlp_bench(args, dev, world):
    """The 64K forward with phi as the two-layer MLP (hidden width d): its two phi stages and
    the step time (stage times from the library's events)."""
    from block_sparse_attention_compress_b200.torch_ops import NSAForward
    c = synth.WORKLOADS["nsa_64k"]
    B, T, hq, hkv, dk, dv = c["B"], c["T"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"]
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=0, device=dev)
    w_k, b_k, w_k2 = synth.phi_mlp_weights(32, dk, seed=1, device=dev)
    w_v, b_v, w_v2 = synth.phi_mlp_weights(32, dv, seed=2, device=dev)
    f = NSAForward(B, T, hq, hkv, dk, dv, w_k, w_v, top_k=c["top_k"], window=c["window"], device=dev,
                   mlp=dict(b_k=b_k, w_k2=w_k2, b_v=b_v, w_v2=w_v2))
    out = torch.empty((B, T, hq, dv), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    nstage = len(STAGES) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage)] for _ in range(args.steps)]
    for es in evs:
        for e in es:
            e.record()
    torch.cuda.synchronize()
    handles = [ctypes_array(es) for es in evs]
    for _ in range(args.warmup):
        flush.zero_()
        f.cfg.stage_events, f.cfg.n_stage_events = None, 0
        f(x.q, x.k, x.v, x.gates, out)
    torch.cuda.synchronize()
    barrier(world)
    for i in range(args.steps):
        flush.zero_()
        f.cfg.stage_events, f.cfg.n_stage_events = handles[i][0], nstage
        f(x.q, x.k, x.v, x.gates, out)
    torch.cuda.synchronize()
    assert f.device_status() == 0, "a device-side wait timed out"
    step_ms = allreduce_max(statistics.mean(es[0].elapsed_time(es[-1]) for es in evs), world, dev)
    stages = {n: statistics.mean(es[j].elapsed_time(es[j + 1]) for es in evs) for j, n in enumerate(STAGES)}
    nc = (T - 32) // 16 + 1
    flops = 2.0 * B * nc * hkv * (32 * dk * dk + dk * dk + 32 * dv * dv + dv * dv)
    phi_ms = stages["phi_k"] + stages["phi_v"]
    return {"workload": "nsa_64k with phi as a two-layer MLP (GELU, hidden width d)",
            "ms_per_step": step_ms, "phi_ms": round(phi_ms, 4),
            "phi_tflops": flops / (phi_ms * 1e-3) / 1e12,
            "stages_ms": {n: round(v, 4) for n, v in stages.items()},
            "gpu_launches": (len(STAGES) + 2) * args.steps}


def dsa_flops(T, h_q, d_k, d_v, h_i, d_i, top_k, B=1):
    """Indexer: 2 * h_i * d_i per (query, key <= query) pair; attention: 2 * (d_k + d_v) per
    (query head, chosen token)."""
    pairs = T * (T + 1) // 2
    chosen = sum(min(t + 1, top_k) for t in range(T))
    return {"indexer": 2.0 * B * pairs * h_i * d_i, "attention": 2.0 * B * chosen * h_q * (d_k + d_v)}


def run_dsa_bench(args, dev, world):
    """DSA forward (lightning indexer, token-wise top-k, attention over the chosen tokens)."""
    import block_sparse_attention_compress_b200 as nsa
    c = synth.WORKLOADS["dsa_8k"]
    B, T, hq, hkv, dk, dv, hi, di, K = (c[n] for n in ("B", "T", "h_q", "h_kv", "d_k", "d_v", "h_i", "d_i", "top_k"))
    x = synth.dsa_inputs(B, T, hq, hkv, dk, dv, hi, di, seed=0, device=dev)
    cfg = nsa.make_config(mode=nsa.NSA_MODE_DSA, batch=B, seqlen=T, h_q=hq, h_kv=hkv, d_k=dk, d_v=dv, top_k=K)
    ws = torch.empty(nsa.nsa_workspace_size(cfg), dtype=torch.uint8, device=dev)
    cfg.workspace, cfg.workspace_bytes = ws.data_ptr(), ws.numel()
    out = torch.empty((B, T, hq, dv), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    names = ["select", "attention"]   # indexer scores + top-k streamed in one kernel, then attention
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    for es in evs:
        for e in es:
            e.record()
    torch.cuda.synchronize()
    handles = [ctypes_array(es) for es in evs]
    args_in = (x.q, x.k, x.v, x.q_idx, x.k_idx, x.w_idx)
    for _ in range(args.warmup):
        flush.zero_()
        cfg.stage_events, cfg.n_stage_events = None, 0
        nsa.nsa_dsa_forward(*args_in, cfg, out)
    torch.cuda.synchronize()
    barrier(world)
    for i in range(args.steps):
        flush.zero_()
        cfg.stage_events, cfg.n_stage_events = handles[i][0], len(names) + 1
        nsa.nsa_dsa_forward(*args_in, cfg, out)
    torch.cuda.synchronize()
    step_ms = allreduce_max(statistics.mean(es[0].elapsed_time(es[-1]) for es in evs), world, dev)
    stages = {n: statistics.mean(es[j].elapsed_time(es[j + 1]) for es in evs) for j, n in enumerate(names)}
    fl = dsa_flops(T, hq, dk, dv, hi, di, K, B)
    peaks, _ = load_peaks()
    return {"workload": f"dsa_8k: B={B} T={T} h_q={hq} h_kv={hkv} d_k={dk} d_v={dv}, indexer {hi} heads x {di}, "
                        f"top_k={K}",
            "ms_per_step": step_ms, "tokens_per_s": world * B * T / (step_ms * 1e-3),
            "tflops_computed": sum(fl.values()) / (step_ms * 1e-3) / 1e12,
            "frac_of_bf16_peak": sum(fl.values()) / (step_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "stages_ms": {n: round(v, 4) for n, v in stages.items()},
            "stage_tflops": {"select": round(fl["indexer"] / (stages["select"] * 1e-3) / 1e12, 1),
                             "attention": round(fl["attention"] / (stages["attention"] * 1e-3) / 1e12, 1)},
            "select_note": "the select stage computes the indexer scores six times (four radix passes, a count "
                           "and an emit); its TFLOP/s counts them once",
            "workspace_bytes": int(ws.numel()),
            "gpu_launches": len(names) * args.steps}


def run_backward_bench(args, dev, world):
    """NSA backward (nsa_backward) of the 8K workload: gradients of q, k, v, gates and phi's weights
    for the blocks a forward chose; at most 3 timed steps (about 42 ms each)."""
    import block_sparse_attention_compress_b200 as nsa
    from block_sparse_attention_compress_b200.torch_ops import NSAForward
    c = synth.WORKLOADS["nsa_8k"]
    B, T, hq, hkv, dk, dv = c["B"], c["T"], c["h_q"], c["h_kv"], c["d_k"], c["d_v"]
    x = synth.nsa_inputs(B, T, hq, hkv, dk, dv, seed=0, device=dev)
    f = NSAForward(B, T, hq, hkv, dk, dv, x.w_k, x.w_v, top_k=c["top_k"], window=c["window"], device=dev)
    f(x.q, x.k, x.v, x.gates)
    dout = torch.randn(B, T, hq, dv, device=dev).to(torch.bfloat16)
    g = dict(dq=torch.empty(B, T, hq, dk, device=dev), dk=torch.empty(B, T, hkv, dk, device=dev),
             dv=torch.empty(B, T, hkv, dv, device=dev), dgates=torch.empty(B, T, hq, 3, device=dev),
             dw_k=torch.empty(32 * dk, dk, device=dev), dw_v=torch.empty(32 * dv, dv, device=dev))

    def step():
        nsa.nsa_backward(x.q, x.k, x.v, x.gates, f.idx, dout, f.cfg, g["dq"], g["dk"], g["dv"], g["dgates"],
                         g["dw_k"], g["dw_v"])

    steps = max(1, min(args.steps, 3))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    barrier(world)
    times = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        step()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = allreduce_max(statistics.mean(times), world, dev)
    fw = nsa_flops(T, hq, hkv, dk, dv, c["top_k"], c["window"], B)
    pairs = sum(fw[s] / (2.0 * (dk + dv)) for s in ("cmp_select", "slc_attn", "swa_combine"))
    flops = 2.0 * pairs * (4 * dk + 3 * dv)   # recompute (S, P.V) + dP + dQ + dK + dV
    return {"workload": f"nsa_8k backward: B={B} T={T} h_q={hq} h_kv={hkv} d_k={dk} d_v={dv} top_k={c['top_k']} "
                        f"window={c['window']} (dq, dk, dv, dgates, dw_k, dw_v)",
            "ms_per_step": ms, "steps": steps, "tokens_per_s": world * B * T / (ms * 1e-3),
            "tflops_computed": flops / (ms * 1e-3) / 1e12, "gpu_launches": 5 * steps}


def run_e2e(args, f, x, out, dev, world):
    """Same step through the public API with inputs in pinned host memory: every step copies
    its q, k, v and gates host -> device, runs nsa_forward and copies its output device -> host,
    all inside the timed region.  As a serving loop would, the steps are pipelined on three
    streams: step i + 1's inputs go up and step i - 1's output comes down while step i computes
    (two device buffers of each; a buffer is refilled only after the step that used it is done
    with it).  The time is from the first upload to the last download."""
    import block_sparse_attention_compress_b200 as nsa
    host_in = [t.cpu().pin_memory() for t in (x.q, x.k, x.v, x.gates)]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dev_in = [[torch.empty_like(t, device=dev) for t in host_in] for _ in range(2)]
    dev_out = [out, torch.empty_like(out)]
    f.cfg.stage_events, f.cfg.n_stage_events = None, 0
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_up, s_run, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()

    def run(n):
        """n pipelined steps; returns (start, end) timing events."""
        up_done, run_done, down_done = [None] * n, [None] * n, [None] * n
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_up)
        s_run.wait_event(t0)
        s_down.wait_event(t0)
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(run_done[i - 2])   # the forward of step i - 2 has read buffer j
                for d, h in zip(dev_in[j], host_in):
                    d.copy_(h, non_blocking=True)
                up_done[i] = ev()
                up_done[i].record(s_up)
            s_run.wait_event(up_done[i])
            if i >= 2:
                s_run.wait_event(down_done[i - 2])      # output buffer j has been read back
            nsa.nsa_forward(*dev_in[j], f.cfg, dev_out[j], stream=s_run)
            run_done[i] = ev()
            run_done[i].record(s_run)
            with torch.cuda.stream(s_down):
                s_down.wait_event(run_done[i])
                host_out[j].copy_(dev_out[j], non_blocking=True)
                down_done[i] = ev()
                down_done[i].record(s_down)
        t1.record(s_down)
        return t0, t1

    run(max(2, args.warmup))
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = run(args.steps)
    torch.cuda.synchronize()
    ms = allreduce_max(t0.elapsed_time(t1), world, dev)
    tokens = world * out.shape[0] * out.shape[1] * args.steps
    return {"value": tokens / (ms / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "timing": "steps pipelined on three streams (upload of step i+1 and download of step i-1 overlap "
                      "the forward of step i); from the first upload to the last download"}


def ctypes_array(events):
    import ctypes
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p)), arr


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def allreduce_max(v, world, dev):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="nsa_64k", choices=["nsa_64k", "nsa_8k", "nsa_tiny"])
    ap.add_argument("--ref-sample", type=int, default=48)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-moba", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-phi-mlp", action="store_true")
    ap.add_argument("--no-dsa", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode step and print its line (for a profiler capture)")
    ap.add_argument("--decode-batch", type=int, default=0, help="decode sequences (default: the workload's 32)")
    ap.add_argument("--moba-only", action="store_true",
                    help="time only the MoBA forward and print its line (for a profiler capture)")
    ap.add_argument("--moba-seqlen", type=int, default=0, help="MoBA tokens (default: the workload's 131072)")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.decode_only:
            dev = torch.device("cuda", local_rank)
            torch.cuda.set_device(dev)
            res = run_decode_bench(args, dev, world)
            if rank == 0:
                print(json.dumps({"metric": METRIC, "decode": res}), flush=True)
            return
        if args.moba_only:
            dev = torch.device("cuda", local_rank)
            torch.cuda.set_device(dev)
            res = run_moba_bench(args, dev, world)
            if rank == 0:
                print(json.dumps({"metric": METRIC, "moba": res}), flush=True)
            return
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
