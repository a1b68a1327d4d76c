#!/usr/bin/env python3
"""Benchmark of the gated window-attention layer (ZGCM-1) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload swa16k]

A step is one pass of the whole hot path: forward + backward of one gated attention layer
over one batch of seeded synthetic inputs already resident in HBM.  The default workload
is the 16K gated sliding-window layer: B=4 sequences x S=16384 tokens, 32 query / 8 KV
heads, head dim 128, window 128 (65,536 tokens per step per GPU).  Under torchrun each
rank runs its own batch (independent sequences, no collective on the data path): weak
scaling, value = tokens of all ranks / max-over-ranks device time.

Prints ONE JSON line (rank 0).  --impl reference times the fp64 CPU oracle instead (rank 0
only; a bounded sample of the same workload per step).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated SWA fwd+bwd tokens/s & % of roofline, 16K seq, GQA 32/8, d=128, 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    # name: (B, S, window, backward?)
    "swa16k": (4, 16384, 128, True),
    "global64k": (1, 65536, 65536, True),
    "swa256k_fwd": (1, 262144, 128, False),
    "global256k_fwd": (1, 262144, 262144, False),
    "tiny_fwd": (1, 1024, 128, False),
    "swa16k_b1_fwd": (1, 16384, 128, False),
    "swa16k_b1": (1, 16384, 128, True),
    "global8k": (1, 8192, 8192, True),      # small global case (profiling captures)
    # one sliding (W=128) and one global (W=S) layer on the same inputs, reported with the
    # 5:1 sliding:global weighted time per layer of the model's layer pattern
    "mix256k_fwd": (1, 262144, 128, False),
}
LAYER_MIX = {"mix256k_fwd": ((128, 5), (None, 1))}   # (window or None = global, weight)
HQ, HKV, D = 32, 8, 128


# ---------------------------------------------------------------- ranks (one process per GPU)
#
# Sequences are independent problems, so the ranks share no data: each draws its own batch
# (seed = rank) and the only cross-rank traffic is the timing reduction below.

def rank_env():
    """(world, rank, local_rank) from the launcher's environment (1, 0, 0 without one)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank, the same on every run."""
    return rank


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over all ranks (every rank receives it); x itself when world == 1."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


def pairs(S: int, W: int) -> int:
    """Visible (i, j) pairs per (batch, head): sum_i min(i+1, W)."""
    if W >= S:
        return S * (S + 1) // 2
    return W * S - W * (W - 1) // 2


def work(B, S, W, bwd, saved=False):
    """Masked FLOPs and algorithmic HBM bytes of one step (and of each dominant kernel).
    `saved`: the forward keeps q~, k~ and the rows' inverse RMS for the backward."""
    npair = pairs(S, W) * B * HQ
    tok = B * S
    qb = tok * HQ * D * 2            # q, g, out, dout, dq, dg (bf16 [B,S,Hq,D])
    kb = tok * HKV * D * 2           # k, v, dk, dv
    lse = tok * HQ * 4
    fwd_bytes = 2 * qb + 2 * kb + qb + lse               # read q,k,v,g; write out, lse
    fwd_flops = 4 * D * npair
    bwd_bytes = 4 * qb + 2 * kb + lse + 2 * qb + 2 * kb  # read q,k,v,g,out,dout,lse; write dq,dk,dv,dg
    bwd_flops = 10 * D * npair
    # per kernel of this build: (algorithmic bytes = each input read once and each output
    # written once at its stored type, masked FLOPs of the products the kernel's job needs)
    # a forward that keeps its activations also writes q~ fp16 and each q and k row's inverse RMS
    keep = (qb + tok * HQ * 4 + tok * HKV * 4) if saved else 0
    kernels = {
        # q, k, v, g -> out, lse (keys normalised in shared memory); in the training pair it
        # reads q~ and k~ fp16 (same sizes) that the two preparation kernels wrote before it
        "fwd_strip_kernel": (fwd_bytes, fwd_flops),
        "fwd_tc_kernel": (fwd_bytes + keep, fwd_flops),
        # tcgen05 forwards: q, K~16 (fp16, prepared from k by fwd_prep_k_kernel), v, g -> out, lse
        "fwd_glob_tc_kernel": (fwd_bytes + keep, fwd_flops),
        # tcgen05 backward: gate pass dout, g, out -> dg, dA16 (fp16), 2^-e and max|dout| per row;
        # Q~16, K~16, V16, dA16, lse, 2^-e, raw q (RMSNorm backward) -> dq, Delta ; S, dP, dQ  |
        # Q~16, K~16, V16, dA16, lse, Delta, 2^-e, max|dout|, raw k -> dk, dv ; S, dP, dV, dK
        "bwd_gate_kernel": (5 * qb + 2 * lse, 0),
        # k, v -> K~, V fp16 (+ per-row inverse RMS and v norm, per-tile V scale); q -> Q~ fp16
        "bwd_prep_kv_kernel": (4 * kb + kb // D, 0),
        "bwd_prep_q_kernel": (2 * qb + qb // (2 * D), 0),
        # given the forward's q~, k~: v -> V fp16 (+ v norm per row, V scale per tile)
        "bwd_prep_v_kernel": (2 * kb + kb // (D // 2), 0),
        "bwd_q_tc_kernel": (4 * qb + 2 * kb + 3 * lse, 6 * D * npair),
        "bwd_kv_tc_kernel": (2 * qb + 5 * kb + 4 * lse, 8 * D * npair),
    }
    return dict(tokens=tok, npair=npair, fwd_bytes=fwd_bytes, fwd_flops=fwd_flops,
                bwd_bytes=bwd_bytes if bwd else 0, bwd_flops=bwd_flops if bwd else 0,
                kernels=kernels)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary, if it was taken on
    the kernel source as it is now (sha of the .cu file), else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        entries = json.load(f)
    for e in entries:
        if e.get("kernel") != kernel or e.get("workload") != workload:
            continue
        src = os.path.join(ROOT, e["source"])
        if not os.path.exists(src):
            return None
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return e["bytes_per_launch"] if sha == e.get("source_sha") else None
    return None


class ClockSampler:
    """nvidia-smi clocks/throttle sampling around the timed region.  The sampler starts before
    the warm-up and the timed region waits for its first row, so a short region is covered;
    `mark_start` / `mark_end` bracket the region on the host clock and the summary takes the
    rows inside it, or, when the region is shorter than the sampling interval, the last row
    before it and the first row after it (reported as "window": "bracketing")."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 20

    def __init__(self, gpu_id: str):
        self.index, self.rows, self.proc = gpu_id, [], None
        self.t_start = self.t_end = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.INTERVAL_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.monotonic(), [x.strip() for x in line.split(",")]))

    def _wait_rows(self, after, limit_s):
        end = time.monotonic() + limit_s
        while self.proc and self.proc.poll() is None and time.monotonic() < end:
            if self.rows and self.rows[-1][0] > after:
                return
            time.sleep(0.005)

    def wait_ready(self):
        self._wait_rows(0.0, 10.0)  # nvidia-smi takes a moment to print its first row

    def mark_start(self):
        self.t_start = time.monotonic()

    def mark_end(self):
        self.t_end = time.monotonic()
        self._wait_rows(self.t_end, 1.0)

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows, window = self.rows, "all"
        if self.t_start is not None and self.t_end is not None:
            inside = [r for r in rows if self.t_start <= r[0] <= self.t_end]
            window = "timed region"
            if not inside:
                before = [r for r in rows if r[0] < self.t_start][-1:]
                after = [r for r in rows if r[0] > self.t_end][:1]
                inside, window = before + after, "bracketing"
            rows = inside
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "window": window}


def cpu_oracle_run(B, S, W, bwd, seed=0):
    """One fp64 oracle pass (forward + full backward) over B x S tokens; returns seconds."""
    import oracle
    from global_attention_b200.synth import make_inputs
    t = make_inputs(B, S, seed=seed, with_dout=bwd)
    P = oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], window=W)
    t0 = time.perf_counter()
    P.forward()
    if bwd:
        P.backward(t["dout"])
    return time.perf_counter() - t0


def pair_scaled(secs, B, S, W, S_full, W_full):
    """Seconds per token of the (S_full, W_full) layer from an oracle run over B x S tokens with
    window W: the oracle's work is proportional to the visible (query, key) pairs."""
    return secs / (B * pairs(S, W)) * pairs(S_full, W_full) / S_full


# The oracle's bounded sample of one layer, shared by the reference arm (one sample per step)
# and the GPU arm's cpu_baseline (samples until about 10 s of CPU time): same heads and
# window as the workload, fewer and shorter sequences.  The oracle's work is proportional to
# the visible (query, key) pairs, so a sample's time per pair scales to the workload's pairs
# per token (a sliding layer past its first W tokens has the same pairs per token).
ORACLE_SAMPLE_TOKENS = {"sliding": 4096, "global": 1024}


def oracle_sample_shape(Sw, W):
    if W >= Sw:            # global layer: a shorter causal sequence
        n = ORACLE_SAMPLE_TOKENS["global"]
        return 1, n, n
    return 1, ORACLE_SAMPLE_TOKENS["sliding"], W


def oracle_sample(workload, seed=0):
    """One sample of a whole step of `workload` on the fp64 oracle (every layer of the step,
    each on its own sample).  Returns (seconds per workload token, seconds it took, text)."""
    Bw, Sw, W, bwd = WORKLOADS[workload]
    spt, took, parts = 0.0, 0.0, []
    for lw, _ in layers_of(workload):
        Bc, Sc, Wc = oracle_sample_shape(Sw, lw)
        secs = cpu_oracle_run(Bc, Sc, Wc, bwd, seed=seed)
        spt += pair_scaled(secs, Bc, Sc, Wc, Sw, lw)
        took += secs
        parts.append(f"{Bc}x{Sc} tokens, window {Wc}")
    text = ("; ".join(parts) + f" per sample, fwd{'+bwd' if bwd else ''} in fp64; time per visible (query, key) "
            "pair scaled to the workload's pairs per token")
    return spt, took, text


def run_reference(args):
    """--impl reference: the fp64 CPU oracle as it stands, each step one bounded sample of the
    workload (oracle_sample); the value is the workload's tokens/s at the sampled rate."""
    _, rank, _ = rank_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    Bw, Sw, W, bwd = WORKLOADS[args.workload]
    for i in range(args.warmup):
        oracle_sample(args.workload, seed=i)
    runs = [oracle_sample(args.workload, seed=i) for i in range(args.steps)]
    spt = sum(r[0] for r in runs) / len(runs)
    val = 1.0 / spt
    cores = oracle.num_threads()
    sample = runs[0][2] + f"; {cores} threads"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        # what one timed step (one sample) took; the workload's own step at this rate is scaled
        "ms_per_step": 1e3 * sum(r[1] for r in runs) / len(runs),
        "workload_ms_per_step_scaled": 1e3 * Bw * Sw * spt,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(args.workload), "sample": sample},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))
    return 0


def layers_of(w):
    """[(window, weight)] of the layers one step of workload w runs."""
    B, S, W, bwd = WORKLOADS[w]
    if w in LAYER_MIX:
        return [(S if lw is None else lw, wt) for lw, wt in LAYER_MIX[w]]
    return [(W, 1)]


def workload_name(w):
    B, S, W, bwd = WORKLOADS[w]
    if w in LAYER_MIX:
        mix = ":".join(str(wt) for _, wt in LAYER_MIX[w])
        return (f"gated sliding W={W} + global (full causal) attention fwd on the same inputs, {mix} layer mix, "
                f"B={B} S={S} Hq={HQ} Hkv={HKV} D={D}")
    kind = "global (full causal)" if W >= S else f"sliding window W={W}"
    return f"gated {kind} attention {'fwd+bwd' if bwd else 'fwd'}, B={B} S={S} Hq={HQ} Hkv={HKV} D={D}"


# decode: B sequences at context position P, one new token each, per layer (window, cache
# slots, weight of the layer in the 5:1 sliding:global pattern)
DECODE_WORKLOADS = {
    "decode16k": (64, 16383, ((128, 128, 5), (16384, 16384, 1))),
}


def decode_bytes(B, P, W, C):
    """Algorithmic HBM bytes of one decode call: every visible cached key (fp16) and value
    (bf16) read once; the new token's q, g, k, v read, out written; its cache slot written."""
    vis = min(W, C, P + 1)
    return (B * vis * HKV * D * 4 + B * HQ * D * 2 * 3 + B * HKV * D * 2 * 2 + B * HKV * D * 4
            + B * HQ * 4)


def run_decode(args):
    """One decode step per layer of the workload: B tokens through zgcm_attn_decode."""
    import torch
    import global_attention_b200 as ga
    world, rank, local = rank_env()
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ga.load()
    B, P, layers = DECODE_WORKLOADS[args.workload]
    gen = torch.Generator().manual_seed(1000 + rank)
    tok = {n: torch.randn((B, h, D), generator=gen).to(torch.bfloat16)
           for n, h in (("q", HQ), ("k", HKV), ("v", HKV), ("g", HQ))}
    gam = {n: torch.rand((D,), generator=gen) + 0.5 for n in ("gamma_q", "gamma_k")}
    host = {n: t.pin_memory() for n, t in {**tok, **gam}.items()}
    d = {n: t.to(dev) for n, t in host.items()}
    pos = torch.full((B,), P, dtype=torch.int32, device=dev)
    caches = []
    for W, C, _ in layers:
        # synthetic cache contents of the shape and scale of normalised keys / raw values
        kc = (torch.randn((B, C, HKV, D), generator=gen) * 1.0).to(torch.float16).to(dev)
        vc = torch.randn((B, C, HKV, D), generator=gen).to(torch.bfloat16).to(dev)
        ws = torch.empty(max(16, ga.zgcm_attn_decode_workspace_size(B, HQ, W, C)), dtype=torch.uint8, device=dev)
        caches.append((kc, vc, ws))
    out = torch.empty((B, HQ, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, HQ), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def call(li, src=d):
        W, C, _ = layers[li]
        kc, vc, ws = caches[li]
        ga.zgcm_attn_decode(src["q"], src["k"], src["v"], src["g"], src["gamma_q"], src["gamma_k"], pos, kc, vc,
                            window=W, out=out, lse=lse, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        for li in range(len(layers)):
            call(li)
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in layers]
          for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        clk.wait_ready()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        t0.record(stream)
        for i in range(args.steps):
            for li in range(len(layers)):
                ev[i][li][0].record(stream)
                call(li)
                ev[i][li][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps
    layer_ms = [statistics.mean(ev[i][li][0].elapsed_time(ev[i][li][1]) for i in range(args.steps))
                for li in range(len(layers))]
    # end to end: the new tokens from pinned host memory, the outputs back, every step
    outs_host = torch.empty_like(out, device="cpu").pin_memory()
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v", "g"))
    d2h = outs_host.numel() * outs_host.element_size()
    dst = {n: torch.empty_like(t) for n, t in d.items()}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        for n in ("q", "k", "v", "g"):
            dst[n].copy_(host[n], non_blocking=True)
        for n in ("gamma_q", "gamma_k"):
            dst[n] = d[n]
        for li in range(len(layers)):
            call(li, dst)
            outs_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        if rank != 0:
            dist.destroy_process_group()
            return 0
    peaks, peak_src = load_peaks()
    # roofline of the heaviest layer's call (HBM-bound: it reads its whole window of cache)
    li = max(range(len(layers)), key=lambda k: layer_ms[k])
    W, C, _ = layers[li]
    nbytes = decode_bytes(B, P, W, C)
    roof = {"bound": "hbm", "achieved": nbytes / (layer_ms[li] / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "traffic": None, "kernel": f"decode_split_kernel + decode_combine_kernel (W={W})",
            "kernel_ms": layer_ms[li], "algorithmic_bytes": nbytes, "peak_source": peak_src}
    roof["frac"] = roof["achieved"] / roof["peak"]
    step_bytes = sum(decode_bytes(B, P, W, C) for W, C, _ in layers)
    t_roof = step_bytes / (peaks["hbm_gbs"] * 1e9)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = decode_cpu_baseline(P, layers)
    wsum = sum(wt for _, _, wt in layers)
    mix_ms = sum(wt * t for (_, _, wt), t in zip(layers, layer_ms)) / wsum
    rec = {
        "metric": METRIC, "value": job_throughput(B, world, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 tokens, N(0,1) fp16 / bf16 cache contents",
        "config": {"workload": f"gated attention decode, {B} sequences at position {P}, one token each through "
                               + " + ".join(f"W={W} (cache {C})" for W, C, _ in layers)
                               + f", Hq={HQ} Hkv={HKV} D={D}",
                   "global_batch": B * world, "seq_len": P + 1, "parallelism": f"dp{world} (independent sequences)",
                   "l2": f"caches larger than L2 ({sum(c[0].numel() * 2 + c[1].numel() * 2 for c in caches) / 1e9:.2f} GB)"},
        "pct_of_roofline": t_roof / (ms / 1e3), "roofline_step_ms": t_roof * 1e3,
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(B, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h * len(layers), "ms_per_step": e2e_ms},
        "gpu_launches": 2 * len(layers) * args.steps,
        "clocks": clk.summary(),
        "layer_mix": {"layers": [{"window": W, "cache": C, "weight": wt, "ms": t}
                                 for (W, C, wt), t in zip(layers, layer_ms)],
                      "weighted_ms_per_layer": mix_ms},
    }
    print(json.dumps(rec))
    return 0


# the Muon optimiser step on one matrix parameter: the SwiGLU projection of the model, hidden
# 4096 x intermediate 11008 (ZGCM-1 summary, section "核心方法")
MUON_WORKLOADS = {"muon4096x11008": (4096, 11008)}
MUON_METRIC = "muon_step_newton_schulz_tflops"


def muon_cpu_baseline(m, n):
    """The fp64 oracle's Muon step on a bounded sample: the matrix at one sixteenth of each
    dimension, in TFLOP/s of its Newton–Schulz products."""
    import numpy as np
    from oracle import muon
    ms, ns = m // 16, n // 16
    rng = np.random.default_rng(0)
    W, G, M = (rng.standard_normal((ms, ns)) for _ in range(3))
    t0 = time.perf_counter()
    reps = 0
    while time.perf_counter() - t0 < 2.0 or reps < 1:
        muon.muon_step(W, G, M)
        reps += 1
    secs = (time.perf_counter() - t0) / reps
    return {"value": muon.ns_flops(ms, ns) / secs / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
            "kind": "oracle", "sample": f"{reps} steps on a {ms} x {ns} matrix (numpy fp64, its BLAS threads), "
                                        f"{secs * 1e3:.1f} ms each"}


def run_muon(args):
    """K Muon steps of one matrix parameter (momentum, scaling, five Newton–Schulz iterations,
    update), the inputs resident; the products' kernel timed on its own as well."""
    import torch
    import global_attention_b200 as ga
    from oracle import muon
    world, rank, local = rank_env()
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ga.load()
    m, n = MUON_WORKLOADS[args.workload]
    gen = torch.Generator().manual_seed(3000 + rank)
    G_host = (torch.randn((m, n), generator=gen) * 1e-2).to(torch.bfloat16).pin_memory()
    W = (torch.randn((m, n), generator=gen) * 2e-2).to(dev)
    G = G_host.to(dev)
    M = torch.zeros((m, n), device=dev)
    ws = torch.empty(ga.zgcm_muon_workspace_size(m, n), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    step = lambda g=G: ga.zgcm_muon_step(W, g, M, workspace=ws, stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        clk.wait_ready()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps
    if ga.zgcm_attn_device_error() != 0:
        print(json.dumps({"error": "device wait expired in the timed region"}))
        return 1
    # the products' kernel alone, on the iteration's two shapes (p = min, q = max): X X^T and
    # (A) X, each a 2 p^2 q multiply-add count
    p_, q_ = min(m, n), max(m, n)
    X = (torch.randn((p_, q_), generator=gen) * 1e-2).to(torch.bfloat16).to(dev)
    A = (torch.randn((p_, p_), generator=gen) * 1e-2).to(torch.bfloat16).to(dev)
    Cx, Ca = torch.empty_like(X), torch.empty_like(A)
    gemms = {"X X^T": lambda: ga.zgcm_muon_gemm(X, X, out=Ca, stream=stream),
             "A X": lambda: ga.zgcm_muon_gemm(A, X, D=X, alpha=-0.5, beta=1.5, b_kn=True, out=Cx, stream=stream)}
    kms = {}
    for name, f in gemms.items():
        for _ in range(3):
            f()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            f()
        e1.record(stream)
        torch.cuda.synchronize()
        kms[name] = e0.elapsed_time(e1) / args.steps
    # end to end: the gradient from pinned host memory and the updated weights back, every step
    W_host = torch.empty((m, n), dtype=torch.float32).pin_memory()
    Gd = torch.empty_like(G)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        Gd.copy_(G_host, non_blocking=True)
        step(Gd)
        W_host.copy_(W, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        if rank != 0:
            dist.destroy_process_group()
            return 0
    peaks, peak_src = load_peaks()
    flops = muon.ns_flops(m, n)
    name = max(kms, key=kms.get)
    gflop = 2 * p_ * p_ * q_
    roof = {"bound": "tensor", "achieved": gflop / (kms[name] / 1e3) / 1e12, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "traffic": None, "kernel": f"muon_gemm_kernel ({name}, {p_} x {q_})",
            "kernel_ms": kms[name], "kernels_ms": kms, "algorithmic_flops": gflop,
            "peak_source": f"{peak_src} (bf16 burst: the kernel timed back to back on its own)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    cpu = None if (world > 1 or args.no_cpu_baseline) else muon_cpu_baseline(m, n)
    launches = 3 + 2 * muon.NS_STEPS + 1  # momentum, norm, scaling; 2 products per step; update
    rec = {
        "metric": MUON_METRIC, "value": flops * world / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0, 0.01^2) bf16 gradient, N(0, 0.02^2) fp32 weights",
        "config": {"workload": f"Muon step of one {m} x {n} matrix (momentum 0.9, Frobenius scaling, "
                               f"{muon.NS_STEPS} Newton-Schulz steps {muon.NS_COEFFS}, lr 2e-4, wd 0.1)",
                   "parallelism": f"dp{world} (one matrix per GPU)",
                   "l2": f"operands larger than L2 ({m * n * 10 / 1e9:.2f} GB of W, G, M)"},
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": flops * world / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": G_host.numel() * 2, "d2h_bytes_per_step": W_host.numel() * 4,
                "ms_per_step": e2e_ms},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(rec))
    return 0


# the projections around the layer for the 16K training batch: x [B*S, 4096] -> q, k, v, g
# (heads 32 / 8 of 128) and the output projection, forward and backward
PROJ_WORKLOADS = {"proj16k": (4 * 16384, 4096, 32, 8, 128)}
PROJ_METRIC = "projections_fwd_bwd_tflops"


def proj_cpu_baseline(T, dm, hq, hkv, d):
    """The fp64 oracle's projections (forward and backward) on a bounded sample of the tokens."""
    import numpy as np
    from oracle import proj
    Ts = 256
    wq, wkv = hq * d, hkv * d
    rng = np.random.default_rng(0)
    x, a = rng.standard_normal((Ts, dm)), rng.standard_normal((Ts, wq))
    w, wo = rng.standard_normal((2 * (wq + wkv), dm)), rng.standard_normal((dm, wq))
    t0 = time.perf_counter()
    q, k, v, g = proj.qkvg_forward(x, w, wq, wkv)
    proj.qkvg_backward(x, w, q, k, v, g)
    y = proj.out_forward(a, wo)
    proj.out_backward(a, wo, y)
    secs = time.perf_counter() - t0
    fl = sum(proj.proj_flops(Ts, dm, wq, wkv, wq).values())
    return {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{Ts} of the {T} tokens (numpy fp64), {secs:.2f} s"}


def run_proj(args):
    """K steps of the projections' forward and backward on resident inputs."""
    import torch
    import global_attention_b200 as ga
    from oracle import proj
    world, rank, local = rank_env()
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ga.load()
    T, dm, hq, hkv, d = PROJ_WORKLOADS[args.workload]
    wq, wkv = hq * d, hkv * d
    gen = torch.Generator().manual_seed(4000 + rank)
    rnd = lambda shape, sc=1.0: (torch.randn(shape, generator=gen) * sc).to(torch.bfloat16).to(dev)
    x_host = torch.randn((T, dm), generator=gen).to(torch.bfloat16).pin_memory()
    x, w, wo = x_host.to(dev), rnd((2 * (wq + wkv), dm), dm ** -0.5), rnd((dm, wq), wq ** -0.5)
    a, dy = rnd((T, wq)), rnd((T, dm))
    parts = tuple(torch.empty((T, h), dtype=torch.bfloat16, device=dev) for h in (wq, wkv, wkv, wq))
    dparts = tuple(rnd(p.shape) for p in parts)
    dx, dw, y, da, dwo = (torch.empty_like(t) for t in (x, w, dy, a, wo))
    stream = torch.cuda.current_stream()
    names = ("qkvg_fwd", "out_fwd", "out_bwd", "qkvg_bwd")
    calls = {"qkvg_fwd": lambda src=x: ga.zgcm_proj_qkvg_fwd(src, w, Hq=hq, Hkv=hkv, D=d, out=parts, stream=stream),
             "out_fwd": lambda: ga.zgcm_proj_out_fwd(a, wo, out=y, stream=stream),
             "out_bwd": lambda: ga.zgcm_proj_out_bwd(a, wo, dy, da=da, dw=dwo, stream=stream),
             "qkvg_bwd": lambda src=x: ga.zgcm_proj_qkvg_bwd(src, w, *dparts, Hq=hq, Hkv=hkv, D=d, dx=dx, dw=dw,
                                                            stream=stream)}
    for _ in range(args.warmup):
        for n in names:
            calls[n]()
    torch.cuda.synchronize()
    ev = {n: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)] for n in names}
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        clk.wait_ready()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        t0.record(stream)
        for i in range(args.steps):
            for n in names:
                ev[n][i][0].record(stream)
                calls[n]()
                ev[n][i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps
    kms = {n: statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev[n]) for n in names}
    # end to end: the layer input from pinned host memory, dx back to the host, every step
    dx_host = torch.empty_like(dx, device="cpu").pin_memory()
    xd = torch.empty_like(x)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        xd.copy_(x_host, non_blocking=True)
        calls["qkvg_fwd"](xd)
        calls["out_fwd"]()
        calls["out_bwd"]()
        calls["qkvg_bwd"](xd)
        dx_host.copy_(dx, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        if rank != 0:
            dist.destroy_process_group()
            return 0
    peaks, peak_src = load_peaks()
    fl = proj.proj_flops(T, dm, wq, wkv, wq)
    total = sum(fl.values())
    top = max(kms, key=kms.get)
    roof = {"bound": "tensor", "achieved": fl[top] / (kms[top] / 1e3) / 1e12, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "traffic": None, "kernel": f"gemm_kernel ({top}: {2 if top.endswith('bwd') else 1} launch(es))",
            "kernel_ms": kms[top], "kernels_ms": kms, "algorithmic_flops": fl[top],
            "peak_source": f"{peak_src} (bf16 burst)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    cpu = None if (world > 1 or args.no_cpu_baseline) else proj_cpu_baseline(T, dm, hq, hkv, d)
    rec = {
        "metric": PROJ_METRIC, "value": total * world / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 activations and gradients, N(0, 1/fan_in) bf16 weights",
        "config": {"workload": f"q/k/v/g and output projections fwd+bwd, {T} tokens, hidden {dm}, heads {hq}/{hkv}x{d}",
                   "parallelism": f"dp{world}", "l2": f"operands larger than L2 ({(x.numel() + a.numel()) * 4 / 1e9:.2f} GB)"},
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": total * world / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": x_host.numel() * 2, "d2h_bytes_per_step": dx_host.numel() * 2,
                "ms_per_step": e2e_ms},
        "gpu_launches": 6 * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(rec))
    return 0


def decode_cpu_baseline(P, layers):
    """The oracle's forward rows for a bounded sample: the last row of 2 sequences of P + 1
    tokens per layer (the row a decode step computes), tokens per second over both layers."""
    import oracle
    from global_attention_b200.synth import make_inputs
    oracle.build()
    spt, parts = 0.0, []
    for W, C, _ in layers:
        t = make_inputs(2, P + 1, seed=7)
        prob = oracle.Problem(t["q"], t["k"], t["v"], t["g"], t["gamma_q"], t["gamma_k"], window=W)
        rows = [P, (P + 1) + P]        # flat row index b * S + i
        t0 = time.perf_counter()
        prob.forward(rows)
        secs = time.perf_counter() - t0
        spt += secs / 2
        parts.append(f"2 rows at position {P}, window {W}: {secs:.2f} s")
    return {"value": 1.0 / spt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "; ".join(parts) + " (the oracle's per-row forward, fp64, including its prologue)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS) + sorted(MUON_WORKLOADS)
                    + sorted(PROJ_WORKLOADS), default="swa16k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=8)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in DECODE_WORKLOADS:
        if args.impl == "reference":
            _, rank, _ = rank_env()
            if rank == 0:
                B, P, layers = DECODE_WORKLOADS[args.workload]
                cpu = decode_cpu_baseline(P, layers)
                print(json.dumps({"impl": "reference", "metric": METRIC, "value": cpu["value"], "unit": "tokens/s",
                                  "n_gpus": args.gpus, "steps": 1, "warmup": 0, "higher_is_better": True,
                                  "dtype": "f64", "data": "synthetic", "cpu_baseline": cpu,
                                  "e2e": {"value": cpu["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                          "d2h_bytes_per_step": 0}}))
            return 0
        return run_decode(args)
    if args.workload in PROJ_WORKLOADS:
        if args.impl == "reference":
            _, rank, _ = rank_env()
            if rank == 0:
                cpu = proj_cpu_baseline(*PROJ_WORKLOADS[args.workload])
                print(json.dumps({"impl": "reference", "metric": PROJ_METRIC, "value": cpu["value"],
                                  "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": 1, "warmup": 0,
                                  "higher_is_better": True, "dtype": "f64", "data": "synthetic",
                                  "cpu_baseline": cpu, "e2e": {"value": cpu["value"], "unit": "TFLOP/s",
                                                               "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
            return 0
        return run_proj(args)
    if args.workload in MUON_WORKLOADS:
        if args.impl == "reference":
            _, rank, _ = rank_env()
            if rank == 0:
                cpu = muon_cpu_baseline(*MUON_WORKLOADS[args.workload])
                print(json.dumps({"impl": "reference", "metric": MUON_METRIC, "value": cpu["value"],
                                  "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": 1, "warmup": 0,
                                  "higher_is_better": True, "dtype": "f64", "data": "synthetic",
                                  "cpu_baseline": cpu, "e2e": {"value": cpu["value"], "unit": "TFLOP/s",
                                                               "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
            return 0
        return run_muon(args)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    import global_attention_b200 as ga
    from global_attention_b200.synth import make_inputs

    world, rank, local = rank_env()
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    ga.load()

    Bw, Sw, W, bwd = WORKLOADS[args.workload]
    layers = layers_of(args.workload)
    # a training step: the forward keeps q~, k~ and the rows' inverse RMS for its backward
    keep = [bwd and ga.zgcm_attn_saved_size(Bw, Sw, HQ, HKV, D, 42, lw) > 0 for lw, _ in layers]
    wks = [work(Bw, Sw, lw, bwd, kp) for (lw, _), kp in zip(layers, keep)]
    wk = {k: sum(x[k] for x in wks) for k in ("fwd_bytes", "fwd_flops", "bwd_bytes", "bwd_flops")}
    wk["tokens"] = Bw * Sw
    t = make_inputs(Bw, Sw, seed=rank_seed(rank), with_dout=bwd)
    host = {k: v.pin_memory() for k, v in t.items()}
    d = {k: v.to(dev) for k, v in host.items()}
    stream = torch.cuda.current_stream()
    out = torch.empty_like(d["q"])
    lse = torch.empty((Bw, HQ, Sw), dtype=torch.float32, device=dev)
    grads = ws = None
    if bwd:
        grads = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]), dv=torch.empty_like(d["v"]),
                     dg=torch.empty_like(d["g"]), dgamma_q=torch.empty(D, device=dev),
                     dgamma_k=torch.empty(D, device=dev))
        ws = torch.empty(max(256, ga.zgcm_attn_bwd_workspace_size(Bw, Sw, HQ, HKV, D, W)),
                         dtype=torch.uint8, device=dev)

    def pair():
        return (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    # per layer: the forward's events, and one event pair per backward kernel
    ev_f = [[pair() for _ in layers] for _ in range(args.steps)]
    bwd_names = [ga.zgcm_attn_bwd_kernel_names(Sw, lw, saved=kp) if bwd else [] for (lw, _), kp in zip(layers, keep)]
    ev_m = [[[pair() for _ in names] for names in bwd_names] for _ in range(args.steps)]

    # forward scratch (normalised keys of the wide-window kernel), allocated once
    fws = [None if n == 0 else torch.empty(n, dtype=torch.uint8, device=dev)
           for n in (ga.zgcm_attn_fwd_workspace_size(Bw, Sw, HQ, HKV, D, 42, lw) for lw, _ in layers)]
    # the activation store of each layer (in place of the forward's workspace), allocated once
    svs = [torch.empty(ga.zgcm_attn_saved_size(Bw, Sw, HQ, HKV, D, 42, lw), dtype=torch.uint8, device=dev)
           if kp else None for (lw, _), kp in zip(layers, keep)]

    def step(i=None, src=d, dst=None):
        o = dst or {"out": out, "lse": lse, "grads": grads}
        for li, (lw, _) in enumerate(layers):
            if i is not None:
                ev_f[i][li][0].record(stream)
            ga.zgcm_attn_fwd(src["q"], src["k"], src["v"], src["g"], src["gamma_q"], src["gamma_k"],
                             window=lw, out=o["out"], lse=o["lse"], workspace=fws[li], saved=svs[li],
                             stream=stream)
            if i is not None:
                ev_f[i][li][1].record(stream)
            if bwd:
                ga.zgcm_attn_bwd(src["q"], src["k"], src["v"], src["g"], src["gamma_q"], src["gamma_k"],
                                 o["out"], o["lse"], src["dout"], window=lw, grads=o["grads"], workspace=ws,
                                 saved=svs[li], stream=stream, kernel_events=None if i is None else ev_m[i][li])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K steps, inputs resident in HBM (5.6 GB per step >> 126 MB L2)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        clk.wait_ready()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    # a bounded device wait that expired means a kernel gave up part of its work: no timing
    derr = ga.zgcm_attn_device_error()
    if derr != 0:
        print(json.dumps({"error": f"device wait expired in the timed region ({ga.zgcm_status_string(derr)})"}))
        return 1
    # per kernel and layer: (mean ms, algorithmic bytes, flops); the key names the kernel, and
    # the layer's window when the step runs more than one layer
    kern, layer_ms = {}, []
    for li, (lw, _) in enumerate(layers):
        tag = "" if len(layers) == 1 else f" (W={lw})"
        fwd_name = ga.zgcm_attn_fwd_kernel_name(Bw, Sw, HQ, HKV, 42, lw)
        fms = statistics.mean(ev_f[i][li][0].elapsed_time(ev_f[i][li][1]) for i in range(args.steps))
        kern[fwd_name + tag] = (fms, *wks[li]["kernels"].get(fwd_name, (0, 0)))
        lms = fms
        for k, n in enumerate(bwd_names[li]):
            kms_ = statistics.mean(ev_m[i][li][k][0].elapsed_time(ev_m[i][li][k][1]) for i in range(args.steps))
            kern[n + tag] = (kms_, *wks[li]["kernels"].get(n, (0, 0)))
            lms += kms_
        layer_ms.append(lms)
    kern_ms = {n: v[0] for n, v in kern.items()}
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps

    # ---- end to end through the public API: pinned host inputs -> HBM -> fwd+bwd -> host.
    # Every step uploads its inputs and downloads its results; the copies run on streams of
    # their own with double-buffered device tensors, so the download of step i overlaps the
    # upload of step i+1 (the two copy directions are independent) and both overlap compute.
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    outs_host = {"out": torch.empty_like(out, device="cpu").pin_memory(),
                 "lse": torch.empty_like(lse, device="cpu").pin_memory()}
    if bwd:
        for k, v in grads.items():
            outs_host[k] = torch.empty_like(v, device="cpu").pin_memory()
    d2h = sum(v.numel() * v.element_size() for v in outs_host.values())
    inbuf = [{k: torch.empty_like(v) for k, v in d.items()} for _ in range(2)]
    outbuf = [{"out": torch.empty_like(out), "lse": torch.empty_like(lse),
               "grads": {k: torch.empty_like(v) for k, v in grads.items()} if bwd else None} for _ in range(2)]
    s_up, s_dn = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_cp = [torch.cuda.Event() for _ in range(2)]
    ev_dn = [torch.cuda.Event() for _ in range(2)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    s_up.wait_event(e0)
    s_dn.wait_event(e0)
    for i in range(args.e2e_steps):
        x = i & 1
        with torch.cuda.stream(s_up):
            s_up.wait_event(ev_cp[x])          # step i-2's compute has read inbuf[x]
            for k in inbuf[x]:
                inbuf[x][k].copy_(host[k], non_blocking=True)
            ev_up[x].record(s_up)
        stream.wait_event(ev_up[x])
        stream.wait_event(ev_dn[x])            # step i-2's results have left outbuf[x]
        step(src=inbuf[x], dst=outbuf[x])
        ev_cp[x].record(stream)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(ev_cp[x])
            outs_host["out"].copy_(outbuf[x]["out"], non_blocking=True)
            outs_host["lse"].copy_(outbuf[x]["lse"], non_blocking=True)
            if bwd:
                for k, v in outbuf[x]["grads"].items():
                    outs_host[k].copy_(v, non_blocking=True)
            ev_dn[x].record(s_dn)
    for x in range(2):
        stream.wait_event(ev_dn[x])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    if world > 1:
        dist.barrier()

    if rank != 0:
        dist.destroy_process_group()
        return 0

    peaks, peak_src = load_peaks()
    tokens_step = wk["tokens"] * world
    value = job_throughput(wk["tokens"], world, ms_step)
    # roofline of the whole step and of the dominant kernel
    step_bytes = wk["fwd_bytes"] + wk["bwd_bytes"]
    step_flops = wk["fwd_flops"] + wk["bwd_flops"]
    t_roof = max(step_bytes / (peaks["hbm_gbs"] * 1e9), step_flops / (peaks["bf16_tflops"] * 1e12))
    kern = {n: v for n, v in kern.items() if v[1] or v[2]}
    name = max(kern, key=lambda k: kern[k][0])
    kms, kbytes, kflops = kern[name]
    t_hbm = kbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = kflops / (peaks["bf16_tflops_sustained"] * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": kbytes / (kms / 1e3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": kflops / (kms / 1e3) / 1e12,
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic_for(name.split(" (W=")[0], args.workload)
    roof.update({"kernel": name, "kernel_ms": kms, "algorithmic_bytes": kbytes, "flops": kflops,
                 "peak_source": peak_src, "kernels_ms": kern_ms})

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        # the reference arm's samples (oracle_sample), repeated until about 10 s of CPU time
        runs, took = [], 0.0
        while took < 10.0 and len(runs) < 64:
            runs.append(oracle_sample(args.workload, seed=len(runs)))
            took += runs[-1][1]
        cpu = {"value": len(runs) / sum(r[0] for r in runs), "unit": "tokens/s", "cores": oracle.num_threads(),
               "kind": "oracle", "sample": f"{len(runs)} samples of " + runs[0][2] + f" ({took:.1f} s in all)"}

    # per layer: the forward's kernels (each tcgen05 forward runs the key preparation kernel
    # first; the wide-window one, keeping its activations, also the query preparation) + every
    # backward kernel
    fwd_launches = []
    for (lw, _), kp in zip(layers, keep):
        fname = ga.zgcm_attn_fwd_kernel_name(Bw, Sw, HQ, HKV, 42, lw)
        # the strip forward keeping its activations runs the two preparation kernels first
        fwd_launches.append((3 if kp else 1) if fname == "fwd_strip_kernel"
                            else 3 if kp and fname == "fwd_glob_tc_kernel" else 2)
    launches_per_step = sum(f + len(n) for f, n in zip(fwd_launches, bwd_names))
    rec = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 q,k,v,g,dout; gamma U(0.5,1.5) fp32",
        "config": {"workload": workload_name(args.workload), "global_batch": Bw * world, "seq_len": Sw,
                   "window": W, "parallelism": f"dp{world} (independent batches, no collective)",
                   "l2": f"inputs larger than L2 ({(step_bytes) / 1e9:.2f} GB moved per step)"},
        "tflops": step_flops / (ms_step / 1e3) / 1e12 * world,
        "pct_of_roofline": t_roof / (ms_step / 1e3),
        "roofline_step_ms": t_roof * 1e3,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(wk["tokens"], world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if len(layers) > 1:
        wsum = sum(wt for _, wt in layers)
        mix_ms = sum(wt * t for (_, wt), t in zip(layers, layer_ms)) / wsum
        rec["layer_mix"] = {"layers": [{"window": lw, "weight": wt, "ms": t} for (lw, wt), t in zip(layers, layer_ms)],
                            "weighted_ms_per_layer": mix_ms,
                            "weighted_tokens_per_s": wk["tokens"] / (mix_ms / 1e3)}
    print(json.dumps(rec))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
