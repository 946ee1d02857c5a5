#!/usr/bin/env python
"""Benchmark of the MLA latent-KV hot path on B200.

Headline workload: DeepSeek-V2-shaped decode (d=5120, n_h=128, d_h=128,
d_R=64, d_c=512, d_c'=1536), batch 64, 8192 cached tokens per sequence plus
one new token each, bf16 storage.  One step = one mla_decode call: the new
tokens' down-projections and cache append, the query up-projection, W_UK
absorption, attention over the latent cache, split combine, W_UV and W_O.
Also reported in the same line: the causal prefill of 16384 tokens at the same
dims, and the V2-Lite (batch 32, 4096 cached tokens) and ragged long-context
(batch 128, seeded log-uniform lengths) decode workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own replica of
the workload (decode shards by sequence with no collective); rank 0 prints
the whole-job throughput measured over the slowest rank.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode tokens/s + latent-cache GB/s as % of roofline; prefill tokens/s"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["v2", "lite", "ragged"], default="v2")
    ap.add_argument("--ctx", type=int, default=0, help="override cached tokens per sequence (profiling cases)")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling cases)")
    ap.add_argument("--cache", choices=["dtype", "e4m3"], default="dtype",
                    help="latent cache rows of the --profile run (the headline line is always bf16 rows)")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the V2-Lite and ragged decode objects")
    ap.add_argument("--profile", action="store_true",
                    help="decode steps only (no clock sampling, e2e, prefill or CPU baseline): for ncu captures")
    ap.add_argument("--profile-prefill", type=int, default=0, metavar="T",
                    help="only `--steps` prefill calls of T tokens at the DeepSeek-V2 dims (for ncu captures)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        j = json.load(open(path))
        return (float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                "measured")
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def workload_lengths(name, ctx=0, batch=0):
    import synth
    p = synth.preset(name)
    L = list(p.seqlen)
    if batch:
        L = (L * ((batch + len(L) - 1) // len(L)))[:batch]
    if ctx:
        L = [ctx] * len(L)
    return p, L


def workload_config(args, world):
    """The `config` object of the JSON line; both arms report the same one."""
    p, L = workload_lengths(args.workload, args.ctx, args.batch)
    cache_bytes = decode_flops_bytes(p.dims, L)[2]
    return {"workload": f"{args.workload} decode: DeepSeek-V2 MLA dims" if args.workload != "lite"
            else "lite decode: DeepSeek-V2-Lite MLA dims",
            "global_batch": world * len(L), "seq_len": max(L) + 1, "cached_tokens": sum(L),
            "parallelism": f"dp-by-sequence replicas x{world}",
            "l2": f"inputs larger than L2 (cache {cache_bytes / 1e6:.0f} MB + weights)"}


def decode_flops_bytes(d, L):
    """Algorithmic FLOPs and HBM bytes of one decode step (bf16 weights; the
    cache rows in their format: bf16, or E4M3 c^KV + bf16 k^R + 16 bytes)."""
    B = len(L)
    ctx = sum(x + 1 for x in L)
    row = d.d_c + d.d_R
    row_bytes = d.d_c + 2 * d.d_R + 16 if getattr(d, "cache", "dtype") == "e4m3" else row * 2
    qin = d.d_cq if d.d_cq else d.d_model
    wrows = {
        "W_DQ": (d.d_cq, d.d_model), "W_UQ": (d.n_h * d.d_h, qin), "W_QR": (d.n_h * d.d_R, qin),
        "W_DKV": (d.d_c, d.d_model), "W_KR": (d.d_R, d.d_model), "W_UK": (d.n_h * d.d_h, d.d_c),
        "W_UV": (d.n_h * d.d_h, d.d_c), "W_O": (d.d_model, d.n_h * d.d_h)}
    welem = sum(a * b for a, b in wrows.values())
    cache_bytes = ctx * row_bytes
    bytes_total = cache_bytes + welem * 2 + B * d.d_model * (2 + 4) + B * row_bytes
    attn_flops = ctx * d.n_h * (2 * row + 2 * d.d_c)
    flops = attn_flops + 2 * welem * B
    return flops, bytes_total, cache_bytes, attn_flops


def prefill_flops(d, T):
    qin = d.d_cq if d.d_cq else d.d_model
    proj = 2 * T * (d.d_cq * d.d_model + d.n_h * (d.d_h + d.d_R) * qin + (d.d_c + d.d_R) * d.d_model
                    + 2 * d.n_h * d.d_h * d.d_c + d.d_model * d.n_h * d.d_h)
    attn = (T * (T + 1) // 2) * d.n_h * 2 * (d.d_h + d.d_R + d.d_h)
    return proj + attn, attn


class ClockSampler:
    """nvidia-smi clocks/throttle sampling in the background during a timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(mhz)}


def traffic_record(kernel_files):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (hash match); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    h = hashlib.sha256()
    for f in kernel_files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    key = h.hexdigest()[:16]
    ent = rec.get("decode_attention")
    if ent and ent.get("source_hash") == key:
        return ent.get("dram_bytes_per_launch")
    return None


ATTN_SOURCES = ["mla_latent_kv_47_b200/csrc/attn_decode_tc.cuh", "mla_latent_kv_47_b200/csrc/ptx.cuh"]


def oracle_decode_seconds(preset_name, n_seq_max=8, budget_s=12.0, seed=0):
    """Times the fp64 oracle (as it stands) on whole sequences of the workload."""
    import numpy as np
    import synth
    from oracle import mla as om
    p = synth.preset(preset_name)
    Wh = synth.weights(p, seed=seed)
    times, n = [], 0
    t_all = time.perf_counter()
    while n < n_seq_max and (time.perf_counter() - t_all) < budget_s:
        h = synth.hidden(p, n, p.seqlen[n] + 1)
        t0 = time.perf_counter()
        u = om.decode_unabsorbed(Wh, h, p.dims)
        times.append(time.perf_counter() - t0)
        assert np.all(np.isfinite(u))
        n += 1
    return times, p


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def reduce_max(x, world, device):
    """Max of a per-rank number over all ranks (the slowest rank sets the time)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank, ms_per_step):
    """Whole-job units per second: every rank processes `units_per_rank` per step."""
    return world * units_per_rank / (ms_per_step * 1e-3)


# ============================================================================ reference arm
def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def reference_sample(p, L, n=2, max_tokens=16384):
    """Sequences of the workload the oracle steps cycle over: the first `n`
    whose cache fits `max_tokens` (all of them at the uniform workloads)."""
    picks = [b for b in range(len(L)) if L[b] + 1 <= max_tokens][:n]
    return picks or [int(min(range(len(L)), key=lambda b: L[b]))]


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import synth
    from oracle import mla as om
    p, L = workload_lengths(args.workload, args.ctx, args.batch)
    Wh = synth.weights(p)
    picks = reference_sample(p, L)
    # inputs are drawn before the timed region: the steps time the oracle alone
    hs = {b: synth.hidden(p, b, L[b] + 1) for b in picks}

    def step(i):
        b = picks[i % len(picks)]
        u = om.decode_unabsorbed(Wh, hs[b], p.dims)
        assert np.all(np.isfinite(u))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = (time.perf_counter() - t0) / args.steps
    value = 1.0 / dt  # one new token per step (one sequence of the batch)
    cores = blas_threads()
    sample = (f"{args.steps} steps, each the fp64 un-absorbed oracle on one whole sequence of the {args.workload} "
              f"workload (sequences {picks}, {[L[b] + 1 for b in picks]} tokens), inputs drawn before timing")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ============================================================================ our arm
class DecodeSetup:
    """Seeded synthetic decode workload resident on the device: random
    N(0,0.02) bf16 weights, a latent cache filled through mla_cache_append
    from N(0,1) hidden states, the new tokens' hidden states and seqlen."""

    def __init__(self, m, dev, g, name, ctx=0, batch=0, cache="dtype"):
        import dataclasses
        import torch
        from mla_latent_kv_47_b200.cache import LatentCache
        from synth import weight_shapes
        self.m = m
        self.p, self.L = workload_lengths(name, ctx, batch)
        d = self.d = dataclasses.replace(self.p.dims, cache=cache)
        self.dims = m.make_dims(d)
        self.B = len(self.L)
        self.Wd = {k: (torch.randn(s, generator=g, device=dev) * 0.02).to(torch.bfloat16)
                   for k, s in weight_shapes(d).items()}
        self.wts = m.make_weights(self.Wd)
        self.cache = LatentCache(self.dims, [x + 1 for x in self.L], device=dev)
        self.ws = m.alloc_workspace(self.dims, self.B, 1, device=dev)
        chunk = 16384
        # E4M3 rows are encoded from the fp32 latents, which need room for a chunk of tokens
        fill_ws = m.alloc_workspace(self.dims, self.B, chunk, device=dev) if cache == "e4m3" else self.ws
        for b, n in enumerate(self.L):
            for t0 in range(0, n, chunk):
                k = min(chunk, n - t0)
                h = torch.randn((k, d.d_model), generator=g, device=dev).to(torch.bfloat16)
                m.cache_append(self.dims, self.wts, h, torch.full((k,), b, dtype=torch.int32, device=dev),
                               torch.arange(t0, t0 + k, dtype=torch.int32, device=dev), self.cache.handle, fill_ws)
        self.h_new = torch.randn((self.B, d.d_model), generator=g, device=dev).to(torch.bfloat16)
        self.seqlen = torch.tensor(self.L, dtype=torch.int32, device=dev)
        self.u = torch.empty((self.B, d.d_model), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        code, detail = m.device_status(fill_ws)
        assert code == 0, ("cache fill fault", code, detail)
        del fill_ws

    def step(self):
        self.m.decode(self.dims, self.wts, self.h_new, self.cache.handle, self.seqlen, self.u, self.ws)

    def check(self):
        code, detail = self.m.device_status(self.ws)
        assert code == 0, ("decode fault", code, detail)


def time_steps(m, step, K, barrier, ev_attn=True):
    """K steps between CUDA events on the current stream, after a barrier and
    a synchronize; the attention kernel of every step is bracketed by its own
    events.  Returns (ms per step, mean attention ms, launches in the region)."""
    import torch
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for e in ev_b + ev_e:  # torch creates the CUDA event on its first record
        e.record()
    barrier()
    torch.cuda.synchronize()
    launches0 = m.kernel_launches()
    t_start.record()
    for i in range(K):
        if ev_attn:
            m.set_attention_events(ev_b[i], ev_e[i])
        step()
    t_end.record()
    launches = m.kernel_launches() - launches0
    torch.cuda.synchronize()
    m.set_attention_events(None, None)
    ms = t_start.elapsed_time(t_end) / K
    attn = statistics.mean(ev_b[i].elapsed_time(ev_e[i]) for i in range(K)) if ev_attn else None
    return ms, attn, launches


def decode_summary(d, L, ms, attn_ms, world, hbm_gbs, bf16_tf):
    """Throughput and roofline fractions of one decode workload."""
    flops, bytes_total, cache_bytes, attn_flops = decode_flops_bytes(d, L)
    roof_ms = max(bytes_total / (hbm_gbs * 1e9), flops / (bf16_tf * 1e12)) * 1e3
    attn_roof_ms = max(cache_bytes / (hbm_gbs * 1e9), attn_flops / (bf16_tf * 1e12)) * 1e3
    return {
        "tokens_per_s": world * len(L) / (ms * 1e-3), "ms": ms, "batch": len(L), "cached_tokens": sum(L),
        "attn_ms": attn_ms, "latent_cache_gbs": cache_bytes / (attn_ms * 1e-3) / 1e9,
        "attn_roofline_frac": attn_roof_ms / attn_ms,
        "step_roofline": {"bytes": bytes_total, "flops": flops, "roofline_ms": roof_ms, "frac": roof_ms / ms},
    }


def profile_prefill(m, dev, g, T, steps, barrier):
    """`steps` prefill calls of T tokens (V2 dims) after one warm-up call, for ncu."""
    import torch
    import synth
    from synth import weight_shapes
    from mla_latent_kv_47_b200.cache import LatentCache
    d = synth.preset("prefill").dims
    dims = m.make_dims(d)
    Wd = {k: (torch.randn(s, generator=g, device=dev) * 0.02).to(torch.bfloat16) for k, s in weight_shapes(d).items()}
    wts = m.make_weights(Wd)
    pc = LatentCache(dims, [T], device=dev)
    wsp = m.alloc_workspace(dims, 1, T, device=dev)
    hp = torch.randn((T, d.d_model), generator=g, device=dev).to(torch.bfloat16)
    up = torch.empty((T, d.d_model), dtype=torch.float32, device=dev)
    m.prefill(dims, wts, hp, 0, pc.handle, 0, up, wsp)
    torch.cuda.synchronize()
    launches0 = m.kernel_launches()
    ms, attn, launches = time_steps(m, lambda: m.prefill(dims, wts, hp, 0, pc.handle, 0, up, wsp), steps, barrier)
    assert m.device_status(wsp)[0] == 0
    print(json.dumps({"profile_run": True, "prefill_tokens": T, "ms_per_call": ms, "attn_ms": attn,
                      "launches_before_timing": launches0, "launches_per_call": launches // steps}), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    import mla_latent_kv_47_b200 as m
    from mla_latent_kv_47_b200.cache import LatentCache

    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    # ---- inputs: seeded, synthetic, resident in HBM before timing
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + rank)
    if args.profile_prefill:
        return profile_prefill(m, dev, g, args.profile_prefill, args.steps, barrier)
    S = DecodeSetup(m, dev, g, args.workload, args.ctx, args.batch, cache=args.cache if args.profile else "dtype")
    d, L, B = S.p.dims, S.L, S.B

    for _ in range(max(args.warmup, 3)):
        S.step()
    torch.cuda.synchronize()
    K = args.steps
    with ClockSampler(dev.index) as clk:
        # keep the GPU busy while the sampler starts, so its samples see load
        t0 = time.perf_counter()
        while not args.profile and time.perf_counter() - t0 < 0.5:
            for _ in range(20):
                S.step()
            torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        launches_before = m.kernel_launches()
        ms, attn_ms, launches = time_steps(m, S.step, K, barrier)
    barrier()
    ms = max_over_ranks(ms)
    attn_ms = max_over_ranks(attn_ms)
    S.check()

    if args.profile:
        print(json.dumps({"profile_run": True, "ms_per_step": ms, "attn_ms": attn_ms,
                          "launches_before_timing": launches_before, "launches_per_step": launches // K}),
              flush=True)
        return 0
    # ---- end to end: host (pinned) inputs in, host output back, every step
    h_host = S.h_new.cpu().pin_memory()
    sl_host = S.seqlen.cpu().pin_memory()
    u_host = torch.empty((B, d.d_model), dtype=torch.float32).pin_memory()
    h_dev, sl_dev = torch.empty_like(S.h_new), torch.empty_like(S.seqlen)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        h_dev.copy_(h_host, non_blocking=True)
        sl_dev.copy_(sl_host, non_blocking=True)
        m.decode(S.dims, S.wts, h_dev, S.cache.handle, sl_dev, S.u, S.ws)
        u_host.copy_(S.u, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K)
    h2d = h_host.numel() * h_host.element_size() + sl_host.numel() * 4
    d2h = u_host.numel() * 4
    S.check()

    main = decode_summary(d, L, ms, attn_ms, world, hbm_gbs, bf16_tf)
    cache_bytes = decode_flops_bytes(d, L)[2]
    del S
    torch.cuda.empty_cache()

    # ---- prefill (secondary): 16384 tokens at the DeepSeek-V2 dims
    prefill = None
    if not args.no_prefill and args.workload == "v2":
        import synth
        from synth import weight_shapes
        T = synth.preset("prefill").prefill_T
        Wd = {k: (torch.randn(s, generator=g, device=dev) * 0.02).to(torch.bfloat16)
              for k, s in weight_shapes(d).items()}
        wts = m.make_weights(Wd)
        dims = m.make_dims(d)
        pc = LatentCache(dims, [T], device=dev)
        wsp = m.alloc_workspace(dims, 1, T, device=dev)
        hp = torch.randn((T, d.d_model), generator=g, device=dev).to(torch.bfloat16)
        up = torch.empty((T, d.d_model), dtype=torch.float32, device=dev)
        for _ in range(3):
            m.prefill(dims, wts, hp, 0, pc.handle, 0, up, wsp)
        torch.cuda.synchronize()
        KP = 3
        pms, pattn, _ = time_steps(m, lambda: m.prefill(dims, wts, hp, 0, pc.handle, 0, up, wsp), KP, barrier)
        pms, pattn = max_over_ranks(pms), max_over_ranks(pattn)
        pf, pattn_flops = prefill_flops(d, T)
        assert m.device_status(wsp)[0] == 0
        prefill = {
            "tokens_per_s": world * T / (pms * 1e-3), "ms": pms, "tokens": T, "steps": KP,
            "tflops": pf / (pms * 1e-3) / 1e12,
            "roofline_frac": (pf / (bf16_tf * 1e12)) / (pms * 1e-3),
            "attention": {"ms": pattn, "tflops": pattn_flops / (pattn * 1e-3) / 1e12,
                          "frac": pattn_flops / (pattn * 1e-3) / 1e12 / bf16_tf},
        }
        del pc, wsp, hp, up, Wd
        torch.cuda.empty_cache()

    # ---- the other decode workloads (secondary objects of the same line):
    # V2-Lite, ragged long context, and the V2 workload over an E4M3 cache
    others = {}
    if args.workload == "v2" and not args.ctx and not args.batch and not args.no_secondary:
        for key, name, fmt in (("lite", "lite", "dtype"), ("ragged", "ragged", "dtype"), ("e4m3", "v2", "e4m3")):
            So = DecodeSetup(m, dev, g, name, cache=fmt)
            for _ in range(5):
                So.step()
            torch.cuda.synchronize()
            K2 = max(10, min(K, 200))
            oms, oattn, _ = time_steps(m, So.step, K2, barrier)
            So.check()
            others[key] = decode_summary(So.d, So.L, max_over_ranks(oms), max_over_ranks(oattn), world,
                                         hbm_gbs, bf16_tf)
            others[key]["steps"] = K2
            del So
            torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    cpu_baseline = None
    if world == 1 and not args.no_cpu_baseline:
        times, pp = oracle_decode_seconds(args.workload)
        cpu_baseline = {"value": len(times) / sum(times), "unit": "tokens/s", "cores": blas_threads(),
                        "cpu_model": cpu_model(), "kind": "oracle",
                        "sample": f"{len(times)} whole sequences of the {args.workload} workload "
                                  f"({pp.seqlen[0] + 1} tokens each) through the fp64 un-absorbed oracle"}

    traffic = traffic_record(ATTN_SOURCES)
    attn_gbs = cache_bytes / (attn_ms * 1e-3) / 1e9
    value = job_throughput(world, B, ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,0.02) weights, N(0,1) hidden states)",
        "config": workload_config(args, world),
        "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": hbm_gbs, "unit": "GB/s",
                     "frac": attn_gbs / hbm_gbs, "traffic": traffic,
                     "kernel": "decode attention (latent-cache stream)",
                     "peak_source": peak_src, "attn_ms": attn_ms},
        "step_roofline": dict(main["step_roofline"], latent_cache_gbs=cache_bytes / (ms * 1e-3) / 1e9),
        "e2e": {"value": world * B / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "cpu_baseline": cpu_baseline,
        "prefill": prefill,
        "lite": others.get("lite"),
        "ragged": others.get("ragged"),
        "v2_e4m3_cache": others.get("e4m3"),
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
