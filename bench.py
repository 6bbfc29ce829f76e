"""Benchmark of one denoising step: a full denoising pass plus the canvas update.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Workload (default): the large pass -- 4 layers, hidden 2816, 16 query / 8 KV heads of
128, 128 experts top-8 with FFN 704, vocabulary 262144, 32768 cached prefix positions
(K/V ~ N(0,1)), a 256-slot canvas of uniform random tokens; one step = dg_denoise_pass +
dg_canvas_update (the first of its 8 steps: 50% re-noised).  The largest of the five
workloads that fits one GPU.  `--workload layer1_bf16` runs the single-layer pass
(hidden 2048, 64 experts top-4, vocabulary 32768, prefix 1024), `denoise8_bf16` the
8-layer one (prefix 2048), and `chained8_bf16` whole chains: a 512-token prompt
prefilled, then 4 canvases of 16 passes each, every canvas appended by prefill.
Weights are seeded N(0, 0.02) bf16 (synthetic, random init).  The metric is canvas
tokens per second per pass (C / step latency), summed over ranks; each rank runs its
own replica (no data-path collective: the pass does not shard), so scaling is weak.

Prints ONE JSON line on rank 0.  --impl reference times the CPU oracle instead (a
bounded sample of the same workload on the host cores).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import threading
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from block_diffusion_lm_masked_b200 import configs as CF  # noqa: E402
from block_diffusion_lm_masked_b200 import roofline as RF  # noqa: E402
from block_diffusion_lm_masked_b200 import synth  # noqa: E402

METRIC = "canvas tokens/sec per denoising pass and pass latency (µs); % of roofline, 1×B200"
UNIT = "canvas tokens/s"
DATA = "synthetic: seeded random-init weights N(0,0.02) bf16, cached prefix K/V N(0,1), uniform canvas tokens"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def _workload_desc(name, cfg):
    where = f"prompt {cfg['prompt']} then {cfg['n_canvases']} canvases" if "prompt" in cfg else f"P{cfg['prefix']}"
    return (f"{name}: {cfg['n_layers']} layer(s), H{cfg['hidden']}, {cfg['n_q_heads']}q/{cfg['n_kv_heads']}kv "
            f"d{cfg['head_dim']}, E{cfg['n_experts']} top-{cfg['top_k']}, F{cfg['expert_ffn']}, V{cfg['vocab']}, "
            f"{where}, C{cfg['canvas']}; step = 1 denoising pass + canvas update")


class Clocks:
    """SM clock and clock-event reasons sampled through NVML (the counters nvidia-smi
    reads) every ~10 ms in a background thread during the timed region; read-only."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device):
        self.dev = device
        self.samples = []
        self.thread = None
        self.stop_flag = threading.Event()
        self.nv = None

    def _handle(self):
        import pynvml as nv
        import torch
        nv.nvmlInit()
        self.nv = nv
        p = torch.cuda.get_device_properties(self.dev)
        try:
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def _run(self, h):
        nv = self.nv
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                self.samples.append((sm, reasons(h)))
            except Exception as e:   # keep sampling; report the first failure
                self.error = self.error or repr(e)
            time.sleep(0.01)

    def start(self):
        self.error = None
        try:
            h = self._handle()
            self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(h, self.nv.NVML_CLOCK_SM)
        except Exception as e:
            self.error = repr(e)
            self.thread = None
            return
        self.thread = threading.Thread(target=self._run, args=(h,), daemon=True)
        self.thread.start()
        time.sleep(0.05)   # the sampler runs before the timed region starts

    def stop(self):
        if self.thread is None:
            return {"unavailable": self.error}
        self.stop_flag.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return {"unavailable": self.error or "no sample in the timed region"}
        nv = self.nv
        reasons = sorted({name for _, r in self.samples for name, attr in self.REASONS
                          if hasattr(nv, attr) and r & getattr(nv, attr)})
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "NVML, 10 ms"}


# clock-event reasons that make a timed region no measurement (a power cap is kept and noted)
SLOWDOWN_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocked(ranks, dev, run, sampler=Clocks):
    """Runs the timed region run() under the clock sampler; returns (run's result, the clock
    record).  A region that saw a hardware or thermal slowdown on any rank is timed once
    more, on every rank so that the ranks' collectives stay matched; the second region's
    record then names the reasons that voided the first under "remeasured_after"."""
    clk = sampler(dev)
    clk.start()
    out = run()
    clocks = clk.stop()
    slowed = sorted(set(clocks.get("reasons") or ()) & set(SLOWDOWN_REASONS))
    if ranks.max(1.0 if slowed else 0.0) > 0:
        ranks.barrier()
        if getattr(dev, "type", None) == "cuda":
            import torch
            torch.cuda.synchronize(dev)
        clk = sampler(dev)
        clk.start()
        out = run()
        clocks = dict(clk.stop(), remeasured_after=slowed)
    return out, clocks


def _oracle_step(host, ocache, canvas, n, prec, step):
    from oracle import dg_oracle as O
    logits, _ = O.denoise_pass(host, ocache, canvas, prec)
    return O.canvas_update(logits, n, synth.SEED_RENOISE, step)


def _oracle_threads():
    """Host threads the C++ oracle's OpenMP loops run on."""
    from oracle import dg_oracle as O
    return O.num_threads()


REF_BUDGET_S = 90.0

# DRAM bytes (read + write) of one launch of a kernel from an ncu capture of this
# workload, valid only for the kernel source it was taken on (sha256 prefix of the
# kernel's source file); any other source reports null.
NCU_TRAFFIC = {("layer1_bf16", "gemm_gate_up"): ("k_tc_gemm.cu", "8f9740b8fc51d669", 457.380608e6 + 6.031104e6),
               # profiles/gemm_gate_up_large4_bf16.md: the launch at the large model's sizes
               ("large4_bf16", "gemm_gate_up"): ("k_tc_gemm.cu", "dba5f1c440f71225", 1073.691e6 + 9.256448e6)}


def _ncu_traffic(workload, kernel):
    import hashlib
    entry = NCU_TRAFFIC.get((workload, kernel))
    if entry is None:
        return None
    src = os.path.join(ROOT, "block_diffusion_lm_masked_b200", "csrc", entry[0])
    try:
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    return entry[2] if digest == entry[1] else None


def _oracle_sample(cfg, host=None):
    """The oracle's inputs for a bounded sample of the workload: (model, cache, canvas,
    re-noise count, precision, what the sample is).  A denoising workload's cached prefix
    is its seeded N(0,1) K/V; the chained workload's first canvas runs after the oracle's
    own prefill of the 512-token prompt (set-up, not timed)."""
    from oracle import dg_oracle as O
    C = cfg["canvas"]
    host = host if host is not None else synth.Model(cfg)
    prec = O.Precision(cfg["dtype"])
    if "prompt" in cfg:
        prompt = synth.tokens(synth.SEED_TOKENS, synth.TID_PREFIX_TOKENS, cfg["prompt"], cfg["vocab"])
        ocache = O.prefill_append(host, O.Cache.empty(cfg), prompt, prec)
        what = "passes + updates of the first canvas after the prompt's prefill (set-up, untimed)"
    else:
        ocache = O.Cache(synth.prefix_cache(cfg, cfg["prefix"]))
        what = "whole oracle steps (denoising pass + update)"
    canvas = synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(0), C, cfg["vocab"])
    n = O.renoise_count(C, cfg["steps"], 0, cfg["renoise_start"], cfg["renoise_end"])
    return host, ocache, canvas, n, prec, what


def run_reference(args, cfg, name):
    """The CPU oracle on the host cores, one oracle step per timed step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    C = cfg["canvas"]
    host, ocache, canvas, n, prec, what = _oracle_sample(cfg)
    # a bounded sample: at most one warm-up step, then whole steps until K are done or
    # REF_BUDGET_S seconds have passed (at least one)
    for w in range(min(args.warmup, 1)):
        _oracle_step(host, ocache, canvas, n, prec, 0)
    t0 = time.perf_counter()
    done = 0
    while done < args.steps and (done == 0 or time.perf_counter() - t0 < REF_BUDGET_S):
        _oracle_step(host, ocache, canvas, n, prec, 0)
        done += 1
    dt = time.perf_counter() - t0
    ms = dt * 1e3 / done
    value = C / (ms / 1e3)
    cores = _oracle_threads()
    sample = (f"{done} of {args.steps} requested {what}, fp64 C++ with OpenMP, of the workload, "
              f"{REF_BUDGET_S:.0f} s budget")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": {"workload": _workload_desc(name, cfg)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(cfg, budget_s=30.0, host=None):
    """Time the oracle as it stands on a bounded sample: whole oracle steps until ~budget
    (at least one).  `host`: the synthetic model already built for the GPU run."""
    C = cfg["canvas"]
    host, ocache, canvas, n, prec, what = _oracle_sample(cfg, host)
    times = []
    t_start = time.perf_counter()
    while not times or (time.perf_counter() - t_start < budget_s / 2 and len(times) < 5):
        t0 = time.perf_counter()
        _oracle_step(host, ocache, canvas, n, prec, 0)
        times.append(time.perf_counter() - t0)
    ms = statistics.median(times) * 1e3
    return {"value": C / (ms / 1e3), "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"{len(times)} {what} of the workload, fp64 C++ with OpenMP; median {ms:.0f} ms per step"}


class Ranks:
    """One process per GPU (torchrun sets WORLD_SIZE / RANK / LOCAL_RANK): the process
    group, barriers, and the max over ranks of a device-timed quantity.  With one rank
    every call is a no-op."""

    def __init__(self, backend="nccl", device=None, timeout_s=120):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self.dist = None
        if self.world > 1:
            import torch.distributed as dist
            from datetime import timedelta
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)
            self.dist = dist

    @property
    def is_root(self):
        return self.rank == 0

    def barrier(self):
        if self.dist:
            self.dist.barrier()

    def max(self, x):
        """The largest x over the ranks (every rank gets it)."""
        if not self.dist:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def job_value(world, C, steps, max_ms):
    """Whole-job canvas tokens per second: every rank processed C * steps tokens; the job
    took as long as its slowest rank."""
    return world * C * steps / (max_ms / 1e3)


def run_variant(args, cfg, name):
    """B canvases per pass through the batched calls (each with its own cache and prefix),
    optionally with the experts in 8-bit (MX-FP8) storage; the same metric, timing rules
    and JSON keys as the default line, whose CPU baseline it does not repeat.  A step is
    one batched pass plus each canvas's update."""
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    from block_diffusion_lm_masked_b200 import dg

    B, lowp, vlowp = args.canvases, args.experts, args.vocab
    P, C, V, k = cfg["prefix"], cfg["canvas"], cfg["vocab"], cfg["top_k"]
    model = dg.Model(synth.Model(cfg), dev)
    if lowp == "mx8":
        model.set_experts_mx8(synth.mx8_experts(cfg))
    elif lowp == "nv4":
        model.set_experts_nv4(synth.nv4_experts(cfg))
    if vlowp == "mx8":
        model.set_vocab_mx8(synth.mx8_vocab(cfg))
    elif vlowp == "nv4":
        model.set_vocab_nv4(synth.nv4_vocab(cfg))
    caches = []
    for b in range(B):
        c = dg.KVCache(cfg, ((P + C + 7) // 8) * 8, dev)
        c.load_prefix(synth.prefix_cache(cfg, P, seed=synth.SEED_WEIGHTS + 100 + b))
        caches.append(c)
    ws = dg.Workspace(cfg, B * C, dev)
    noise = torch.from_numpy(np.stack([synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(rank * B + b), C, V)
                                       for b in range(B)]))
    canv_in = noise.to(dev)
    canv_out = canv_in.clone()
    logits = torch.empty(B, C, V, device=dev)
    n_ren = dg.renoise_count(C, 1, 0, cfg["renoise_start"], cfg["renoise_end"])
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step(s):
        if args.fused_update:  # the canvas is the call's input and output: each step denoises the last result
            dg.denoise_update(model, caches[0], canv_out[0], n_ren, ws, seed=synth.SEED_RENOISE, step=s)
            return
        dg.denoise_pass_batched(model, caches, canv_in, logits, ws)
        for b in range(B):
            dg.canvas_update(logits[b], n_ren, synth.SEED_RENOISE + b, s, canv_out[b], ws)

    unions = torch.zeros(cfg["n_layers"], dtype=torch.int32, device=dev)
    model.set_taps({"unions": unions, "rows": B * C})
    step(0)
    model.set_taps(None)
    torch.cuda.synchronize(dev)
    unions_h = [int(u) for u in unions.cpu()]
    for w in range(args.warmup):
        step(w)
    dg.device_status(ws)

    def timed(K, profile):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        if profile:
            dg.profile_reset()
            dg.profile_enable(True)
        l0 = dg.launch_count()
        for s_ in range(K):
            flush.zero_()
            ev[s_][0].record(stream)
            step(s_)
            ev[s_][1].record(stream)
        torch.cuda.synchronize(dev)
        if profile:
            dg.profile_enable(False)
        return sum(a.elapsed_time(b) for a, b in ev), dg.launch_count() - l0

    ranks.barrier()
    torch.cuda.synchronize(dev)
    (total_ms, launches), clocks = clocked(ranks, dev, lambda: timed(args.steps, profile=False))
    dg.device_status(ws)
    total_ms = ranks.max(total_ms)
    ranks.barrier()
    prof_ms, _ = timed(min(args.steps, 200), profile=True)
    kern = {}
    for kname in dg.KERNEL_KINDS:
        ms, n = dg.profile_read(kname)
        if n:
            kern[kname] = {"launches": n, "avg_us": ms * 1e3 / n, "share": ms / max(prof_ms, 1e-9)}

    h_in, h_out = noise.clone().pin_memory(), torch.empty_like(noise).pin_memory()
    # the step's input: the canvases the batched pass reads, or for the fused call the canvas
    # it reads and overwrites
    dst_in = canv_out if args.fused_update else canv_in
    e2e_ms = []
    for s_ in range(args.steps + args.warmup):
        flush.zero_()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dst_in.copy_(h_in, non_blocking=True)
        step(s_)
        h_out.copy_(canv_out, non_blocking=True)
        b_.record(stream)
        b_.synchronize()
        if s_ >= args.warmup:
            e2e_ms.append(a.elapsed_time(b_))
    e2e_total = ranks.max(sum(e2e_ms))
    dg.device_status(ws)

    hbm, tf_burst, _, peak_src = _peaks()
    ew = {"mx8": RF.MX8_WBYTES, "nv4": RF.NV4_WBYTES}.get(lowp)
    vw = {"mx8": RF.MX8_WBYTES, "nv4": RF.NV4_WBYTES}.get(vlowp)
    flops = B * RF.pass_flops(cfg, P, C)
    nbytes = RF.pass_bytes_batched(cfg, [P] * B, C, unions_h, ew, vw) + B * 8 * C
    if args.fused_update:  # no logits written or read back: the tile records instead
        nbytes += 2 * 16 * C * ((V + 127) // 128) - 2 * 4 * C * V
    t_roof = RF.time_bound(flops, nbytes, tf_burst * 1e12, hbm * 1e9)
    ms_step = total_ms / args.steps
    roof = None
    gu = kern.get("gemm_gate_up")
    if gu:
        per_launch = RF.gate_up_bytes(cfg, unions_h[0], B * C * k, ew)
        achieved = per_launch / (gu["avg_us"] * 1e-6) / 1e9
        roof = {"kernel": "gemm_gate_up" + ("" if lowp == "bf16" else "_" + lowp), "bound": "hbm",
                "achieved": achieved,
                "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "traffic": None,
                "peak_source": f"{peak_src} hbm_gbs", "bytes_per_launch": per_launch}
    line = {
        "metric": METRIC, "value": job_value(world, B * C, args.steps, total_ms), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
        "config": {"workload": _workload_desc(name, cfg), "canvases_per_pass": B, "attention": _attention_kind(),
                   "update": "fused into the vocabulary projection" if args.fused_update else "two kernels on logits",
                   "experts": {"bf16": "bf16", "mx8": "mx8 (E4M3 + E8M0 per 32, synthetic codes)",
                               "nv4": "nv4 (E2M1 + E4M3 per 16 + fp32 tensor scale, synthetic codes)"}[lowp],
                   "vocab_weights": {"bf16": "bf16", "mx8": "mx8 (E4M3 + E8M0 per 32, synthetic codes)",
                                     "nv4": "nv4 (E2M1 + E4M3 per 16 + fp32 tensor scale, synthetic codes)"}[vlowp],
                   "l2": "flushed between steps (256 MB write)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU", "expert_union": unions_h},
        "roofline": roof,
        "pass_roofline": {"t_roof_us": t_roof * 1e6, "frac": t_roof * 1e3 / ms_step, "flops": flops,
                          "bytes": nbytes, "peak_source": peak_src},
        "kernels": kern,
        "e2e": {"value": job_value(world, B * C, args.steps, e2e_total), "unit": UNIT,
                "h2d_bytes_per_step": B * C * 4, "d2h_bytes_per_step": B * C * 4},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    ranks.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_chained(args, cfg, name):
    """--workload chained8_bf16: one step = one whole chain through the public calls --
    the prompt's prefill (dg_prefill_append), then for each canvas dg_generate_canvas (16
    passes with re-noising, then the canvas appended by prefill).  The line's value is
    canvas tokens per second over the chain's passes (canvases x steps x C / chain time,
    prefills included); the chain's end-to-end time, its prefill times and the passes'
    median latency are reported beside it."""
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    from block_diffusion_lm_masked_b200 import dg

    T0, C, S, NC, V = cfg["prompt"], cfg["canvas"], cfg["steps"], cfg["n_canvases"], cfg["vocab"]
    r0, r1 = cfg["renoise_start"], cfg["renoise_end"]
    cap = T0 + NC * C
    host = synth.Model(cfg)
    model = dg.Model(host, dev)
    cache = dg.KVCache(cfg, cap, dev)
    ws = dg.Workspace(cfg, max(T0, C), dev)
    prompt_h = torch.from_numpy(synth.tokens(synth.SEED_TOKENS, synth.TID_PREFIX_TOKENS, T0, V)).pin_memory()
    noise_h = torch.from_numpy(np.stack([synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(rank * NC + c), C, V)
                                         for c in range(NC)])).pin_memory()
    prompt = prompt_h.to(dev)
    noise = noise_h.to(dev)
    canv = noise.clone()
    logits = torch.empty(C, V, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def chain(s, marks=None):
        cache.len = 0
        dg.prefill_append(model, cache, prompt, ws)
        if marks is not None:
            marks[0].record(stream)
        for c in range(NC):
            canv[c].copy_(noise[c])
            dg.generate_canvas(model, cache, canv[c], S, r0, r1, synth.SEED_RENOISE + s, True, logits, ws)
            if marks is not None:
                marks[c + 1].record(stream)

    for w in range(args.warmup):
        chain(w)
    dg.device_status(ws)
    ranks.barrier()
    torch.cuda.synchronize(dev)

    def timed_chains():
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        marks = [[torch.cuda.Event(enable_timing=True) for _ in range(NC + 1)] for _ in range(args.steps)]
        l0 = dg.launch_count()
        for s_ in range(args.steps):
            flush.zero_()
            ev[s_][0].record(stream)
            chain(s_, marks[s_])
            ev[s_][1].record(stream)
        torch.cuda.synchronize(dev)
        return ev, marks, dg.launch_count() - l0

    (ev, marks, launches), clocks = clocked(ranks, dev, timed_chains)
    dg.device_status(ws)
    chain_ms = [a.elapsed_time(b) for a, b in ev]
    prompt_ms = statistics.median(ev[i][0].elapsed_time(marks[i][0]) for i in range(args.steps))
    canvas_ms = [statistics.median(marks[i][c].elapsed_time(marks[i][c + 1]) for i in range(args.steps))
                 for c in range(NC)]
    total_ms = ranks.max(sum(chain_ms))
    ranks.barrier()

    # the passes alone, and one append, at each canvas's prefix length (per-kernel profile)
    dg.profile_reset()
    dg.profile_enable(True)
    chain(0)
    torch.cuda.synchronize(dev)
    dg.profile_enable(False)
    kern = {}
    tot = 0.0
    for kname in dg.KERNEL_KINDS:
        ms, n = dg.profile_read(kname)
        if n:
            kern[kname] = {"launches": n, "avg_us": ms * 1e3 / n}
            tot += ms
    for v in kern.values():
        v["share"] = v["avg_us"] * v["launches"] / 1e3 / max(tot, 1e-9)

    # end to end through the public calls with host buffers: prompt and noise canvases in,
    # finished canvases out, every chain
    out_h = torch.empty_like(noise_h).pin_memory()
    e2e_ms = []
    for s_ in range(args.steps + args.warmup):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        prompt.copy_(prompt_h, non_blocking=True)
        noise.copy_(noise_h, non_blocking=True)
        chain(s_)
        out_h.copy_(canv, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if s_ >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_total = ranks.max(sum(e2e_ms))
    dg.device_status(ws)

    hbm, tf_burst, tf_sust, peak_src = _peaks()
    # the expert union of every layer of every call of one chain (an untimed chain run
    # call by call with the union tap; the same passes as dg_generate_canvas): converging
    # canvases repeat tokens, so later passes touch fewer experts
    L = cfg["n_layers"]
    uni = torch.zeros(L, dtype=torch.int32, device=dev)
    model.set_taps({"unions": uni, "rows": max(T0, C)})

    def unions_now():
        torch.cuda.synchronize(dev)
        return [int(u) for u in uni.cpu()]

    cache.len = 0
    dg.prefill_append(model, cache, prompt, ws)
    prefill_unions = [unions_now()]
    pass_unions = []
    for c in range(NC):
        canv[c].copy_(noise[c])
        per = []
        for st_ in range(S):
            dg.denoise_pass(model, cache, canv[c], logits, ws)
            per.append(unions_now())
            dg.canvas_update(logits, dg.renoise_count(C, S, st_, r0, r1), synth.SEED_RENOISE, st_, canv[c], ws)
        pass_unions.append(per)
        dg.prefill_append(model, cache, canv[c], ws)
        prefill_unions.append(unions_now())
    model.set_taps(None)
    dg.device_status(ws)

    # roofline of the chain: every pass at its prefix length, every prefill, with the
    # measured unions
    t_roof = 0.0
    flops_total = bytes_total = 0.0
    for c in range(NC):
        P = T0 + c * C
        f = RF.pass_flops(cfg, P, C)
        for u in pass_unions[c]:
            b = RF.pass_bytes(cfg, P, C, u) + 8 * C
            t_roof += RF.time_bound(f, b, tf_burst * 1e12, hbm * 1e9)
            flops_total += f
            bytes_total += b
    for (P, T), u in zip([(0, T0)] + [(T0 + c * C, C) for c in range(NC)], prefill_unions):
        f = RF.prefill_flops(cfg, P, T)
        b = RF.prefill_bytes(cfg, P, T, u)
        t_roof += RF.time_bound(f, b, tf_burst * 1e12, hbm * 1e9)
        flops_total += f
        bytes_total += b
    ms_chain = total_ms / args.steps
    passes = NC * S
    value = job_value(world, passes * C, args.steps, total_ms)
    # per-launch algorithmic bytes of the expert GEMMs, averaged over the chain's launches
    # (each pass: L launches of C rows; each prefill: L - 1 launches of T rows)
    k = cfg["top_k"]
    eg = [(u, C * k) for per in pass_unions for us in per for u in us]
    eg += [(u, T * k) for T, us in zip([T0] + [C] * NC, prefill_unions) for u in us[:L - 1]]
    expert_bytes = {"gemm_gate_up": sum(RF.gate_up_bytes(cfg, u, r) for u, r in eg) / len(eg),
                    "gemm_down": sum(RF.down_bytes(cfg, u, r) for u, r in eg) / len(eg)}
    kroof = kernel_rooflines(cfg, T0 + (NC - 1) * C / 2, C, None, kern, hbm, tf_sust, peak_src,
                             expert_bytes=expert_bytes)
    roof = None
    if kroof:
        dom = max(kroof, key=lambda n: kern[n]["share"])
        roof = dict(kroof[dom], kernel=dom, traffic=_ncu_traffic(name, dom),
                    note="per-launch averages over the chain (expert GEMM bytes from the measured unions of every "
                         "call); attention FLOPs at the mean prefix length")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_chain, "pass_latency_us": statistics.median(canvas_ms) * 1e3 / S,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
        "config": {"workload": (f"{name}: {cfg['n_layers']} layers of H{cfg['hidden']}, E{cfg['n_experts']} "
                                f"top-{cfg['top_k']}, V{V}; a {T0}-token prompt prefilled, then {NC} canvases of "
                                f"{C} x {S} passes, each appended by prefill; step = one whole chain"),
                   "l2": "flushed between chains (256 MB write)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "chain_ms": {"median": statistics.median(chain_ms), "prompt_prefill": prompt_ms,
                     "per_canvas_incl_append": canvas_ms},
        "roofline": roof,
        "chain_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_chain, "flops": flops_total,
                           "bytes": bytes_total, "peak_source": peak_src},
        "kernels": kern, "kernel_rooflines": kroof,
        "e2e": {"value": job_value(world, passes * C, args.steps, e2e_total), "unit": UNIT,
                "h2d_bytes_per_step": 4 * (T0 + NC * C), "d2h_bytes_per_step": 4 * NC * C,
                "chain_ms": e2e_total / args.steps},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, host=host)
    ranks.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def kernel_rooflines(cfg, P, C, unions, kern, hbm, tf_peak, peak_src, rows=None, expert_bytes=None, fused=False):
    """Achieved rate and fraction of its bound for each big kernel of the step: the expert
    and vocabulary GEMMs and the update statistics against HBM bandwidth (algorithmic
    bytes per launch), attention against the bf16 tensor peak (algorithmic FLOPs).
    `expert_bytes`: per-launch bytes of the expert GEMMs when they are not those of one
    pass with per-layer `unions`."""
    rows = C if rows is None else rows
    k, L = cfg["top_k"], cfg["n_layers"]
    out = {}

    def hbm_entry(kname, nbytes_launch):
        if kname in kern:
            a = nbytes_launch / (kern[kname]["avg_us"] * 1e-6) / 1e9
            out[kname] = {"bound": "hbm", "achieved": a, "peak": hbm, "unit": "GB/s", "frac": a / hbm,
                          "bytes_per_launch": nbytes_launch, "peak_source": f"{peak_src} hbm_gbs"}
    if expert_bytes is None:
        expert_bytes = {"gemm_gate_up": sum(RF.gate_up_bytes(cfg, u, rows * k) for u in unions) / L,
                        "gemm_down": sum(RF.down_bytes(cfg, u, rows * k) for u in unions) / L}
    for kname, nb in expert_bytes.items():
        hbm_entry(kname, nb)
    if fused:   # the vocabulary GEMM writes tile records; the row merge reads them
        hbm_entry("gemm_vocab", RF.vocab_bytes(cfg, rows) - 4 * rows * cfg["vocab"] + RF.update_record_bytes(cfg, rows))
        hbm_entry("update_partial", RF.update_record_bytes(cfg, rows))
    else:
        hbm_entry("gemm_vocab", RF.vocab_bytes(cfg, rows))
        hbm_entry("update_partial", RF.update_bytes(cfg, rows))
    if "attention" in kern:
        fl = RF.attention_flops(cfg, P, C)
        a = fl / (kern["attention"]["avg_us"] * 1e-6) / 1e12
        out["attention"] = {"bound": "tensor", "achieved": a, "peak": tf_peak, "unit": "TFLOP/s",
                            "frac": a / tf_peak, "flops_per_launch": fl,
                            "peak_source": f"{peak_src} bf16_tflops_sustained (timed inside the step)",
                            "note": "algorithmic QK^T and PV FLOPs; the kernel issues about twice as many "
                                    "(query and probabilities as bf16 hi + lo terms)"}
    return out


def _graph_time(call, steps, warmup):
    """Median device time (us) of one `call`, captured once into a CUDA graph and replayed
    with CUDA events around each replay: the host work of the call (tensor-map encoding,
    argument checks) stays out of the timed region, which then holds only the call's
    device work."""
    import torch

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            call()
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    del graph
    return statistics.median(ts)


def run_kernel_attention(args):
    """--kernel attention: the block-masked attention launch alone (debug entry: the
    attention kernel and its split-KV merge) on synthetic bf16 data, the canvas's queries
    at the last positions of the key range, bidirectional.  One JSON line: median
    CUDA-event time per call and the algorithmic FLOP rate 4 * queries * heads * d * keys
    / time against the bf16 peak.  Used for ncu captures of attention at a chosen key
    count without the rest of the model on the device."""
    import torch

    from block_diffusion_lm_masked_b200 import dg

    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(7)
    d, n_q, n_keys, nq, nkv = 128, args.queries, args.keys, args.heads, args.kv_heads
    cap = ((n_keys + 7) // 8) * 8
    q = torch.randn(nq, n_q, d, generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn(nkv, cap, d, generator=g, device=dev).to(torch.bfloat16)
    vt = torch.randn(nkv, d, cap, generator=g, device=dev).to(torch.bfloat16)
    cfg = dict(CF.CONFIGS["layer1_bf16"], n_q_heads=nq, n_kv_heads=nkv, hidden=128, expert_ffn=64, n_experts=1,
               top_k=1, vocab=128, n_layers=1)
    ws = dg.Workspace(cfg, n_q, dev)
    out = torch.zeros(n_q, nq * d, dtype=torch.bfloat16, device=dev)
    lo = torch.zeros_like(out)
    fn = dg.debug_attention_pair_bf16 if args.attn_pair else dg.debug_attention_bf16
    us = _graph_time(lambda: fn(q, k, vt, n_keys, n_keys - n_q, False, out, ws, out_lo=lo), args.steps,
                     args.warmup)
    dg.device_status(ws)
    hbm, tf_burst, _, peak_src = _peaks()
    fl = 4.0 * n_q * nq * d * n_keys
    tf = fl / (us * 1e-6) / 1e12
    line = {"metric": "block-masked attention call latency (attention + split-KV merge)", "value": us, "unit": "us",
            "higher_is_better": False, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
            "data": "synthetic: q, K, V ~ N(0,1) bf16",
            "config": {"workload": f"attention: {n_q} queries x {nq} heads ({nkv} KV heads) d{d} over {n_keys} keys, "
                                   f"bidirectional", "attention": "head pairs, 128-key chunks" if args.attn_pair
                       else "one head, 128-key chunks", "l2": "K/V re-read between calls"},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": tf_burst, "unit": "TFLOP/s", "frac": tf / tf_burst,
                         "flops_per_call": fl, "peak_source": f"{peak_src} bf16_tflops"}}
    print(json.dumps(line), flush=True)
    return 0


def run_kernel_mma(args):
    """The tensor-pipe rate probe: one CTA per SM issuing MMAs of 128 x n x 16 back to back
    (A from shared memory or from TMEM), for the shapes the pass issues; one JSON line per
    shape with the cycles per instruction and the aggregate rate."""
    import torch
    from block_diffusion_lm_masked_b200 import dg
    torch.cuda.init()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    hbm, tf_burst, _, peak_src = _peaks()
    count = 1 << 14
    for a_tmem in (False, True):
        for n in (64, 128, 256):
            dg.debug_mma_rate(a_tmem, n, 256, sms)  # warm-up
            cyc, ms = dg.debug_mma_rate(a_tmem, n, count, sms)
            tf = 2.0 * 128 * n * 16 * count * sms / (ms * 1e-3) / 1e12
            print(json.dumps({"metric": "tcgen05 MMA instruction rate (one issuing thread per SM)",
                              "value": cyc / count, "unit": "cycles per instruction", "higher_is_better": False,
                              "dtype": "bf16", "data": "zero operands",
                              "config": {"workload": f"{count} MMAs of 128 x {n} x 16, A from "
                                                     f"{'TMEM' if a_tmem else 'shared memory'}, B from shared "
                                                     f"memory, {sms} CTAs"},
                              "tflops": tf, "frac_of_peak": tf / tf_burst,
                              "peak_source": f"{peak_src} bf16_tflops"}), flush=True)
    return 0


def run_kernel_gemm(args):
    """--kernel gemm --gemm vocab|gate_up|down: one GEMM launch of the large model's shapes
    through the debug entry (the pass's persistent tcgen05 kernel) on synthetic bf16 data:
    the vocabulary projection (262144 x 2816 weights, 256 tokens, fp32 out), or the grouped
    expert GEMMs over 128 experts with 16 rows each (gate/up with the SwiGLU epilogue, two-term
    tokens; down, fp32 out).  One JSON line: median CUDA-event time per launch and the
    algorithmic bytes per launch against the HBM bandwidth.  Used for ncu captures of the
    GEMMs at the large model's sizes without the rest of the model on the device."""
    import torch

    from block_diffusion_lm_masked_b200 import dg

    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(11)
    cfg = CF.CONFIGS["large4_bf16"]
    H, F, V, E, k, C = cfg["hidden"], cfg["expert_ffn"], cfg["vocab"], cfg["n_experts"], cfg["top_k"], cfg["canvas"]
    rows = C * k

    def bf(*shape, scale=0.02):
        return (torch.randn(*shape, generator=g, device=dev) * scale).to(torch.bfloat16)

    err = torch.zeros(1, dtype=torch.int32, device=dev)
    if args.gemm == "vocab":
        W, X = bf(1, V, H), bf(C, H, scale=1.0)
        out = torch.empty(C, V, device=dev)
        scratch = dg.debug_gemm_scratch(C, 1)
        call = lambda: dg.debug_gemm_bf16(W, X, out, V, err, scratch)
        nbytes = RF.vocab_bytes(cfg, C)
    else:
        off = torch.arange(0, rows + 1, rows // E, dtype=torch.int32, device=dev)
        if args.gemm == "gate_up":
            W, W2 = bf(E, F, H), bf(E, F, H)
            Xf = torch.randn(rows, H, generator=g, device=dev)
            X = Xf.to(torch.bfloat16)
            X_lo = (Xf - X.float()).to(torch.bfloat16)
            out = torch.empty(rows, F, dtype=torch.bfloat16, device=dev)
            out_lo = torch.empty_like(out)
            scratch = dg.debug_gemm_scratch(rows, E)
            call = lambda: dg.debug_gemm_bf16(W, X, out, F, err, scratch, W2=W2, X_lo=X_lo, group_off=off,
                                              out_lo=out_lo)
            nbytes = RF.gate_up_bytes(cfg, E, rows)
        else:
            W = bf(E, H, F)
            Xf = torch.randn(rows, F, generator=g, device=dev)
            X = Xf.to(torch.bfloat16)
            X_lo = (Xf - X.float()).to(torch.bfloat16)
            out = torch.empty(rows, H, device=dev)
            scratch = dg.debug_gemm_scratch(rows, E)
            call = lambda: dg.debug_gemm_bf16(W, X, out, H, err, scratch, X_lo=X_lo, group_off=off)
            nbytes = RF.down_bytes(cfg, E, rows)
    us = _graph_time(call, args.steps, args.warmup)
    if err.item() != 0:
        raise RuntimeError(f"GEMM error word {err.item()}")
    hbm, _, _, peak_src = _peaks()
    gbs = nbytes / (us * 1e-6) / 1e9
    line = {"metric": f"GEMM launch latency ({args.gemm}, large model's shape)", "value": us, "unit": "us",
            "higher_is_better": False, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16",
            "data": "synthetic: weights N(0, 0.02), tokens N(0, 1), bf16",
            "config": {"workload": f"gemm {args.gemm}: H{H}, F{F}, V{V}, {E} experts x {rows // E} rows, C{C}",
                       "l2": "weights larger than L2 except the debug entry's token operand"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "bytes_per_launch": nbytes, "peak_source": f"{peak_src} hbm_gbs"}}
    print(json.dumps(line), flush=True)
    return 0


def _attention_kind():
    """Which attention kernel the library runs (DG_ATTN_PAIR=1: the head-pair kernel)."""
    return ("head pairs, 128-key chunks" if os.environ.get("DG_ATTN_PAIR", "")[:1] == "1"
            else "one head, 128-key chunks")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dg", choices=["dg", "reference"])
    ap.add_argument("--workload", default="large4_bf16", choices=CF.ORDER,
                    help="default: the 4-layer, 262K-vocabulary pass over a 32768-position prefix, the largest "
                         "single-GPU workload; chained8_bf16 times whole chains (prompt prefill, then canvases of "
                         "16 passes each appended)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--canvases", type=int, default=1,
                    help="canvases per pass (each its own request and cache) through the batched calls")
    ap.add_argument("--update", choices=["fused", "two-call"], default="fused",
                    help="fused (default): one call per step, the pass with the update's statistics as the "
                         "vocabulary projection's epilogue (no logits); two-call: dg_denoise_pass writes the "
                         "logits and dg_canvas_update reads them (always so for several canvases or 8/4-bit "
                         "weights)")
    ap.add_argument("--experts", default="bf16", choices=["bf16", "mx8", "nv4"],
                    help="expert weight storage; mx8 and nv4 run through the batched calls")
    ap.add_argument("--vocab", default="bf16", choices=["bf16", "mx8", "nv4"],
                    help="output-matrix storage; mx8 and nv4 run through the batched calls")
    ap.add_argument("--attn-pair", action="store_true",
                    help="run attention through the head-pair kernel instead of the single-head kernel "
                         "(sets DG_ATTN_PAIR=1)")
    ap.add_argument("--kernel", choices=["attention", "gemm", "mma"], default=None,
                    help="time one kernel alone on synthetic data instead of the step (attention: the "
                         "block-masked attention call over --keys keys; gemm: one GEMM of the large model's "
                         "shapes, --gemm; mma: the tensor-pipe rate probe for 128 x n x 16 instructions)")
    ap.add_argument("--gemm", choices=["vocab", "gate_up", "down"], default="vocab",
                    help="--kernel gemm: which GEMM")
    ap.add_argument("--keys", type=int, default=8192, help="--kernel attention: key count")
    ap.add_argument("--queries", type=int, default=256, help="--kernel attention: canvas queries")
    ap.add_argument("--heads", type=int, default=16, help="--kernel attention: query heads")
    ap.add_argument("--kv-heads", type=int, default=8, help="--kernel attention: KV heads")
    args = ap.parse_args()
    if args.kernel == "attention":
        return run_kernel_attention(args)
    if args.kernel == "gemm":
        return run_kernel_gemm(args)
    if args.kernel == "mma":
        return run_kernel_mma(args)
    if args.attn_pair:  # read by the library at its first attention call
        os.environ["DG_ATTN_PAIR"] = "1"
    name = args.workload
    cfg = CF.CONFIGS[name]
    if args.impl == "reference":
        return run_reference(args, cfg, name)
    if name == "chained8_bf16":
        return run_chained(args, cfg, name)
    if args.canvases < 1:
        ap.error("--canvases must be >= 1")
    variant = args.canvases > 1 or args.experts != "bf16" or args.vocab != "bf16"
    # the fused call runs one canvas with bf16 experts and output matrix
    args.fused_update = args.update == "fused" and not variant
    if variant:
        return run_variant(args, cfg, name)

    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank

    from block_diffusion_lm_masked_b200 import dg

    P, C, V = cfg["prefix"], cfg["canvas"], cfg["vocab"]
    host = synth.Model(cfg)
    model = dg.Model(host, dev)
    cache = dg.KVCache(cfg, ((P + C + 7) // 8) * 8, dev)
    cache.load_prefix(synth.prefix_cache(cfg, P))
    ws = dg.Workspace(cfg, C, dev)
    noise = torch.from_numpy(synth.tokens(synth.SEED_TOKENS, synth.tid_canvas_noise(rank), C, V))
    canvas = noise.to(dev)
    logits = torch.empty(C, V, device=dev)
    n_ren = dg.renoise_count(C, 1, 0, cfg["renoise_start"], cfg["renoise_end"])
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > 126 MB L2

    fused = args.fused_update
    if fused:
        # one call per step reads the canvas and writes the updated one in place: each step
        # denoises the previous step's result (the same shapes and work every step)
        canvas_in = canvas_out = canvas

        def step(s):
            dg.denoise_update(model, cache, canvas, n_ren, ws, seed=synth.SEED_RENOISE, step=s)
    else:
        # every step denoises the same input canvas; the update writes a second buffer
        canvas_in = canvas
        canvas_out = torch.empty_like(canvas)

        def step(s):
            dg.denoise_pass(model, cache, canvas_in, logits, ws)
            dg.canvas_update(logits, n_ren, synth.SEED_RENOISE, s, canvas_out, ws)

    # expert union per layer of this input (read once, outside the timed region)
    unions = torch.zeros(cfg["n_layers"], dtype=torch.int32, device=dev)
    model.set_taps({"unions": unions, "rows": C})
    step(0)
    model.set_taps(None)
    torch.cuda.synchronize(dev)
    unions_h = [int(u) for u in unions.cpu()]

    for w in range(args.warmup):
        step(w)
    dg.device_status(ws)

    def timed(K, profile):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        if profile:
            dg.profile_reset()
            dg.profile_enable(True)
        l0 = dg.launch_count()
        for s in range(K):
            flush.zero_()
            ev[s][0].record(stream)
            step(s)
            ev[s][1].record(stream)
        torch.cuda.synchronize(dev)
        if profile:
            dg.profile_enable(False)
        per = [a.elapsed_time(b) for a, b in ev]
        timed.last = per
        return sum(per), dg.launch_count() - l0

    ranks.barrier()
    torch.cuda.synchronize(dev)
    (total_ms, launches), clocks = clocked(ranks, dev, lambda: timed(args.steps, profile=False))
    dg.device_status(ws)
    total_ms = ranks.max(total_ms)
    ranks.barrier()

    step_median_us = statistics.median(timed.last) * 1e3
    step_p10_us, step_p90_us = (float(v) * 1e3 for v in np.percentile(timed.last, [10, 90]))

    # the pass alone (no update), same timing rules
    def pass_only(s):
        dg.denoise_pass(model, cache, canvas_in, logits, ws)
    k2 = min(args.steps, 500)
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k2)]
    for s_ in range(k2):
        flush.zero_()
        ev2[s_][0].record(stream)
        pass_only(s_)
        ev2[s_][1].record(stream)
    torch.cuda.synchronize(dev)
    pass_us = [a.elapsed_time(b) * 1e3 for a, b in ev2]

    # the step replayed from a CUDA graph (host launch cost removed), same flush rule
    graph = None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step(0)  # warm the capture stream
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g):
            step(0)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        ev3 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k2)]
        for s_ in range(k2):
            flush.zero_()
            ev3[s_][0].record(stream)
            g.replay()
            ev3[s_][1].record(stream)
        torch.cuda.synchronize(dev)
        dg.device_status(ws)
        gus = [a.elapsed_time(b) * 1e3 for a, b in ev3]
        graph = {"median_us": statistics.median(gus), "mean_us": sum(gus) / len(gus), "replays": k2}
        del g
    except Exception as e:  # report, do not fail the bench line
        graph = {"unavailable": repr(e)[:200]}

    # per-kernel breakdown with CUDA events on the launching stream (separate timed run,
    # at most 200 steps: it records an event pair around every launch)
    prof_ms, _ = timed(min(args.steps, 200), profile=True)
    kern = {}
    for kname in dg.KERNEL_KINDS:
        ms, n = dg.profile_read(kname)
        if n:
            kern[kname] = {"launches": n, "avg_us": ms * 1e3 / n, "share": ms / max(prof_ms, 1e-9)}

    # end to end through the public API with host buffers: H2D canvas, pass, update, D2H canvas
    h_in = noise.clone().pin_memory()
    h_out = torch.empty_like(h_in).pin_memory()
    e2e_ms = []
    for s in range(args.steps + args.warmup):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        canvas_in.copy_(h_in, non_blocking=True)
        step(s)
        h_out.copy_(canvas_out, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if s >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_total = ranks.max(sum(e2e_ms))

    ms_step = total_ms / args.steps
    value = job_value(world, C, args.steps, total_ms)
    e2e_value = job_value(world, C, args.steps, e2e_total)
    hbm, tf_burst, tf_sust, peak_src = _peaks()

    # whole-pass roofline (slower of FLOPs at the bf16 peak and bytes at HBM bandwidth)
    flops = RF.pass_flops(cfg, P, C)
    # the pass's bytes already hold the logits' write and the update's read of them; the
    # update adds its canvas in / out; the fused step writes and reads 16-byte tile records
    # (one per token and 128 vocabulary ids) instead of the logits
    nbytes = RF.pass_bytes(cfg, P, C, unions_h) + 8 * C
    if fused:
        nbytes += 2 * RF.update_record_bytes(cfg, C) - 2 * 4 * C * V
    t_roof = RF.time_bound(flops, nbytes, tf_burst * 1e12, hbm * 1e9)
    # every big kernel against its own bound: algorithmic units per launch / average
    # CUDA-event duration of its launches inside the step (the per-layer expert union
    # varies, so the expert GEMMs' bytes per launch are the layers' average)
    kroof = kernel_rooflines(cfg, P, C, unions_h, kern, hbm, tf_sust, peak_src, fused=fused)
    # the dominant kernel (largest share of the step) is the line's roofline
    roof = None
    if kroof:
        dom = max(kroof, key=lambda n: kern[n]["share"])
        roof = dict(kroof[dom], kernel=dom, traffic=_ncu_traffic(name, dom))

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "pass_latency_us": ms_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": DATA,
        "config": {"workload": _workload_desc(name, cfg), "l2": "flushed between steps (256 MB write)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "attention": _attention_kind(), "expert_union": unions_h,
                   "update": "fused into the vocabulary projection (one call per step)" if fused
                   else "two calls: logits written, then read by the update"},
        "roofline": roof,
        "pass_roofline": {"t_roof_us": t_roof * 1e6, "frac": t_roof * 1e3 / ms_step, "flops": flops,
                          "bytes": nbytes, "bound": "hbm" if nbytes / (hbm * 1e9) > flops / (tf_burst * 1e12)
                          else "tensor", "peak_source": peak_src},
        "kernels": kern,
        "kernel_rooflines": kroof,
        "step_median_us": step_median_us,
        "step_p10_p90_us": [step_p10_us, step_p90_us],
        "pass_only_us": {"median": statistics.median(pass_us), "mean": sum(pass_us) / len(pass_us), "steps": k2,
                         "note": "dg_denoise_pass alone (logits written), no update"},
        "graph_step_us": graph,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": C * 4, "d2h_bytes_per_step": C * 4},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    ranks.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
