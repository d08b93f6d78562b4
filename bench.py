"""Benchmark of the fused attention hot path on B200.

One step = one causal GQA prefill forward through the C ABI on the workload
the headline metric is quoted on: B=4, Hq=32, Hkv=8, S_q=S_k=4096, d=128,
bf16 in/out, fp32 accumulation, scale 1/sqrt(128), seeded N(0,1) inputs.
FLOPs per step count the 128x128 tiles of a fixed grid that intersect the
causal band: 4*d*128*128 per tile (0.5669 TFLOP).  The same run also times
the int8-KV decode (B=16, Hq=32, Hkv=8, d=128, cache lengths U[1024,32768]
from seed 0; bytes = codes + scales + Q + O) and the KV quantiser on that
cache's 4,361,088 rows, each against its roofline.

Inputs of every timed launch are larger than L2 (126 MB): prefill reads
201 MB of Q/K/V, decode 576 MB of cache, the quantiser 1.1 GB; no flush.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun (N > 1) every rank runs its own replica of the workload (the
path shards by independent (sequence, head) units: no collective), and the
step time is the max over ranks.  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill attention TFLOP/s and int8-KV decode GB/s, as % of B200 roofline"
TILE = 128


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


KERNEL_SOURCES = {
    "prefill_tc_kernel<128,bf16>": ["prefill_tc.cu", "umma.cuh", "device.cuh", "layout.cuh"],
    "prefill_tc_kernel<128,int8>": ["prefill_tc.cu", "umma.cuh", "device.cuh", "layout.cuh"],
    "prefill_tc_kernel<64,bf16>": ["prefill_tc.cu", "umma.cuh", "device.cuh", "layout.cuh"],
    "decode_sk_kernel<128>": ["decode.cu", "device.cuh"],
    "decode_sk_kernel<128,bf16>": ["decode.cu", "device.cuh"],
    "compress_rows8_kernel<bf16,16>": ["quant.cu", "device.cuh"],
}


def measured_traffic(kernel):
    """DRAM bytes per launch from the committed ncu record, if the kernel's
    sources still hash the same as when the counters were taken; else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if kernel not in KERNEL_SOURCES or not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "flashattention_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    sha = h.hexdigest()[:16]
    for line in open(path):
        f = line.split()
        if len(f) >= 3 and not line.startswith("#") and f[0] == kernel and f[1] == sha:
            return int(f[2])
    return None


def band_tiles(s_q, s_k, causal, window):
    """128x128 tiles of a fixed grid that intersect the visible band of one
    (sequence, head), and the exact number of visible (query, key) pairs."""
    tiles = 0
    pairs = 0
    for qb in range((s_q + TILE - 1) // TILE):
        i0, i1 = qb * TILE, min(s_q, qb * TILE + TILE) - 1
        lo = max(0, i0 + s_k - s_q - window + 1) if window > 0 else 0
        hi = min(s_k, i1 + s_k - s_q + 1) if causal else s_k
        if hi > lo:
            tiles += (hi + TILE - 1) // TILE - lo // TILE
    for i in range(s_q):
        p = i + s_k - s_q
        lo = max(0, p - window + 1) if window > 0 else 0
        hi = min(s_k, p + 1) if causal else s_k
        pairs += max(0, hi - lo)
    return tiles, pairs


def prefill_flops(w):
    tiles, pairs = band_tiles(w.seqlen_q, w.seqlen_k, w.causal, w.window)
    per = w.batch * w.hq * 4 * w.d
    return per * tiles * TILE * TILE, per * pairs


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock, power and clock-event reasons of one GPU every
    5 ms from a background thread through NVML (the data nvidia-smi prints),
    and summarises the samples taken inside the marked timed region.  Falls
    back to an `nvidia-smi -lms 20` child process when NVML is unavailable."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []   # (time, sm_mhz, max_mhz, power_w, [reasons])
        self.window = None
        self.stop = None
        self.thread = None
        self.proc = None
        self.path = os.path.join("/tmp", f"fa_bench_clocks_{os.getpid()}.csv")

    def _nvml_loop(self, nv, h):
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.perf_counter(), float(sm), float(mx), pw,
                                     [n for n, bit in self.REASONS if rs & bit]))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
            ent = vis[self.dev] if self.dev < len(vis) else str(self.dev)
            h = (nv.nvmlDeviceGetHandleByUUID(ent) if ent.startswith(("GPU-", "MIG-"))
                 else nv.nvmlDeviceGetHandleByIndex(int(ent)))
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "20"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            except OSError:
                self.proc = None
        time.sleep(0.3)
        return self

    def mark(self, t0, t1):
        """The timed region, as perf_counter() times."""
        self.window = (t0, t1)

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            try:
                for line in open(self.path):
                    f = [x.strip() for x in line.split(",")]
                    if len(f) >= 7 and f[0].replace(".", "").isdigit():
                        rs = [n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                                 "sw_power_cap"), f[3:7]) if v.lower().startswith("active")]
                        self.samples.append((None, float(f[0]), float(f[1]),
                                             float(f[2]) if f[2].replace(".", "").isdigit() else 0.0, rs))
            except OSError:
                pass

    def summary(self):
        rows = self.samples
        if self.window is not None and rows and rows[0][0] is not None:
            t0, t1 = self.window
            inside = [r for r in rows if t0 <= r[0] <= t1]
            rows = inside or rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = sorted({n for r in rows for n in r[4]})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max(r[2] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": round(max(r[3] for r in rows), 1),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


# ---------------------------------------------------------------------------- GPU arm
def time_launches(fn, steps, warmup, torch, dist=None, clocks=None):
    """Warm up, then time exactly `steps` calls between barriers and
    synchronisations with CUDA events on the current stream; max over ranks.
    `clocks` (a ClockSampler) is told the host-side span of the timed region."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.mark(t0, time.perf_counter())
    if dist is not None:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, torch, "cuda")
    return ms / steps


def pipelined_e2e(torch, fa, w, host_in, host_out, steps, warmup, dist=None):
    """ms per step of host-to-host prefill steps (pinned copies in, the
    prefill, the copy out), pipelined over two device buffer sets."""
    dev = torch.device("cuda", torch.cuda.current_device())
    bufs = [[torch.empty_like(t, device=dev) for t in host_in] + [torch.empty(host_out.shape, dtype=host_out.dtype,
                                                                                device=dev)] for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_comp = torch.cuda.current_stream()
    done_in = [torch.cuda.Event() for _ in range(2)]
    done_comp = [torch.cuda.Event() for _ in range(2)]
    done_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def run(n):
        for i in range(n):
            j = i % 2
            q, k, v, o = bufs[j]
            with torch.cuda.stream(s_in):
                if started[j]:
                    s_in.wait_event(done_comp[j])  # the compute that read this buffer set is done
                for d, h in zip((q, k, v), host_in):
                    d.copy_(h, non_blocking=True)
                done_in[j].record(s_in)
            s_comp.wait_event(done_in[j])
            if started[j]:
                s_comp.wait_event(done_out[j])  # its previous output has left the device
            fa.attention_fwd(q, k, v, hq=w.hq, hkv=w.hkv, causal=True, out=o)
            done_comp[j].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_comp[j])
                host_out.copy_(o, non_blocking=True)
                done_out[j].record(s_out)
            started[j] = True

    run(warmup)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    run(steps)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, torch, "cuda")
    return ms / steps


def max_over_ranks(x: float, dist, torch, device) -> float:
    """The largest of every rank's x (the job is as slow as its slowest
    rank); x itself without a process group."""
    if dist is None:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def prefill_config(w, flops_tiles, flops_exact, world):
    """The headline step's config (the same dict on both arms)."""
    return {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv, "seq_len": w.seqlen_q,
            "head_dim": w.d, "causal": True, "window": 0, "epilogue": [],
            "flops_per_step": flops_tiles, "flops_counting": "128x128 tiles intersecting the band",
            "flops_exact_pairs": flops_exact, "l2": "inputs larger than L2 (201 MB), no flush",
            "parallelism": f"replicas x{world} (no collective)"}


def gpu_arm(args, rank, world, dist):
    import torch
    from flashattention_attention_b200 import fa, inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    w = inputs.gqa_causal_prefill()
    flops_tiles, flops_exact = prefill_flops(w)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    out = torch.empty_like(q)

    def prefill():
        fa.attention_fwd(q, k, v, hq=w.hq, hkv=w.hkv, causal=True, out=out)

    if args.only in ("decode", "quant"):
        return decode_and_quant(args, dev, peaks, world, dist, {})
    if args.only in ("prefill_int8", "varlen"):
        res = {}
        other_prefills(args, dev, peaks, world, dist, res)
        return res
    if args.only == "ring":
        res = {}
        ring_rank_steps(args, dev, peaks, world, dist, res)
        return res
    if args.only == "tq":
        res = {}
        turboquant_decode(args, dev, peaks, world, dist, res)
        return res
    l0 = fa.kernel_launches()
    with ClockSampler(dev.index or 0) as clocks:
        ms = time_launches(prefill, args.steps, args.warmup, torch, dist, clocks)
    launches = fa.kernel_launches() - l0 - args.warmup * 1
    clk = clocks.summary()
    assert fa.check_device_error() == fa.FA_OK
    tflops = flops_tiles / (ms * 1e-3) / 1e12

    # e2e: the same call with host buffers: every step copies its q/k/v from
    # pinned host memory, runs the prefill and copies the output back.  Steps
    # are pipelined over two buffer sets and three streams (copy in, compute,
    # copy out), so step i + 1's inputs cross PCIe while step i computes and
    # step i - 1's output returns; every copy of every timed step is inside
    # the timed region (events on the first copy-in and the last copy-out).
    hq_, hk_, hv_ = w.q.pin_memory(), w.k.pin_memory(), w.v.pin_memory()
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_ms = pipelined_e2e(torch, fa, w, (hq_, hk_, hv_), ho, max(3, args.steps // 10), 2, dist)
    h2d = sum(t.numel() * t.element_size() for t in (hq_, hk_, hv_))
    d2h = ho.numel() * ho.element_size()
    del q, k, v, out, hq_, hk_, hv_, ho
    torch.cuda.empty_cache()

    result = {
        "metric": METRIC, "value": round(tflops * world, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), numpy PCG64 -> fp32 -> bf16)",
        "config": prefill_config(w, flops_tiles, flops_exact, world),
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel<128,bf16>", "achieved": round(tflops, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tflops / peaks["bf16_tflops"], 4),
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "traffic": measured_traffic("prefill_tc_kernel<128,bf16>"),
                     "frac_of_nominal_2250": round(tflops / 2250.0, 4)},
        "e2e": {"value": round(flops_tiles / (e2e_ms * 1e-3) / 1e12 * world, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "schedule": "pinned host q/k/v -> device -> prefill -> out to pinned host every step; steps "
                            "pipelined over two buffer sets on copy-in / compute / copy-out streams"},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if args.only == "all":
        result["gqa_causal_prefill_paged"] = paged_prefill(args, w, flops_tiles, peaks, world, dist, dev)
        other_prefills(args, dev, peaks, world, dist, result)
        ring_rank_steps(args, dev, peaks, world, dist, result)
        decode_and_quant(args, dev, peaks, world, dist, result)
        turboquant_decode(args, dev, peaks, world, dist, result)
        if world > 1:
            ring_across_ranks(args, dev, peaks, world, dist, result)
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, flops_tiles, flops_exact, args.cpu_seconds)
    summarise(result)
    return result


def summarise(result):
    """A compact {workload: roofline fraction} table of every timed line,
    kept inside the headline roofline object and repeated as the line's last
    key (both places survive a reader that keeps only known keys or the end
    of the line)."""
    table = {"gqa_causal_prefill": {"frac": result["roofline"]["frac"], "achieved": result["roofline"]["achieved"],
                                    "unit": result["roofline"]["unit"]}}
    for key, val in result.items():
        if isinstance(val, dict) and isinstance(val.get("roofline"), dict) and "frac" in val["roofline"]:
            rf = val["roofline"]
            table[key] = {"frac": rf["frac"], "achieved": rf["achieved"], "unit": rf["unit"]}
            if "frac_of_nominal_8000" in rf:
                table[key]["frac_of_nominal_8000"] = rf["frac_of_nominal_8000"]
    result["roofline"]["all_workloads"] = table
    result["summary"] = table


def paged_prefill(args, w, flops_tiles, peaks, world, dist, dev):
    """The causal GQA prefill with K/V read from 256-token pages that a random
    permutation scatters over a pool (dense queries, per-sequence key counts)."""
    import torch
    from flashattention_attention_b200 import fa
    P = 256
    B, hkv, S, d = w.batch, w.hkv, w.seqlen_k, w.d
    mp = S // P
    perm = torch.randperm(B * mp, generator=torch.Generator().manual_seed(4)).to(dev)

    def pool_of(t):
        src = t.to(dev).view(B, hkv, mp, P, d).transpose(1, 2).reshape(B * mp, hkv, P, d)
        pool = torch.empty_like(src)
        pool[perm] = src
        return pool

    kp, vp = pool_of(w.k), pool_of(w.v)
    table = perm.view(B, mp).to(torch.int32).contiguous()
    cu_k = torch.arange(0, (B + 1) * S, S, dtype=torch.int32, device=dev)
    q = w.q.to(dev)
    out = torch.empty_like(q)

    def step():
        fa.attention_fwd_paged(q, kp, vp, cu_k, table, hq=w.hq, hkv=hkv, causal=True, out=out)

    ms = time_launches(step, max(20, args.steps // 2), args.warmup, torch, dist)
    assert fa.check_device_error() == fa.FA_OK
    tf = flops_tiles / (ms * 1e-3) / 1e12
    del kp, vp, q, out
    torch.cuda.empty_cache()
    return {"workload": w.name + "_paged256_shuffled", "value": round(tf * world, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "flops_per_step": flops_tiles,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4)}}


def varlen_flops(w):
    tiles = pairs = 0
    for L in w.lengths:
        t, pr = band_tiles(L, L, w.causal, w.window)
        tiles += t
        pairs += pr
    per = w.hq * 4 * w.d
    return per * tiles * TILE * TILE, per * pairs


def other_prefills(args, dev, peaks, world, dist, result):
    """The varlen sliding-window prefill (d=64, epilogue) and the long-context
    prefill over an int8 KV cache, each timed like the main step."""
    steps = max(10, args.steps // 4)

    if args.only != "prefill_int8":
        varlen_prefill(args, dev, peaks, world, dist, result, steps)
    if args.only != "varlen":
        int8_long_prefill(args, dev, peaks, world, dist, result, steps)


def varlen_prefill(args, dev, peaks, world, dist, result, steps):
    import torch
    from flashattention_attention_b200 import fa, inputs
    w = inputs.varlen_window_prefill()
    cu = inputs.cu_from_lengths(w.lengths).to(dev)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    out = torch.empty_like(q)
    ms = time_launches(lambda: fa.attention_fwd(q, k, v, hq=w.hq, hkv=w.hkv, causal=True, window=w.window,
                                                epilogue=w.epilogue, cu_seqlens_q=cu,
                                                max_seqlen_q=max(w.lengths), out=out),
                       steps, args.warmup, torch, dist)
    ft, fe = varlen_flops(w)
    tf = ft / (ms * 1e-3) / 1e12
    result["varlen_window_prefill"] = {
        "workload": w.name, "lengths": w.lengths, "value": round(tf * world, 2), "unit": "TFLOP/s",
        "flops_counting": "128x128 tiles intersecting the band", "flops_per_step": ft,
        "flops_exact_pairs": fe, "exact_pairs_tflops": round(fe / (ms * 1e-3) / 1e12, 2),
        "ms_per_step": round(ms, 4),
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel<64,bf16>", "achieved": round(tf, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tf / peaks["bf16_tflops"], 4),
                     "traffic": measured_traffic("prefill_tc_kernel<64,bf16>")}}
    del q, k, v, out


def int8_long_prefill(args, dev, peaks, world, dist, result, steps):
    import torch
    from flashattention_attention_b200 import fa, inputs
    w = inputs.int8kv_long_prefill(s=8192) if args.profile_small else inputs.int8kv_long_prefill()
    kc, ks = fa.compress_kv(w.k.to(dev))
    vc, vs = fa.compress_kv(w.v.to(dev))
    q = w.q.to(dev)
    out = torch.empty_like(q)
    ms = time_launches(lambda: fa.attention_fwd(q, kc, vc, k_scales=ks, v_scales=vs, hq=w.hq, hkv=w.hkv,
                                                causal=True, epilogue=w.epilogue, out=out),
                       steps, args.warmup, torch, dist)
    ft, fe = prefill_flops(w)
    tf = ft / (ms * 1e-3) / 1e12
    result["int8kv_long_prefill"] = {
        "workload": w.name, "value": round(tf * world, 2), "unit": "TFLOP/s",
        "flops_counting": "128x128 tiles intersecting the band", "flops_per_step": ft,
        "flops_exact_pairs": fe, "ms_per_step": round(ms, 4),
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel<128,int8>", "achieved": round(tf, 2),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tf / peaks["bf16_tflops"], 4),
                     "traffic": measured_traffic("prefill_tc_kernel<128,int8>")}}
    del q, kc, vc, ks, vs, out
    torch.cuda.empty_cache()


def ring_rank_steps(args, dev, peaks, world, dist, result):
    """The device work of the busiest rank of a 4-way context-parallel causal
    prefill (the last one: its own block causal, three earlier blocks in full),
    run through ring.attend_blocks (one fa_attention_fwd_acc per block, the
    merge inside the kernel's epilogue) on blocks already in this GPU's
    memory, i.e. without the block transfers.  For comparison: the same steps
    as partial results merged by the separate merge kernel, and that merge
    kernel alone (HBM-bound)."""
    import torch
    from flashattention_attention_b200 import fa, inputs, ring
    w = inputs.ring_cp_last_rank()
    R, blk = w.seqlen_k // w.seqlen_q, w.seqlen_q
    rank = R - 1
    q = w.q.to(dev)
    kb = [w.k[:, b * blk:(b + 1) * blk].contiguous().to(dev) for b in range(R)]
    vb = [w.v[:, b * blk:(b + 1) * blk].contiguous().to(dev) for b in range(R)]
    blocks = [((rank - s) % R, kb[(rank - s) % R], vb[(rank - s) % R]) for s in range(R)]
    steps = max(10, args.steps // 4)

    def step():
        ring.attend_blocks(q, blocks, rank=rank, n_blocks=R, hq=w.hq, hkv=w.hkv, causal=True)

    l0 = fa.kernel_launches()
    ms = time_launches(step, steps, args.warmup, torch, dist)
    launches = (fa.kernel_launches() - l0) / (steps + args.warmup)
    per = w.batch * w.hq * 4 * w.d * TILE * TILE
    flops = per * (band_tiles(blk, blk, True, 0)[0] + (R - 1) * band_tiles(blk, blk, False, 0)[0])
    tf = flops / (ms * 1e-3) / 1e12

    acc_o = torch.empty(q.shape, dtype=torch.float32, device=dev)
    acc_l = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    out = torch.empty_like(q)

    def unfused():
        acc_o.zero_()
        acc_l.fill_(float("-inf"))
        for b, k, v in blocks:
            if b <= rank:
                o, lse = fa.attention_fwd_lse(q, k, v, hq=w.hq, hkv=w.hkv, causal=b == rank)
                fa.attention_merge(acc_o, acc_l, o, lse)
        fa.attention_merge(acc_o, acc_l, out=out)

    ms_unfused = time_launches(unfused, steps, args.warmup, torch, dist)
    o, lse = fa.attention_fwd_lse(q, kb[0], vb[0], hq=w.hq, hkv=w.hkv)
    ms_merge = time_launches(lambda: fa.attention_merge(acc_o, acc_l, o, lse), steps, args.warmup, torch, dist)
    assert fa.check_device_error() == fa.FA_OK
    rows = q.shape[0] * q.shape[1]
    # o_acc read + written (fp32), o_part read (bf16), lse_acc read + written, lse_part read
    merge_bytes = rows * w.d * (4 + 4 + 2) + rows * 3 * 4
    gbs = merge_bytes / (ms_merge * 1e-3) / 1e9
    result["ring_cp4_last_rank"] = {
        "workload": w.name, "value": round(tf * world, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
        "flops_per_step": flops, "flops_counting": "128x128 tiles intersecting each block's band",
        "transfers": "not timed (blocks resident; one GPU)", "launches_per_step": launches,
        "roofline": {"bound": "tensor", "kernel": "prefill_tc_kernel<128,bf16> (accumulate)",
                     "achieved": round(tf, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tf / peaks["bf16_tflops"], 4)},
        "unfused_lse_then_merge": {"ms": round(ms_unfused, 4),
                                   "achieved": round(flops / (ms_unfused * 1e-3) / 1e12, 2), "unit": "TFLOP/s"},
        "merge_kernel": {"ms": round(ms_merge, 4), "bytes": merge_bytes,
                         "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                                      "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4)}}}
    del q, kb, vb, blocks, o, lse, acc_o, acc_l, out
    torch.cuda.empty_cache()


def ring_job_flops(world, block=4096, batch=4, hq=32, d=128):
    """FLOPs of the causal prefill over world * block positions that the
    ring computes (128x128 tiles intersecting the band), all ranks together."""
    S = world * block
    return batch * hq * 4 * d * TILE * TILE * band_tiles(S, S, True, 0)[0]


def ring_across_ranks(args, dev, peaks, world, dist, result):
    """The context-parallel ring itself on N GPUs: each rank holds one
    4096-position block of every sequence (B=4, Hq=32, Hkv=8, d=128, causal)
    and ring.ring_attention_fwd passes the K/V blocks around the ranks with
    NCCL point-to-point sends between the ranks' own memory (no peer loads,
    no multicast) while each step's kernel merges its block in the
    epilogue.  Each rank draws its own block (seed = rank).  The step time
    is the max over ranks; value is the whole causal attention over N * 4096
    positions divided by it."""
    import torch
    from flashattention_attention_b200 import fa, inputs, ring
    rank = dist.get_rank()
    w = inputs.dense_prefill(f"ring_block{rank}", batch=4, hq=32, hkv=8, s_q=4096, s_k=4096, d=128,
                             dtype=torch.bfloat16, causal=True, seed=100 + rank)
    q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
    steps = max(10, args.steps // 4)

    def step():
        ring.ring_attention_fwd(q, k, v, hq=w.hq, hkv=w.hkv, causal=True, group=dist.group.WORLD)

    try:
        ms = time_launches(step, steps, args.warmup, torch, dist)
        assert fa.check_device_error() == fa.FA_OK
        flops = ring_job_flops(world)
        tf = flops / (ms * 1e-3) / 1e12
        result["ring_cp_across_ranks"] = {
            "workload": f"ring_cp{world}_causal_b4_hq32_hkv8_block4096_d128_bf16", "value": round(tf, 2),
            "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "nccl_ranks": world, "flops_per_step": flops,
            "flops_counting": "128x128 tiles of the whole causal band over all ranks' positions",
            "transfers": "NCCL point-to-point K/V blocks between ranks, timed",
            "roofline": {"bound": "tensor", "achieved": round(tf / world, 2), "per": "GPU", "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / world / peaks["bf16_tflops"], 4)}}
    except Exception as e:  # reported in the line, never fatal to it
        result["ring_cp_across_ranks"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    del q, k, v
    torch.cuda.empty_cache()


def turboquant_decode(args, dev, peaks, world, dist, result):
    """The decode workload's cache (B=16, Hq=32, Hkv=8, d=128, lengths
    U[1024, 32768]) compressed TurboQuant K4/V2; one decode step timed (the
    split kernel and the merge + inverse rotation), and the compression of
    the whole cache."""
    import torch
    from flashattention_attention_b200 import fa, inputs
    w = inputs.int8kv_decode(batch=4) if args.profile_small else inputs.int8kv_decode()
    s = inputs.rotation_signs(w.d, 0).to(dev)
    lk, lv = fa.tq_codebook(w.d, 4).to(dev), fa.tq_codebook(w.d, 2).to(dev)
    k, v = w.k.to(dev), w.v.to(dev)
    kc, kn = fa.tq_compress(k, s, lk, 4)
    vc, vn = fa.tq_compress(v, s, lv, 2)
    steps = max(20, args.steps // 2)
    rows = k.shape[0] * k.shape[1]
    ms_c = time_launches(lambda: fa.tq_compress(k, s, lk, 4, codes=kc, norms=kn), max(10, steps // 4), args.warmup,
                         torch, dist)
    c_bytes = rows * (w.d * 2 + w.d * 4 // 8 + 4)
    del k, v
    torch.cuda.empty_cache()
    q = w.q.reshape(-1, w.d).to(dev)
    lens = torch.tensor(w.lengths, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    ws = torch.empty(fa.tq_decode_workspace_size(w.batch, w.hq, w.d, kc.shape[1]), dtype=torch.uint8, device=dev)

    def step():
        fa.tq_attention_decode(q, kc, kn, vc, vn, lens, hq=w.hq, hkv=w.hkv, k_bits=4, v_bits=2, k_levels=lk,
                               v_levels=lv, signs=s, out=out, workspace=ws)

    ms = time_launches(step, steps, args.warmup, torch, dist)
    assert fa.check_device_error() == fa.FA_OK
    keys = int(sum(w.lengths))
    per_key = (w.d * 4 // 8 + 4) + (w.d * 2 // 8 + 4)
    dec_bytes = keys * w.hkv * per_key + 2 * q.numel() * 2
    gbs = dec_bytes / (ms * 1e-3) / 1e9
    cgbs = c_bytes / (ms_c * 1e-3) / 1e9
    result["turboquant_k4v2_decode"] = {
        "workload": w.name + "_tq_k4v2", "value": round(gbs * world, 1), "unit": "GB/s",
        "us_per_step": round(ms * 1e3, 2), "bytes_per_step": dec_bytes,
        "bytes_counting": "K (d/2 + 4) and V (d/4 + 4) bytes per (key, KV head), q and out",
        "roofline": {"bound": "hbm", "kernel": "tq_decode_kernel<128,4,2,4> + tq_merge_kernel<128>",
                     "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 4)},
        "compress_k4": {"us": round(ms_c * 1e3, 2), "rows": rows, "bytes": c_bytes, "achieved": round(cgbs, 1),
                        "unit": "GB/s", "frac": round(cgbs / peaks["hbm_gbs"], 4)}}
    del kc, kn, vc, vn, q, out, ws
    torch.cuda.empty_cache()


def decode_and_quant(args, dev, peaks, world, dist, result):
    """int8-KV decode and the quantiser on the decode workload."""
    import torch
    from flashattention_attention_b200 import fa, inputs
    dw = inputs.int8kv_decode(batch=4) if args.profile_small else inputs.int8kv_decode()
    if args.only in ("all", "quant"):
        # the quantiser over every valid (token, kv-head) row of K and V, packed
        rows = torch.cat([t[b * dw.hkv:(b + 1) * dw.hkv, :dw.lengths[b]].reshape(-1, dw.d)
                          for t in (dw.k, dw.v) for b in range(dw.batch)]).to(dev)
        codes = torch.empty(rows.shape, dtype=torch.int8, device=dev)
        scales = torch.empty(rows.shape[0], dtype=torch.float32, device=dev)
        quant_ms = time_launches(lambda: fa.compress_kv(rows, codes, scales), max(10, args.steps // 4),
                                 args.warmup, torch, dist)
        quant_rows = int(rows.shape[0])
        quant_bytes = quant_rows * (2 * dw.d + dw.d + 4)
        quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
        result["quantiser"] = {"rows": quant_rows, "value": round(quant_gbs * world, 1), "unit": "GB/s",
                               "us_per_step": round(quant_ms * 1e3, 2), "bytes_per_step": quant_bytes,
                               "roofline": {"bound": "hbm", "kernel": "compress_rows8_kernel<bf16,16>",
                                            "achieved": round(quant_gbs, 1), "peak": peaks["hbm_gbs"],
                                            "unit": "GB/s", "frac": round(quant_gbs / peaks["hbm_gbs"], 4),
                                            "traffic": measured_traffic("compress_rows8_kernel<bf16,16>")}}
        del rows, codes, scales
    if args.only in ("all", "decode"):
        kc, ks = fa.compress_kv(dw.k.to(dev))
        vc, vs = fa.compress_kv(dw.v.to(dev))
        torch.cuda.synchronize()
        torch.cuda.empty_cache()  # the bf16 copies are gone: only the int8 cache stays resident
        lens = torch.tensor(dw.lengths, dtype=torch.int32, device=dev)
        dq = dw.q.reshape(-1, dw.d).to(dev)
        dout = torch.empty_like(dq)
        ws = torch.empty(fa.decode_workspace_size(dw.batch, dw.hq, dw.cache_capacity, dw.d),
                         dtype=torch.uint8, device=dev)
        maxlen = max(dw.lengths)

        def decode():
            fa.attention_decode(dq, kc, vc, lens, hq=dw.hq, hkv=dw.hkv, k_scales=ks, v_scales=vs,
                                max_seqlen=maxlen, workspace=ws, out=dout)

        dec_ms = time_launches(decode, max(20, args.steps), args.warmup, torch, dist)
        dec_bytes = sum(dw.lengths) * dw.hkv * 2 * (dw.d + 4) + 2 * dq.numel() * 2
        dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9
        result["decode"] = {"workload": dw.name, "value": round(dec_gbs * world, 1), "unit": "GB/s",
                            "us_per_step": round(dec_ms * 1e3, 2), "bytes_per_step": dec_bytes,
                            "roofline": {"bound": "hbm", "kernel": "decode_sk_kernel<128> (merge fused) + decode_plan_kernel",
                                         "achieved": round(dec_gbs, 1), "peak": peaks["hbm_gbs"],
                                         "unit": "GB/s", "frac": round(dec_gbs / peaks["hbm_gbs"], 4),
                                         "frac_of_nominal_8000": round(dec_gbs / 8000.0, 4),
                                         "traffic": measured_traffic("decode_sk_kernel<128>")}}
        result["decode_paged"] = decode_paged(args, dw, dq, dout, ws, kc, vc, ks, vs, lens, maxlen, dec_bytes,
                                              peaks, world, dist)
        result["decode_step_graph"] = decode_step_graph(args, dw, dq, dout, ws, kc, vc, ks, vs, peaks, world, dist)
        del kc, vc, ks, vs
        torch.cuda.empty_cache()
        # the same decode over an uncompressed bf16 cache (2 * 2d bytes per key and KV head)
        kb, vb = dw.k.to(dev), dw.v.to(dev)

        def decode_bf16():
            fa.attention_decode(dq, kb, vb, lens, hq=dw.hq, hkv=dw.hkv, max_seqlen=maxlen, workspace=ws, out=dout)

        bf_ms = time_launches(decode_bf16, max(20, args.steps), args.warmup, torch, dist)
        bf_bytes = sum(dw.lengths) * dw.hkv * 2 * (2 * dw.d) + 2 * dq.numel() * 2
        bf_gbs = bf_bytes / (bf_ms * 1e-3) / 1e9
        result["decode_bf16"] = {"workload": dw.name.replace("int8kv", "bf16kv"), "value": round(bf_gbs * world, 1),
                                 "unit": "GB/s", "us_per_step": round(bf_ms * 1e3, 2), "bytes_per_step": bf_bytes,
                                 "roofline": {"bound": "hbm", "kernel": "decode_sk_kernel<128,bf16> + decode_plan_kernel",
                                              "achieved": round(bf_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                              "frac": round(bf_gbs / peaks["hbm_gbs"], 4),
                                              "traffic": measured_traffic("decode_sk_kernel<128,bf16>")}}
        del kb, vb
        torch.cuda.empty_cache()
    assert fa.check_device_error() == fa.FA_OK
    return result


def decode_paged(args, dw, dq, dout, ws, kc, vc, ks, vs, lens, maxlen, dec_bytes, peaks, world, dist):
    """The int8-KV decode over the same cache cut into 256-token pages that a
    random permutation scatters over a pool, read through a block table (the
    same keys and bytes as the dense decode)."""
    import torch
    from flashattention_attention_b200 import fa
    P = 256
    B, hkv, cap, d = dw.batch, dw.hkv, dw.cache_capacity, dw.d
    mp = cap // P
    perm = torch.randperm(B * mp, generator=torch.Generator().manual_seed(3)).cuda()

    def pool_of(t, tail):
        src = t.view(B, hkv, mp, P, *tail).transpose(1, 2).reshape(B * mp, hkv, P, *tail)
        pool = torch.empty_like(src)
        pool[perm] = src
        return pool

    kp, vp = pool_of(kc, (d,)), pool_of(vc, (d,))
    ksp, vsp = pool_of(ks, ()), pool_of(vs, ())
    table = perm.view(B, mp).to(torch.int32).contiguous()

    def decode():
        fa.attention_decode_paged(dq, kp, vp, lens, table, hq=dw.hq, hkv=hkv, k_scales=ksp, v_scales=vsp,
                                  max_seqlen=maxlen, workspace=ws, out=dout)

    ms = time_launches(decode, max(20, args.steps), args.warmup, torch, dist)
    assert fa.check_device_error() == fa.FA_OK
    gbs = dec_bytes / (ms * 1e-3) / 1e9
    del kp, vp, ksp, vsp
    torch.cuda.empty_cache()
    return {"workload": dw.name + "_paged256_shuffled", "value": round(gbs * world, 1), "unit": "GB/s",
            "us_per_step": round(ms * 1e3, 2), "bytes_per_step": dec_bytes,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4)}}


def decode_step_graph(args, dw, dq, dout, ws, kc, vc, ks, vs, peaks, world, dist):
    """One decode step of the int8-KV workload as a captured CUDA graph: append
    the step's new K/V rows at the device-side cur_pos (quantised on the way
    in), decode over cache_seqlens = cur_pos + 1, advance cur_pos.  Each
    replay is a new step (the cache grows by one token per sequence)."""
    import numpy as np
    import torch
    from flashattention_attention_b200 import fa
    rng = np.random.default_rng(5)
    rows = dw.batch * dw.hkv
    kn = torch.from_numpy(rng.standard_normal((rows, dw.d)).astype(np.float32)).bfloat16().cuda()
    vn = torch.from_numpy(rng.standard_normal((rows, dw.d)).astype(np.float32)).bfloat16().cuda()
    lens0 = torch.tensor(dw.lengths, dtype=torch.int32)
    cur = lens0.cuda()
    lens = lens0.cuda()

    def step():
        fa.kv_append(kn, vn, kc, vc, cur, hkv=dw.hkv, k_scales=ks, v_scales=vs, cache_seqlens=lens)
        fa.attention_decode(dq, kc, vc, lens, hq=dw.hq, hkv=dw.hkv, k_scales=ks, v_scales=vs,
                            max_seqlen=dw.cache_capacity, workspace=ws, out=dout)
        cur.add_(1)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    steps = max(20, args.steps)
    if int(lens0.max()) + 1 + steps + args.warmup + 1 > dw.cache_capacity:
        steps = dw.cache_capacity - int(lens0.max()) - args.warmup - 2
    start = int(cur[0].item()) - dw.lengths[0]  # steps already taken (warm-up on the side stream)
    ms = time_launches(graph.replay, steps, args.warmup, torch, dist)
    assert fa.check_device_error() == fa.FA_OK
    # bytes: each timed step reads every cached key (codes + scales) once, Q, and
    # writes O, plus the append (bf16 rows in, codes + scales out)
    first = start + args.warmup
    keys = sum((sum(dw.lengths) + dw.batch * (first + s + 1)) for s in range(steps)) / steps
    step_bytes = keys * dw.hkv * 2 * (dw.d + 4) + 2 * dq.numel() * 2 + 2 * rows * (2 * dw.d + dw.d + 4)
    gbs = step_bytes / (ms * 1e-3) / 1e9
    del graph
    return {"workload": dw.name + "_append_decode_graph", "value": round(gbs * world, 1), "unit": "GB/s",
            "us_per_step": round(ms * 1e3, 2), "bytes_per_step": int(step_bytes),
            "launches_per_step": "append + plan + decode + position advance, one graph replay",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4)}}


# ---------------------------------------------------------------------------- CPU oracle
def _oracle_sample(w, n_rows, seed):
    """Time the fp64 oracle, as it stands, on n_rows random causal rows of
    one head plane of the prefill workload (its cost is per row).  Returns
    (seconds, visible pairs)."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(seed)
    qf = w.q[0:1].double().numpy()
    kf = w.k[0:1].double().numpy()
    vf = w.v[0:1].double().numpy()
    rows = [(0, 0, int(i)) for i in rng.integers(0, w.seqlen_q, n_rows)]
    t0 = time.perf_counter()
    oracle.attention(qf, kf, vf, hq=1, hkv=1, causal=True, rows=rows)
    dt = time.perf_counter() - t0
    return dt, sum(i + 1 for _, _, i in rows)


def _cores():
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return int(os.environ.get("OMP_NUM_THREADS", cores))


def _oracle_rows_for(w, seconds, seed):
    """Rows of an oracle sample that takes about `seconds` on these cores:
    calibrated on 1024 rows (enough that fixed costs do not dominate), then
    re-measured once at the estimated size."""
    n = 1024
    dt, _ = _oracle_sample(w, n, seed)
    for s in (seed + 1, seed + 2):
        n = int(min(4_000_000, max(1024, n * seconds / max(dt, 1e-4))))
        dt, _ = _oracle_sample(w, n, s)
        if dt >= 0.5 * seconds:
            break
    return int(min(4_000_000, max(1024, n * seconds / max(dt, 1e-4))))


def _oracle_rate(w, flops_tiles, flops_exact, dt, pairs):
    """The sample's rate expressed in the step's metric: TFLOP/s of the
    whole step (tile count) if the oracle ran it at the sample's pace."""
    return flops_tiles / (dt * flops_exact / (4 * w.d * pairs)) / 1e12


def _single_core_rate(w, flops_tiles, flops_exact, seconds):
    """The same oracle on one core (a child process with OMP_NUM_THREADS=1,
    so the thread count is fixed before its OpenMP runtime starts)."""
    code = ("import json, sys; sys.path.insert(0, %r); import bench; from flashattention_attention_b200 import inputs; "
            "w = inputs.gqa_causal_prefill(); n = bench._oracle_rows_for(w, %f, 11); "
            "dt, pairs = bench._oracle_sample(w, n, 14); print(json.dumps([n, dt, pairs]))" % (ROOT, seconds))
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                           timeout=30 * seconds + 120)
        n, dt, pairs = json.loads(r.stdout.strip().splitlines()[-1])
    except Exception as e:  # reported, never fatal to the GPU line
        return {"error": f"single-core sample failed: {type(e).__name__}"}
    return {"value": _oracle_rate(w, flops_tiles, flops_exact, dt, pairs), "unit": "TFLOP/s", "cores": 1,
            "sample": f"{n} random causal rows of one head plane ({pairs} visible pairs, {dt:.2f} s)"}


def cpu_baseline(w, flops_tiles, flops_exact, budget_s):
    """The oracle on the host cores over a bounded sample (about budget_s
    seconds of CPU work) sized exactly as the reference arm sizes its steps,
    scaled to the whole step by the exact pair count; and on one core."""
    n = _oracle_rows_for(w, budget_s, 1)
    dt, pairs = _oracle_sample(w, n, 4)
    full_s = dt * flops_exact / (4 * w.d * pairs)
    return {"value": flops_tiles / full_s / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": f"{n} random causal rows of one head plane ({pairs} visible pairs, {dt:.2f} s of fp64 "
                      f"CPU work), scaled to the whole step by its exact pair count",
            "seconds_sampled": round(dt, 3),
            "single_core": _single_core_rate(w, flops_tiles, flops_exact, max(2.0, budget_s / 4))}


def reference_arm(args, world):
    """The oracle timed on host cores on this arm's workload, metric and unit.
    Every step is the same bounded sample size (rows chosen once, during
    warm-up, so a step takes about --ref-step-seconds), and the line's
    ms_per_step is the measured time of those sampled steps; value is the
    sampled rate expressed for the whole step (exact pair count scaling)."""
    from flashattention_attention_b200 import inputs
    w = inputs.gqa_causal_prefill()
    flops_tiles, flops_exact = prefill_flops(w)
    n = _oracle_rows_for(w, args.ref_step_seconds, 1)
    times, rates = [], []
    for s in range(args.warmup + args.steps):
        dt, pairs = _oracle_sample(w, n, 100 + s)
        if s >= args.warmup:
            times.append(dt)
            rates.append(_oracle_rate(w, flops_tiles, flops_exact, dt, pairs))
    value = statistics.median(rates)
    ms = statistics.mean(times) * 1e3
    sample = (f"each step: {n} random causal rows of one head plane, fp64 (about {args.ref_step_seconds:g} s), "
              f"scaled to the whole step by its exact pair count")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "ms_per_step_is": "measured time of one sampled step (not the whole workload)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1), numpy PCG64 -> fp32 -> bf16)",
            "config": prefill_config(w, flops_tiles, flops_exact, world),
            "rows_per_sampled_step": n,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=2.0,
                    help="oracle seconds per sampled step of --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-small", action="store_true",
                    help="profiler captures: the int8-KV long prefill at S=8192 and the decodes (int8, bf16, "
                         "TurboQuant) over 4 of the 16 sequences (same kernels, inputs still larger than L2)")
    ap.add_argument("--only", default="all", choices=["all", "prefill", "decode", "quant", "prefill_int8", "varlen", "ring", "tq"],
                    help="time one part only (used for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # rank 0 alone times the CPU oracle; other ranks exit without work
        if rank == 0:
            print(json.dumps(reference_arm(args, world)), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        res = gpu_arm(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
