"""Benchmark of the exact-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole path over one batch of synthetic inputs:
  1. attn_fwd, causal, on the LLaMA-7B-shaped prefill (B=2, H=32, N=2048, d=128)
  2. attn_fwd, non-causal, same shape
  3. attn_decode_splitkv + 4. attn_combine on single-query decode
     (B=1, Hq=32, Hkv=8, L=131072, d=128; the default split count).
The decode pair is timed as one interval (the combine is launched with
programmatic stream serialization, so its launch overlaps the decode's end).
After the timed loop every decode kernel is also timed alone, and the same
pair at L=32768 for B=1 and B=8 (L2 flushed before every launch); both are
reported beside the step's kernels.
The printed `value` is the causal prefill's TFLOPS (4*B*H*N^2*d/2 per launch
over the kernel's CUDA-event time, summed over all ranks); the decode's KV-read
GB/s is reported beside it. Inputs are seeded N(0,1) bf16, resident in HBM
before the timed region. The 537 MB KV stream of the decode (and a 256 MB
buffer write) run between consecutive prefill launches, so every launch starts
with a cold L2 (126 MB).

With N > 1 (launched under torch.distributed.run) every rank runs the same
per-GPU workload on its own batch (weak scaling, no data-path collective); the
elapsed time is the max over ranks.

--impl reference times the float64 CPU oracle (the checker) on the host cores
on a bounded sample of the same causal prefill workload; rank 0 only.

    python bench.py profile fwd|decode|merge|ring|bwd [--B ..] [--H ..] ...

runs one kernel of the library a few times on seeded inputs (no timing loop,
no oracle) and prints the CUDA-event time of the last launch: the command that
the ncu captures under profiles/ wrap.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import seeded_inputs as si  # noqa: E402

METRIC = "attn fwd TFLOPS (% BF16 TC peak); split-KV decode GB/s (% HBM peak)"
PREFILL = si.PrefillShape("llama7b B2 H32 N2048 d128", 2, 32, 32, 2048, 128, True, seed=1001)
PREFILL_NC = si.PrefillShape("llama7b B2 H32 N2048 d128 non-causal", 2, 32, 32, 2048, 128, False, seed=1001)
DECODE = si.DecodeShape("decode B1 Hq32 Hkv8 L131072 d128", 1, 32, 8, 131072, 128, seed=1004)
# every decode the bench times: (kernels key, shape); the first is the step's decode,
# the others are timed after the step loop
DECODES = [("decode", DECODE),
           ("decode_b1_l32k", si.DecodeShape("decode B1 Hq32 Hkv8 L32768 d128", 1, 32, 8, 32768, 128, seed=1005)),
           ("decode_b8_l32k", si.DecodeShape("decode B8 Hq32 Hkv8 L32768 d128", 8, 32, 8, 32768, 128, seed=1006))]
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch from one ncu capture, valid only for the kernel source
# it was taken on (sha256 of the kernel file, first 16 hex digits).
NCU_TRAFFIC = {
    # decode_splitkv_keys_kernel<16,3>: B1 Hq32 Hkv8 L131072 d128 (the step's decode) and the two
    # L32768 decodes; attn_fwd_kernel<128, causal / non-causal>: B2 H32 N2048 d128. Read + write
    # with cold caches (ncu flushes them before each captured launch); the prefill's O (33.5 MB)
    # mostly stays dirty in L2 when the kernel ends, so its write-back is not counted here.
    "decode": {"bytes_per_launch": 536959744 + 3461376, "source_sha": "eaaf414296e5590d"},
    "decode_b1_l32k": {"bytes_per_launch": 134302976 + 3129856, "source_sha": "eaaf414296e5590d"},
    "decode_b8_l32k": {"bytes_per_launch": 1073927168 + 3971072, "source_sha": "eaaf414296e5590d"},
    "attn_fwd_causal": {"bytes_per_launch": 141966080 + 13459968, "source_sha": "0fb1c2cb5c296374"},
    # the non-causal call is two launches at this shape (the plain kernel, then the last round in
    # 128-row halves): their sum
    "attn_fwd_noncausal": {"bytes_per_launch": 87900416 + 9707008 + 13959680 + 0, "source_sha": "0fb1c2cb5c296374"},
}


def kernel_sha(name: str) -> str:
    path = os.path.join(ROOT, "exact_attention_ring_b200", "csrc", name)
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, flag in zip(names, parts[5:9]):
                if flag.lower() in ("active", "1"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        loaded = [x for x in sm if x > 0.5 * (smax or max(sm))] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def physical_gpu(local: int) -> str:
    """nvidia-smi's id (index or UUID) of this process's CUDA device."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], device="cuda", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


# ----------------------------------------------------------------- our arm --

def measure_extra_paths(eab, q, k, v, o, lse, p, flush_l2, stream, iters=10, warm=3):
    """The backward pass and the FP8 forward on the prefill workload (causal),
    each timed alone with CUDA events after the timed step (L2 flushed before
    every launch); median of `iters` launches."""
    def timed(fn):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(iters):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return sorted(ts)[len(ts) // 2]

    do = si.make_dout(p.seed + 1, p.B, p.Hq, p.N, p.d).to(q.device)
    eab.attn_fwd(q, k, v, o, lse, True, p.scale, stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    delta = torch.empty_like(lse)
    t_bwd = timed(lambda: eab.attn_bwd(q, k, v, o, lse, do, delta, dq, dk, dv, True, p.scale, stream))
    q8, sq = eab.quantize_fp8(q, stream=stream)
    k8, sk = eab.quantize_fp8(k, stream=stream)
    vt8, sv = eab.quantize_fp8(v, per_plane=True, transpose=True, stream=stream)
    o8 = torch.empty_like(o)
    lse8 = torch.empty_like(lse)
    t_fp8 = timed(lambda: eab.attn_fwd_fp8(q8, k8, vt8, sq, sk, sv, o8, lse8, True, p.scale, stream))
    t_quant = timed(lambda: (eab.attn_quant_fp8(q, q8, sq, stream=stream), eab.attn_quant_fp8(k, k8, sk, stream=stream),
                             eab.attn_quant_fp8(v, vt8, sv, per_plane=True, transpose=True, stream=stream)))
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    return t_bwd, t_fp8, t_quant


def fwd_launch_count(B, Hq, N, causal, sms):
    """Kernel launches of one attn_fwd call: two for a non-causal problem whose
    last round of 256-row query blocks holds at most half as many blocks as
    there are SMs (and N spans two key tiles), whose tail runs as a second
    launch in 128-row halves; else one."""
    if causal:
        return 1
    rem = (B * Hq * ((N + 255) // 256)) % sms
    return 2 if ((N + 127) // 128 >= 2 and rem > 0 and 2 * rem <= sms) else 1


# Causal d = 128 prefill at the longer shapes of the sequence sweep and at the
# grouped-query shapes (B, Hq, Hkv, N): timed alone after the step like the
# extra paths, so that the bench line carries the causal rate beyond N = 2048.
CAUSAL_SWEEP = [(4, 16, 16, 4096), (2, 16, 16, 8192), (1, 16, 16, 16384), (1, 32, 8, 8192), (1, 32, 1, 8192)]


def measure_causal_sweep(eab, flush_l2, stream, tc_peak, iters=10, warm=3, seed=4242):
    out = []
    gen = torch.Generator(device="cuda")
    for (B, Hq, Hkv, N) in CAUSAL_SWEEP:
        d = 128
        gen.manual_seed(seed + N + Hkv)
        q = torch.randn(B, Hq, N, d, device="cuda", generator=gen).to(torch.bfloat16)
        k = torch.randn(B, Hkv, N, d, device="cuda", generator=gen).to(torch.bfloat16)
        v = torch.randn(B, Hkv, N, d, device="cuda", generator=gen).to(torch.bfloat16)
        o = torch.empty_like(q)
        lse = torch.empty(B, Hq, N, device="cuda")
        fn = lambda: eab.attn_fwd(q, k, v, o, lse, True, d ** -0.5, stream)
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(iters):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = sorted(ts)[len(ts) // 2]
        tf = 2.0 * B * Hq * N * N * d / (ms * 1e-3) / 1e12
        out.append({"workload": f"B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} causal", "ms": round(ms, 5),
                    "tflops": round(tf, 1), "frac": round(tf / tc_peak, 4)})
        del q, k, v, o, lse
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    return out


def run_ours(args):
    import exact_attention_ring_b200 as eab

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    # inputs resident in HBM before timing (rank-specific seeds: independent batches)
    p = PREFILL
    q, k, v = (t.to(dev) for t in si.make_qkv(p.seed + 17 * rank, p.B, p.Hq, p.Hkv, p.N, p.d))
    o = torch.empty_like(q)
    lse = torch.empty(p.B, p.Hq, p.N, device=dev)
    o2 = torch.empty_like(q)
    lse2 = torch.empty_like(lse)
    dc = DECODE
    dec_sets = []
    for name, shp in DECODES:
        qd, kd, vd = (t.to(dev) for t in si.make_decode(shp.seed + 17 * rank, shp.B, shp.Hq, shp.Hkv, shp.L, shp.d))
        Sd = eab.attn_decode_default_splits(shp.B, shp.Hq, shp.Hkv, shp.L)
        dec_sets.append(dict(name=name, shape=shp, q=qd, k=kd, v=vd, S=Sd,
                             o_part=torch.empty(shp.B, shp.Hq, Sd, shp.d, device=dev),
                             lse_part=torch.empty(shp.B, shp.Hq, Sd, device=dev),
                             o=torch.empty(shp.B, shp.Hq, shp.d, device=dev, dtype=torch.bfloat16),
                             lse=torch.empty(shp.B, shp.Hq, device=dev)))
    S = dec_sets[0]["S"]
    flush = torch.empty(L2_FLUSH_BYTES // 4, device=dev, dtype=torch.float32)
    flush_read = torch.ones(2 * L2_FLUSH_BYTES // 4, device=dev, dtype=torch.float32)  # 512 MB
    flush_sum = torch.empty((), device=dev, dtype=torch.float32)

    n_ev = 4
    def flush_l2():
        # write a buffer larger than L2, then read another: the next kernel starts
        # with none of its inputs in L2 and no dirty lines to write back
        flush.fill_(float(rank))
        torch.sum(flush_read, dim=0, out=flush_sum)

    def run_decode(ds, combine=True):
        # the pair back to back: the combine is launched with programmatic stream
        # serialization, so its launch overlaps the decode's last blocks
        eab.attn_decode_splitkv(ds["q"], ds["k"], ds["v"], ds["o_part"], ds["lse_part"], ds["S"],
                                ds["shape"].scale, stream)
        if combine:
            eab.attn_combine(ds["o_part"], ds["lse_part"], ds["o"], ds["lse"], stream)

    def median_ms(fn, n=10):
        # n launches of fn, each after a flush, timed alone: the median (every rank
        # runs the same launches)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for a, b in evs:
            flush_l2()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in evs), world)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        eab.attn_fwd(q, k, v, o, lse, True, p.scale, stream)
        if ev is not None:
            ev[1].record(stream)
        eab.attn_fwd(q, k, v, o2, lse2, False, p.scale, stream)
        if ev is not None:
            ev[2].record(stream)
        run_decode(dec_sets[0])
        if ev is not None:
            ev[3].record(stream)
        flush_l2()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(physical_gpu(local)) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(events[i])
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = max_over_ranks(start.elapsed_time(end), world)
    t_fwd_c = sum(e[0].elapsed_time(e[1]) for e in events) / args.steps
    t_fwd_n = sum(e[1].elapsed_time(e[2]) for e in events) / args.steps
    t_fwd_c, t_fwd_n = (max_over_ranks(x, world) for x in (t_fwd_c, t_fwd_n))
    # the step's decode + combine, as one interval (the metric's time)
    dec_sets[0]["t_pair"] = max_over_ranks(sum(e[2].elapsed_time(e[3]) for e in events) / args.steps, world)
    # after the loop: every decode kernel alone (for its roofline), and the L = 32768
    # decode + combine pairs; median of 10 launches, each after a flush
    for ds in dec_sets:
        for _ in range(3):
            run_decode(ds)
        ds["t_dec"] = median_ms(lambda: run_decode(ds, combine=False))
        if ds is not dec_sets[0]:
            ds["t_pair"] = median_ms(lambda: run_decode(ds))
    t_dec, t_pair = dec_sets[0]["t_dec"], dec_sets[0]["t_pair"]
    assert eab.attn_device_status() == 0
    assert eab.attn_device_status() == 0

    tflops_c = p.flops() / (t_fwd_c * 1e-3) / 1e12
    tflops_n = PREFILL_NC.flops() / (t_fwd_n * 1e-3) / 1e12
    kv_bytes = dc.kv_bytes()
    dec_gbs = kv_bytes / (t_pair * 1e-3) / 1e9
    dec_kernel_gbs = kv_bytes / (t_dec * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers (causal prefill).
    # Every step copies its inputs host -> device, runs attn_fwd and copies o and
    # lse back, as a caller streaming batches would: two device buffer sets, the
    # copies on their own streams (one per direction, separate copy engines) and
    # events between them, so step i's kernel and step i+1's input copy overlap.
    qh, kh, vh = (t.pin_memory() for t in si.make_qkv(p.seed + 17 * rank, p.B, p.Hq, p.Hkv, p.N, p.d))
    sets = [dict(q=q, k=k, v=v, o=o, lse=lse)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    host_out = [dict(o=torch.empty(q.shape, dtype=torch.bfloat16).pin_memory(),
                     lse=torch.empty(lse.shape, dtype=torch.float32).pin_memory()) for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of set b copied
    ev_done = [torch.cuda.Event() for _ in range(2)]  # kernel on set b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]   # outputs of set b copied out
    def e2e_run(n_steps, start_ev=None, end_ev=None):
        for i in range(n_steps):
            b = i & 1
            bs, ho = sets[b], host_out[b]
            with torch.cuda.stream(s_h2d):
                if i == 0 and start_ev is not None:
                    start_ev.record(s_h2d)
                if i >= 2:
                    s_h2d.wait_event(ev_done[b])  # the kernel two steps back has read this set
                bs["q"].copy_(qh, non_blocking=True)
                bs["k"].copy_(kh, non_blocking=True)
                bs["v"].copy_(vh, non_blocking=True)
                ev_in[b].record(s_h2d)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # its outputs have been copied out
            eab.attn_fwd(bs["q"], bs["k"], bs["v"], bs["o"], bs["lse"], True, p.scale, stream)
            ev_done[b].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_done[b])
                ho["o"].copy_(bs["o"], non_blocking=True)
                ho["lse"].copy_(bs["lse"], non_blocking=True)
                ev_out[b].record(s_d2h)
        if end_ev is not None:
            s_h2d.wait_stream(s_d2h)
            s_h2d.wait_stream(stream)
            end_ev.record(s_h2d)
    e2e_run(max(2, args.warmup))
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 20))
    barrier(world)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, s2, e2)
    torch.cuda.synchronize()
    oh, lh = host_out[(e2e_steps - 1) & 1]["o"], host_out[(e2e_steps - 1) & 1]["lse"]
    e2e_ms = max_over_ranks(s2.elapsed_time(e2) / e2e_steps, world)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    # ---- roofline of each kernel; the dominant one goes in "roofline"
    tc_peak = peaks["bf16_tflops"]
    hbm_peak = peaks["hbm_gbs"]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    fwd_sha = kernel_sha("attn_fwd_sm100.cuh")
    dec_sha = kernel_sha("decode_sm100.cuh")
    def traffic(name, sha):
        rec = NCU_TRAFFIC.get(name)
        return rec["bytes_per_launch"] if rec and rec["source_sha"] == sha else None
    roof_fwd = {"kernel": "attn_fwd_kernel<128,causal>", "bound": "tensor", "achieved": round(tflops_c, 1),
                "peak": tc_peak, "unit": "TFLOP/s", "frac": round(tflops_c / tc_peak, 4),
                "traffic": traffic("attn_fwd_causal", fwd_sha), "ms": round(t_fwd_c, 5),
                "peak_source": f"{peak_src} bf16_tflops (burst)"}
    nc_launches = fwd_launch_count(p.B, p.Hq, p.N, False, sms)
    roof_fwd_nc = {"kernel": "attn_fwd_kernel<128,noncausal>" + (" and its split last round (two launches, one "
                                                                  "event interval)" if nc_launches == 2 else ""),
                   "bound": "tensor", "achieved": round(tflops_n, 1),
                   "peak": tc_peak, "unit": "TFLOP/s", "frac": round(tflops_n / tc_peak, 4),
                   "traffic": traffic("attn_fwd_noncausal", fwd_sha), "ms": round(t_fwd_n, 5)}
    dec_roofs = {}
    for ds in dec_sets:
        shp = ds["shape"]
        gbs = shp.kv_bytes() / (ds["t_dec"] * 1e-3) / 1e9
        dec_roofs[ds["name"]] = {
            "kernel": "decode_splitkv_keys_kernel<16,3> (keys as tile rows)", "bound": "hbm", "achieved": round(gbs, 1),
            "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
            "traffic": traffic(ds["name"], dec_sha), "ms": round(ds["t_dec"], 5),
            "ms_with_combine": round(ds["t_pair"], 5),
            "with_combine_gbs": round(shp.kv_bytes() / (ds["t_pair"] * 1e-3) / 1e9, 1),
            "workload": f"B{shp.B} Hq{shp.Hq} Hkv{shp.Hkv} L{shp.L} d{shp.d}, {ds['S']} splits",
            "peak_source": f"{peak_src} hbm_gbs"}
    roof_dec = dec_roofs["decode"]
    for ds in dec_sets:
        dec_roofs[ds["name"]]["timed"] = ("kernel alone after the step loop, L2 flushed before each launch, median "
                                          "of 10; with the combine: " + ("the step's interval" if ds is dec_sets[0]
                                                                         else "the same, the pair back to back"))
    # the dominant kernel: the one that takes the most time in the step
    times = {"fwd_causal": t_fwd_c, "fwd_noncausal": t_fwd_n, "decode": t_pair}
    dominant = max(times, key=times.get)
    roofline = {"fwd_causal": roof_fwd, "fwd_noncausal": roof_fwd_nc, "decode": roof_dec}[dominant]

    # the backward pass and the FP8 forward, outside the timed step (one GPU only:
    # no collective runs on this path)
    extra = None
    if world == 1:
        try:
            t_bwd, t_fp8, t_quant = measure_extra_paths(eab, q, k, v, o, lse, p, flush_l2, stream)
            fl_bwd = 2.5 * p.flops()  # the five N x N x d products of the backward pass
            extra = {
                "note": "timed alone after the step, same prefill workload (causal), L2 flushed, median of 10",
                "backward": {"ms": round(t_bwd, 5), "tflops": round(fl_bwd / (t_bwd * 1e-3) / 1e12, 1),
                             "frac_bf16_peak": round(fl_bwd / (t_bwd * 1e-3) / 1e12 / tc_peak, 4),
                             "launches": "bwd_delta_kernel, bwd_tile_kernel dK/dV, bwd_tile_kernel dQ"},
                "fp8_forward": {"ms": round(t_fp8, 5), "tflops": round(p.flops() / (t_fp8 * 1e-3) / 1e12, 1),
                                "peak": round(2 * tc_peak, 1),
                                "peak_source": f"{peak_src} bf16_tflops x 2 (nominal fp8 / bf16 ratio)",
                                "frac": round(p.flops() / (t_fp8 * 1e-3) / 1e12 / (2 * tc_peak), 4),
                                "quant_ms_q_k_v": round(t_quant, 5)},
            }
        except Exception as exc:  # the headline line is printed regardless
            extra = {"error": f"{type(exc).__name__}: {exc}"}
        try:
            extra["prefill_causal_d128"] = {
                "note": "sequence-sweep and grouped-query shapes, bf16 N(0,1) drawn on the device; timed alone "
                        "after the step, L2 flushed before each launch, median of 10",
                "shapes": measure_causal_sweep(eab, flush_l2, stream, tc_peak)}
        except Exception as exc:
            extra["prefill_causal_d128"] = {"error": f"{type(exc).__name__}: {exc}"}

    cpu = cpu_baseline_sample(budget_s=args.cpu_budget) if (rank == 0 and world == 1 and not args.no_cpu) else None

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(tflops_c * world, 2),
            "unit": "TFLOPS",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1), bf16)",
            "config": {
                "workload": "prefill B2 H32 N2048 d128 causal (LLaMA-7B shape); step also runs the non-causal "
                            "prefill and split-KV decode + combine at B1 Hq32 Hkv8 L131072 d128; B1 and B8 "
                            "L32768 decodes are timed alone after the step loop",
                "prefill": {"B": p.B, "Hq": p.Hq, "Hkv": p.Hkv, "N": p.N, "d": p.d, "causal": True},
                "decode": {"B": dc.B, "Hq": dc.Hq, "Hkv": dc.Hkv, "L": dc.L, "d": dc.d, "num_splits": S},
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "l2": "flushed: between steps a 256 MB buffer write and then a 512 MB buffer read (> 126 MB L2), "
                      "so each prefill starts with a cold L2 holding no dirty lines; the step's decode K/V (537 MB) "
                      "is cold; the L32768 decodes get the same flush before each launch",
            },
            "decode": {"value": round(dec_gbs * world, 1), "unit": "GB/s", "kernel_gbs": round(dec_kernel_gbs, 1),
                       "frac_hbm": round(dec_kernel_gbs / hbm_peak, 4), "ms_decode": round(t_dec, 5),
                       "ms_decode_and_combine": round(t_pair, 5), "kv_bytes": kv_bytes,
                       "timing": "value: the step's decode + combine as one event interval; kernel_gbs: the "
                                 "decode kernel alone after the loop (flushed L2, median of 10)"},
            "prefill_noncausal": {"value": round(tflops_n * world, 2), "unit": "TFLOPS",
                                  "frac": round(tflops_n / tc_peak, 4)},
            "roofline": roofline,
            "kernels": {"fwd_causal": roof_fwd, "fwd_noncausal": roof_fwd_nc, **dec_roofs},
            "e2e": {"value": round(p.flops() * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOPS",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                    "pipeline": "per step: H2D of q,k,v, attn_fwd, D2H of o,lse; copies on their own streams, "
                                "so step i's kernel overlaps step i+1's input copy and step i-1's output copy"},
            "gpu_launches": (3 + fwd_launch_count(p.B, p.Hq, p.N, False, sms)) * args.steps,
            "extra_paths": extra,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
            "peaks": {"source": peak_src, "bf16_tflops": tc_peak, "hbm_gbs": hbm_peak},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------ oracle timing --

class OracleSampler:
    """Times the float64 oracle on whole (b, h) slices of the causal prefill
    workload (same seeded inputs as the GPU arm, drawn once), walking a fixed
    random order of the slices. The CPU baseline of our arm and the reference
    arm both time through this one sampler, so their figures are the same
    measurement (per-slice work is identical: every slice is 2048 causal rows)."""

    SLICES_PER_STEP = 4  # reference arm: slices timed per step

    def __init__(self):
        import oracle
        self.oracle = oracle
        p = PREFILL
        self.q, self.k, self.v = si.make_qkv(p.seed, p.B, p.Hq, p.Hkv, p.N, p.d)
        self.per_slice = 4.0 * p.N * (p.N + 1) / 2 * p.d  # causal: row i sees i+1 keys
        self.order = torch.randperm(p.B * p.Hq, generator=torch.Generator().manual_seed(5)).tolist()
        self.next = 0

    def time(self, n_slices, budget_s=float("inf")):
        """(flops, seconds, slices) for the next `n_slices` slices, stopping early
        once `budget_s` seconds of oracle time have been spent."""
        p = PREFILL
        done, elapsed = 0, 0.0
        while done < n_slices and elapsed < budget_s:
            sl = self.order[self.next % len(self.order)]
            self.next += 1
            rows = torch.arange(sl * p.N, (sl + 1) * p.N, dtype=torch.int64)
            t0 = time.perf_counter()
            self.oracle.attention(self.q, self.k, self.v, True, p.scale, rows=rows)
            elapsed += time.perf_counter() - t0
            done += 1
        return done * self.per_slice, elapsed, done


def cpu_baseline_sample(budget_s=15.0):
    smp = OracleSampler()
    smp.time(1)  # warm-up: thread pool and first-touch pages
    flops, secs, k = smp.time(PREFILL.B * PREFILL.Hq, budget_s)
    return {"value": flops / secs / 1e12, "unit": "TFLOPS", "cores": smp.oracle.hardware_threads(), "kind": "oracle",
            "sample": f"{k} of {PREFILL.B * PREFILL.Hq} (b,h) slices of the causal prefill B2 H32 N2048 d128, all "
                      f"2048 rows each ({secs:.1f} s of float64 CPU work, all host threads), after one warm-up slice"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    p = PREFILL
    smp = OracleSampler()
    for _ in range(args.warmup):
        smp.time(1)
    flops, secs = 0.0, 0.0
    for _ in range(args.steps):
        f, sec, _ = smp.time(OracleSampler.SLICES_PER_STEP)
        flops += f
        secs += sec
    val = flops / secs / 1e12
    cores = smp.oracle.hardware_threads()
    k = OracleSampler.SLICES_PER_STEP
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), bf16 widened to f64)",
        "config": {"workload": f"prefill B2 H32 N2048 d128 causal (LLaMA-7B shape); {k} (b,h) slices per step",
                   "prefill": {"B": p.B, "Hq": p.Hq, "Hkv": p.Hkv, "N": p.N, "d": p.d, "causal": True}},
        "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": f"{k} (b,h) slices (2048 causal rows each) of the causal prefill per step, "
                                   f"the same slice sampler as our arm's cpu_baseline"},
        "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------- profile cases --

def run_profile_case(argv):
    """One kernel of the library a few times on seeded inputs, for profilers
    (one kernel, a few launches, inputs larger than L2 but a few GB at most)."""
    import exact_attention_ring_b200 as eab
    ap = argparse.ArgumentParser(prog="bench.py profile")
    ap.add_argument("kernel", choices=["fwd", "decode", "merge", "ring", "bwd", "fp8"])
    ap.add_argument("--B", type=int, default=4)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=0)
    ap.add_argument("--N", type=int, default=2048)
    ap.add_argument("--L", type=int, default=131072)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--causal", type=int, default=1)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--world", type=int, default=4, help="ring: virtual ranks emulated on this GPU")
    a = ap.parse_args(argv)
    Hkv = a.Hkv or a.H
    dev = torch.device("cuda", 0)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    scale = a.d ** -0.5
    if a.kernel in ("fwd", "bwd", "ring", "fp8"):
        q, k, v = (t.to(dev) for t in si.make_qkv(1001, a.B, a.H, Hkv, a.N, a.d))
    if a.kernel == "fwd":
        o = torch.empty_like(q)
        lse = torch.empty(a.B, a.H, a.N, device=dev)
        fn = lambda: eab.attn_fwd(q, k, v, o, lse, bool(a.causal), scale)  # noqa: E731
        work = 4.0 * a.B * a.H * a.N * a.N * a.d / (2 if a.causal else 1)
    elif a.kernel == "fp8":
        # the forward on E4M3 codes (the three quantisations run once, before)
        q8, sq = eab.quantize_fp8(q)
        k8, sk = eab.quantize_fp8(k)
        vt8, sv = eab.quantize_fp8(v, per_plane=True, transpose=True)
        o = torch.empty_like(q)
        lse = torch.empty(a.B, a.H, a.N, device=dev)
        fn = lambda: eab.attn_fwd_fp8(q8, k8, vt8, sq, sk, sv, o, lse, bool(a.causal), scale)  # noqa: E731
        work = 4.0 * a.B * a.H * a.N * a.N * a.d / (2 if a.causal else 1)
    elif a.kernel == "merge":
        # one merge step of a ring: fp32 accumulator read and written, fp32 block
        # and the two LSE vectors read
        rows = a.B * a.H * a.N
        g = torch.Generator().manual_seed(1005)
        o_acc = torch.randn(rows, a.d, generator=g).to(dev)
        lse_acc = torch.randn(rows, generator=g).to(dev)
        o_blk = torch.randn(rows, a.d, generator=g).to(dev)
        lse_blk = torch.randn(rows, generator=g).to(dev)
        fn = lambda: eab.attn_merge(o_acc, lse_acc, o_blk, lse_blk)  # noqa: E731
        work = rows * (a.d * (4 + 4 + 4) + 4 * 3)
    elif a.kernel == "bwd":
        # the three launches of attn_bwd (Delta, dK/dV, dQ) on the forward's O, LSE;
        # FLOPs counted as the five N x N x d products of the backward pass
        do = si.make_dout(1002, a.B, a.H, a.N, a.d).to(dev)
        o, lse = eab.attention(q, k, v, bool(a.causal), scale)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        delta = torch.empty_like(lse)
        fn = lambda: eab.attn_bwd(q, k, v, o, lse, do, delta, dq, dk, dv, bool(a.causal), scale)  # noqa: E731
        work = 10.0 * a.B * a.H * a.N * a.N * a.d / (2 if a.causal else 1)
    elif a.kernel == "ring":
        # every virtual rank's steps of the ring, one after another on this GPU
        fn = lambda: eab.ring_attention_emulated(q, k, v, a.world, bool(a.causal), scale)  # noqa: E731
        work = 4.0 * a.B * a.H * a.N * a.N * a.d / (2 if a.causal else 1)
    else:
        qd, kd, vd = (t.to(dev) for t in si.make_decode(1004, a.B, a.H, Hkv, a.L, a.d))
        S = eab.attn_decode_default_splits(a.B, a.H, Hkv, a.L)
        o_part = torch.empty(a.B, a.H, S, a.d, device=dev)
        lse_part = torch.empty(a.B, a.H, S, device=dev)
        fn = lambda: eab.attn_decode_splitkv(qd, kd, vd, o_part, lse_part, S, scale)  # noqa: E731
        work = 2.0 * a.B * Hkv * a.L * a.d * 2
    for _ in range(a.iters):
        start.record()
        fn()
        end.record()
    torch.cuda.synchronize()
    assert eab.attn_device_status() == 0
    ms = start.elapsed_time(end)
    tensor = a.kernel in ("fwd", "ring", "bwd", "fp8")
    print(f"{a.kernel}: {ms:.4f} ms  {work / (ms * 1e-3) / (1e12 if tensor else 1e9):.1f} "
          f"{'TFLOPS' if tensor else 'GB/s'}")


def main():
    if len(sys.argv) > 1 and sys.argv[1] == "profile":
        run_profile_case(sys.argv[2:])
        return
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
