"""Benchmark of the exact-attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workloads (seeded synthetic N(0,1) bf16 inputs; the pages' own benchmark,
fp16/bf16 x head dim 64/128 x sequence 512..16k, ships no data):

* headline step: forward + backward of causal attention, B=2, Hq=Hkv=32,
  S=8192, D=128 (q, k, v, dO resident in HBM; 402 MB of q/k/v, larger than
  the 126 MB L2, so no flush is needed between steps). FLOPs are counted as
  4*D per visible (query, key) pair for the forward and 10*D for the
  backward; masked pairs are not counted.
* varlen forward: 65536 packed tokens, GQA 32/8, window (4096, 0), softcap 50.
* paged decode: B=64, GQA 32/8, D=128, cache lengths 1024..32768, page 256,
  num_splits 1, 4, 16; algorithmic bytes = every visible K and V row once.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
torch.cuda.synchronize(), measured with CUDA events on the launching stream;
with N > 1 ranks (torchrun) every rank runs its own replica and the maximum
time over ranks is used. SM clocks and throttle reasons are sampled through
NVML during the timed region.

`--impl reference` times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on rank 0.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import attn_workloads as W  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    out = dict(PEAKS_FALLBACK)
    out["source"] = "fallback"
    return out


def kernel_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the last ncu capture recorded in
    profiles/kernel_traffic.json, or None when the kernel's source files have
    changed since that capture (their SHA-256 no longer matches)."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "kernel_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    h = hashlib.sha256()
    for rel in rec["source_files"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec["source_sha256"]:
        return None
    return {"bytes_per_launch": rec["dram_bytes_per_launch"], "workload": rec["workload"]}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only: no data-path collective)
# ---------------------------------------------------------------------------
class Dist:
    """One process per GPU (torchrun env vars). Every rank runs its own
    replica of the workload; the process group is used only for barriers and
    the max-over-ranks of the timings (NCCL on GPUs, gloo on CPU)."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.backend = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            self.backend = "nccl" if torch.cuda.is_available() else "gloo"
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.01)

    def start(self):
        if self.ok:
            self._stop.clear()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def replica_throughput(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput of N independent replicas: all ranks' units over
    the slowest rank's time (units per second)."""
    return world * units_per_rank / (ms_max * 1e-3)


def timed(fn, steps, warmup, dist: Dist, sampler: ClockSampler | None = None, fa_mod=None):
    """Run fn() warmup times, then time `steps` calls with CUDA events on the
    current stream; returns max-over-ranks milliseconds per call. With
    `fa_mod`, the library's per-kernel event timing is switched on for the
    timed calls only (reset first, so the records cover exactly those)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if fa_mod is not None:
        fa_mod.fa_kernel_timing_reset()
        fa_mod.fa_kernel_timing_enable(True)
    if sampler is not None:
        sampler.start()
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    if fa_mod is not None:
        fa_mod.fa_kernel_timing_enable(False)
    if sampler is not None:
        sampler.stop()
    dist.barrier()
    ms = start.elapsed_time(end) / steps
    return dist.max(ms)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def e2e_pipeline(fa, c, inp, have_bwd, steps, dist: Dist):
    """Milliseconds per step of fwd (+ bwd) through the public API with the
    inputs copied in from pinned host memory and o, dq, dk, dv copied back,
    every step, pipelined over two buffer sets (see the caller)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    names = ("q", "k", "v", "do")
    host_in = {n: inp[n].pin_memory() for n in names}
    bufs = []
    for _ in range(2):
        b = {n: torch.empty_like(inp[n], device=dev) for n in names}
        b["out"] = torch.empty_like(b["q"])
        b["lse"] = torch.empty((c.B, c.Hq, c.S), dtype=torch.float32, device=dev)
        b["dq"], b["dk"], b["dv"] = torch.empty_like(b["q"]), torch.empty_like(b["k"]), torch.empty_like(b["v"])
        b["ws"] = torch.empty(fa.fa_bwd_workspace_size(c.B, c.Hq, c.S, c.D), dtype=torch.uint8, device=dev)
        b["h_out"] = torch.empty(b["q"].shape, dtype=b["q"].dtype).pin_memory()
        b["h_dq"] = torch.empty(b["q"].shape, dtype=b["q"].dtype).pin_memory()
        b["h_dk"] = torch.empty(b["k"].shape, dtype=b["k"].dtype).pin_memory()
        b["h_dv"] = torch.empty(b["v"].shape, dtype=b["v"].dtype).pin_memory()
        for e in ("in_ready", "fwd_done", "done", "out_copied"):
            b[e] = torch.cuda.Event()
        bufs.append(b)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def copy_in(b):
        with torch.cuda.stream(s_in):
            s_in.wait_event(b["done"])        # the step that last read these buffers
            for n in names:
                b[n].copy_(host_in[n], non_blocking=True)
            b["in_ready"].record(s_in)

    def run(n_steps):
        for b in bufs:                        # nothing outstanding on either set
            b["done"].record(comp)
            b["out_copied"].record(comp)
        copy_in(bufs[0])
        for i in range(n_steps):
            b = bufs[i % 2]
            if i + 1 < n_steps:
                copy_in(bufs[(i + 1) % 2])
            comp.wait_event(b["in_ready"])
            comp.wait_event(b["out_copied"])  # its outputs of two steps ago are home
            fa.fwd(b["q"], b["k"], b["v"], scale=c.scale, causal=True, out=b["out"], lse=b["lse"])
            b["fwd_done"].record(comp)
            if have_bwd:
                fa.bwd(b["q"], b["k"], b["v"], b["out"], b["lse"], b["do"], scale=c.scale, causal=True,
                       dq=b["dq"], dk=b["dk"], dv=b["dv"], workspace=b["ws"])
            b["done"].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(b["fwd_done"])
                b["h_out"].copy_(b["out"], non_blocking=True)
                if have_bwd:
                    s_out.wait_event(b["done"])
                    b["h_dq"].copy_(b["dq"], non_blocking=True)
                    b["h_dk"].copy_(b["dk"], non_blocking=True)
                    b["h_dv"].copy_(b["dv"], non_blocking=True)
                b["out_copied"].record(s_out)
        for b in bufs:                        # the timed region ends with every copy home
            comp.wait_event(b["out_copied"])

    run(2)                                    # warm-up
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    run(steps)
    end.record(comp)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(start.elapsed_time(end) / steps)
    h2d = sum(host_in[n].numel() * host_in[n].element_size() for n in names)
    d2h = bufs[0]["h_out"].numel() * 2 + ((bufs[0]["h_dq"].numel() + bufs[0]["h_dk"].numel() +
                                           bufs[0]["h_dv"].numel()) * 2 if have_bwd else 0)
    del bufs, host_in
    return {"unit": "TFLOP/s", "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipeline": "two buffer sets; H2D and D2H on their own streams, overlapping the compute"}


def prefill_inputs(dev):
    c = W.CONFIGS[3]
    inp = W.make_fwd_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, c.dtype, seed=1000 + c.cid, with_do=True)
    pairs = W.visible_pairs(c.S, c.S, c.causal, *c.window) * c.B
    return c, inp, pairs


def run_only(args, dist: Dist):
    """One kernel family on its headline workload, few launches: the command
    the ncu captures in profiles/ run (`--only fwd|bwd|varlen|decode`)."""
    import exact_attention_149_b200 as fa

    peaks = load_peaks()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    out = {"impl": "ours", "only": args.only, "steps": args.steps, "warmup": args.warmup}
    if args.only in ("fwd", "bwd"):
        c, inp, pairs = prefill_inputs(dev)
        q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
        o, lse = fa.fwd(q, k, v, scale=c.scale, causal=True)
        if args.only == "fwd":
            fn = lambda: fa.fwd(q, k, v, scale=c.scale, causal=True, out=o, lse=lse)  # noqa: E731
            flop = W.fwd_flops(pairs, c.D, c.Hq)
        else:
            ws = torch.empty(fa.fa_bwd_workspace_size(c.B, c.Hq, c.S, c.D), dtype=torch.uint8,
                             device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            fn = lambda: fa.bwd(q, k, v, o, lse, do, scale=c.scale, causal=True, dq=dq, dk=dk,  # noqa: E731
                                dv=dv, workspace=ws)
            flop = W.bwd_flops(pairs, c.D, c.Hq)
        ms = timed(fn, args.steps, args.warmup, dist)
        out.update(ms=ms, tflops=flop / (ms * 1e-3) / 1e12)
        out["frac_of_bf16_peak"] = out["tflops"] / peaks["bf16_tflops"]
    elif args.only == "fp8":
        c = W.CONFIGS[3]
        d = W.make_fp8_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, seed=1000 + c.cid)
        q8, k8, v8 = (d[n].to(dev) for n in ("q", "k", "v"))
        o8 = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
        l8 = torch.empty((c.B, c.Hq, c.S), dtype=torch.float32, device=dev)
        fn = lambda: fa.fwd_fp8(q8, k8, v8, d["q_descale"], d["k_descale"], d["v_descale"],  # noqa: E731
                                scale=c.scale, causal=True, out=o8, lse=l8)
        flop = W.fwd_flops(W.visible_pairs(c.S, c.S, True) * c.B, c.D, c.Hq)
        ms = timed(fn, args.steps, args.warmup, dist)
        out.update(ms=ms, tflops=flop / (ms * 1e-3) / 1e12)
        out["frac_of_fp8_peak"] = out["tflops"] / (2.0 * peaks["bf16_tflops"])
    elif args.only == "varlen":
        cv = W.CONFIGS[4]
        vin = W.make_varlen_inputs(None, cv.Hq, cv.Hkv, cv.D, cv.dtype, seed=1000 + cv.cid,
                                   total=cv.total, len_lo=cv.len_lo, len_hi=cv.len_hi)
        vq, vk, vv = (vin[n].to(dev) for n in ("q", "k", "v"))
        cu = vin["cu_seqlens"].to(dev)
        flop = W.fwd_flops(W.varlen_visible_pairs(vin["lengths"], cv.causal, *cv.window), cv.D, cv.Hq)
        fn = lambda: fa.fwd(vq, vk, vv, scale=cv.scale, causal=True, window=cv.window,  # noqa: E731
                            softcap=cv.softcap, cu_seqlens=cu, max_seqlen=max(vin["lengths"]))
        ms = timed(fn, args.steps, args.warmup, dist)
        out.update(ms=ms, tflops=flop / (ms * 1e-3) / 1e12)
    elif args.only == "decode":
        cd = W.CONFIGS[5]
        B = args.decode_batch or cd.B
        st = W.make_decode_structure(B, cd.Hq, cd.Hkv, cd.D, cd.len_lo, cd.len_hi,
                                     cd.page_size, cd.dtype, seed=1000 + cd.cid)
        shape = (st["num_pages"], st["page_size"], cd.Hkv, cd.D)
        kc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        vc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        W.fill_paged_pool(st, kc, vc)
        q = st["q"].to(dev)
        kn, vn = st["k_new"].to(dev), st["v_new"].to(dev)
        cs, bt = st["cache_seqlens"].to(dev), st["block_table"].to(dev)
        kv_bytes = W.decode_kv_bytes(st["cache_seqlens"], cd.Hkv, cd.D)
        if args.int8 or args.int4:
            quant = fa.kv_quantize_int4 if args.int4 else fa.kv_quantize_int8
            kc, ksc = quant(kc)
            vc, vsc = quant(vc)
            torch.cuda.empty_cache()
            kv_bytes = (W.decode_kv_bytes_int4 if args.int4 else W.decode_kv_bytes_int8)(
                st["cache_seqlens"], cd.Hkv, cd.D)
            fn = lambda: fa.fwd_kvcache(q, kc, vc, cs, bt, k_new=kn, v_new=vn, scale=cd.scale,  # noqa: E731
                                        causal=True, num_splits=args.splits, k_scale=ksc,
                                        v_scale=vsc)
        else:
            fn = lambda: fa.fwd_kvcache(q, kc, vc, cs, bt, k_new=kn, v_new=vn, scale=cd.scale,  # noqa: E731
                                        causal=True, num_splits=args.splits)
        ms = timed(fn, args.steps, args.warmup, dist)
        gbs = kv_bytes / (ms * 1e-3) / 1e9
        out.update(ms=ms, gbs=gbs, frac_of_hbm=gbs / peaks["hbm_gbs"], splits=args.splits, B=B,
                   cache="int4" if args.int4 else ("int8" if args.int8 else "16-bit"))
    return out


def run_ours(args, dist: Dist):
    import exact_attention_149_b200 as fa

    peaks = load_peaks()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    res = {}
    # -------------------- headline: causal prefill fwd + bwd --------------------
    c, inp, pairs = prefill_inputs(dev)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    fwd_flop = W.fwd_flops(pairs, c.D, c.Hq)
    bwd_flop = W.bwd_flops(pairs, c.D, c.Hq)
    have_bwd = True
    out = torch.empty_like(q)
    lse = torch.empty((c.B, c.Hq, c.S), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(c.B, c.Hq, c.S, c.D), dtype=torch.uint8, device=dev)

    def step_fwd():
        fa.fwd(q, k, v, scale=c.scale, causal=True, out=out, lse=lse)

    def step_bwd():
        fa.bwd(q, k, v, out, lse, do, scale=c.scale, causal=True, dq=dq, dk=dk, dv=dv,
               workspace=ws)

    step_fwd()
    torch.cuda.synchronize()
    try:
        step_bwd()
        torch.cuda.synchronize()
    except fa.FaError:
        have_bwd = False

    def step():
        step_fwd()
        if have_bwd:
            step_bwd()

    sampler = ClockSampler(dev.index) if dist.rank == 0 else None
    ms_step = timed(step, args.steps, args.warmup, dist, sampler, fa_mod=fa)
    kern = {}
    # matmul FLOPs each kernel executes (per visible pair and query head):
    # fwd S, PV = 4D; bwd_dkdv S, dP, dV, dK = 8D; bwd_dq S, dP, dQ = 6D.
    # The backward's algorithmic count is 10D (S, dP, dV, dK, dQ); the split
    # into two kernels recomputes S and dP once more (14D executed).
    executed = {"fwd": 4, "bwd_dkdv": 8, "bwd_dq": 6}
    algorithmic = {"fwd": 4, "bwd_dkdv": 8, "bwd_dq": 2}
    for name in ("fwd", "bwd_pre", "bwd_dkdv", "bwd_dq"):
        tot, n = fa.fa_kernel_timing_read(name)
        if n:
            kern[name] = {"ms_avg": tot / n, "launches": n}
            if name in executed:
                f_exec = executed[name] * c.D * pairs * c.Hq
                f_alg = algorithmic[name] * c.D * pairs * c.Hq
                kern[name]["tflops_executed"] = f_exec / (tot / n * 1e-3) / 1e12
                kern[name]["tflops_algorithmic"] = f_alg / (tot / n * 1e-3) / 1e12
    fa.fa_kernel_timing_reset()
    ms_fwd = timed(step_fwd, args.steps, 1, dist)
    ms_bwd = timed(step_bwd, args.steps, 1, dist) if have_bwd else None
    flop_step = fwd_flop + (bwd_flop if have_bwd else 0)
    value = replica_throughput(flop_step, ms_step, dist.world) / 1e12
    res["fwd"] = {"ms": ms_fwd, "tflops": fwd_flop / (ms_fwd * 1e-3) / 1e12,
                  "flop": fwd_flop}
    res["fwd"]["frac_of_bf16_peak"] = res["fwd"]["tflops"] / peaks["bf16_tflops"]
    if have_bwd:
        res["bwd"] = {"ms": ms_bwd, "tflops": bwd_flop / (ms_bwd * 1e-3) / 1e12, "flop": bwd_flop}
        res["bwd"]["frac_of_bf16_peak"] = res["bwd"]["tflops"] / peaks["bf16_tflops"]

    # -------------------- the same step with ALiBi slopes --------------------
    if have_bwd:
        slopes = W.alibi_slopes(c.Hq).to(dev)

        def step_alibi():
            fa.fwd(q, k, v, scale=c.scale, causal=True, out=out, lse=lse, alibi_slopes=slopes)
            fa.bwd(q, k, v, out, lse, do, scale=c.scale, causal=True, dq=dq, dk=dk, dv=dv,
                   workspace=ws, alibi_slopes=slopes)

        ms_al = timed(step_alibi, args.steps, args.warmup, dist, fa_mod=fa)
        res["alibi_fwd_bwd"] = {"ms": ms_al, "tflops": flop_step / (ms_al * 1e-3) / 1e12,
                                "slopes": "2^(-8(h+1)/Hq)", "kernels": {}}
        for name in ("fwd", "bwd_dkdv", "bwd_dq"):
            tot, n = fa.fa_kernel_timing_read(name)
            if n:
                res["alibi_fwd_bwd"]["kernels"][name] = {
                    "ms_avg": tot / n,
                    "vs_without_alibi": (tot / n) / kern[name]["ms_avg"] if name in kern else None}
        fa.fa_kernel_timing_reset()
        res["alibi_fwd_bwd"]["frac_of_bf16_peak"] = res["alibi_fwd_bwd"]["tflops"] / peaks["bf16_tflops"]

    # -------------------- end to end through the public API --------------------
    # A user's training loop: every step copies its inputs in from pinned host
    # memory and its outputs (o, dq, dk, dv) back, all inside the timed
    # region. The copies run on their own streams with two sets of device
    # buffers, so step i+1's inputs and step i's outputs cross PCIe (both
    # directions at once) while step i computes; the compute stream waits
    # only for its own step's inputs and for the copy-out of the buffers it
    # reuses.
    e2e = e2e_pipeline(fa, c, inp, have_bwd, max(4, args.steps // 2), dist)
    h2d, d2h = e2e["h2d_bytes_per_step"], e2e["d2h_bytes_per_step"]
    e2e["value"] = dist.world * flop_step / (e2e["ms_per_step"] * 1e-3) / 1e12

    # -------------------- varlen forward (GQA, window, softcap) --------------------
    cv = W.CONFIGS[4]
    vin = W.make_varlen_inputs(None, cv.Hq, cv.Hkv, cv.D, cv.dtype, seed=1000 + cv.cid,
                               total=cv.total, len_lo=cv.len_lo, len_hi=cv.len_hi)
    vq, vk, vv = (vin[n].to(dev) for n in ("q", "k", "v"))
    cu = vin["cu_seqlens"].to(dev)
    vout = torch.empty_like(vq)
    vlse = torch.empty((cv.Hq, cv.total), dtype=torch.float32, device=dev)
    vpairs = W.varlen_visible_pairs(vin["lengths"], cv.causal, *cv.window)
    vflop = W.fwd_flops(vpairs, cv.D, cv.Hq)

    def step_varlen():
        fa.fwd(vq, vk, vv, scale=cv.scale, causal=True, window=cv.window, softcap=cv.softcap,
               cu_seqlens=cu, max_seqlen=max(vin["lengths"]), out=vout, lse=vlse)

    ms_var = timed(step_varlen, args.steps, args.warmup, dist)
    res["varlen_fwd"] = {"ms": ms_var, "tflops": vflop / (ms_var * 1e-3) / 1e12, "flop": vflop,
                         "lengths": vin["lengths"]}
    res["varlen_fwd"]["frac_of_bf16_peak"] = res["varlen_fwd"]["tflops"] / peaks["bf16_tflops"]
    res["varlen_fwd"]["traffic"] = kernel_traffic("fwd_varlen")
    del vq, vk, vv, vout, vlse

    # -------------------- FP8 forward on the headline shape --------------------
    # E4M3 q, k, v with per-tensor descales, bf16 output; FLOPs counted as for
    # the 16-bit forward. The peak is the measured bf16 burst figure times the
    # nominal fp8 : bf16 dense ratio of 2 (no fp8 GEMM is measured).
    try:
        d8 = W.make_fp8_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, seed=1000 + c.cid)
        q8, k8, v8 = (d8[n].to(dev) for n in ("q", "k", "v"))
        o8 = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
        l8 = torch.empty((c.B, c.Hq, c.S), dtype=torch.float32, device=dev)

        def step_fp8():
            fa.fwd_fp8(q8, k8, v8, d8["q_descale"], d8["k_descale"], d8["v_descale"],
                       scale=c.scale, causal=True, out=o8, lse=l8)

        ms_8 = timed(step_fp8, args.steps, args.warmup, dist, fa_mod=fa)
        kt, kn = fa.fa_kernel_timing_read("fwd_fp8")
        fa.fa_kernel_timing_reset()
        fp8_peak = 2.0 * peaks["bf16_tflops"]
        res["fp8_fwd"] = {"ms": ms_8, "tflops": fwd_flop / (ms_8 * 1e-3) / 1e12, "flop": fwd_flop,
                          "workload": "fwd causal B2 Hq32 Hkv32 S8192 D128, E4M3 q/k/v, bf16 out",
                          "peak_tflops": fp8_peak,
                          "peak_source": peaks["source"] + " bf16 burst x 2 (nominal fp8:bf16 ratio)"}
        res["fp8_fwd"]["frac_of_fp8_peak"] = res["fp8_fwd"]["tflops"] / fp8_peak
        if kn:
            res["fp8_fwd"]["kernel_ms_avg"] = kt / kn
        res["fp8_fwd"]["traffic"] = kernel_traffic("fwd_fp8")
        del q8, k8, v8, o8, l8
    except Exception as e:  # recorded in the line; the headline measurement stands
        res["fp8_fwd"] = {"error": f"{type(e).__name__}: {e}"}

    # -------------------- paged split-KV decode --------------------
    cd = W.CONFIGS[5]
    st = W.make_decode_structure(cd.B, cd.Hq, cd.Hkv, cd.D, cd.len_lo, cd.len_hi, cd.page_size,
                                 cd.dtype, seed=1000 + cd.cid)
    shape = (st["num_pages"], st["page_size"], cd.Hkv, cd.D)
    kc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    W.fill_paged_pool(st, kc, vc)
    dq_ = st["q"].to(dev)
    kn, vn = st["k_new"].to(dev), st["v_new"].to(dev)
    cs, bt = st["cache_seqlens"].to(dev), st["block_table"].to(dev)
    kv_bytes = W.decode_kv_bytes(st["cache_seqlens"], cd.Hkv, cd.D)
    dec = {"kv_bytes": kv_bytes, "splits": {}}
    dout = torch.empty_like(dq_)
    dlse = torch.empty((cd.B, cd.Hq, 1), dtype=torch.float32, device=dev)
    for splits in cd.splits:
        wsd = fa.fa_kvcache_workspace_size(cd.B, 1, cd.Hq, cd.D, splits)
        wsb = torch.empty(max(wsd, 1), dtype=torch.uint8, device=dev)

        def step_dec(splits=splits, wsb=wsb):
            fa.fwd_kvcache(dq_, kc, vc, cs, bt, k_new=kn, v_new=vn, scale=cd.scale, causal=True,
                           num_splits=splits, out=dout, lse=dlse, workspace=wsb)

        ms_d = timed(step_dec, max(args.steps, 20), args.warmup, dist, fa_mod=fa)
        ksplit, nsplit = fa.fa_kernel_timing_read("decode_split")
        fa.fa_kernel_timing_reset()
        gbs = kv_bytes / (ms_d * 1e-3) / 1e9
        entry = {"ms": ms_d, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}
        if nsplit:
            ks = ksplit / nsplit
            entry["decode_split_kernel"] = {
                "ms_avg": ks, "gbs": kv_bytes / (ks * 1e-3) / 1e9,
                "frac_of_hbm": kv_bytes / (ks * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        dec["splits"][str(splits)] = entry
    best = max(dec["splits"].values(), key=lambda d: d["gbs"])
    dec["best_gbs"] = best["gbs"]
    dec["best_frac_of_hbm"] = best["frac_of_hbm"]
    trd = kernel_traffic("decode_split")
    dec["roofline"] = {"kernel": "decode_split", "bound": "hbm",
                       "achieved": best.get("decode_split_kernel", best)["gbs"],
                       "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": best.get("decode_split_kernel", best)["gbs"] / peaks["hbm_gbs"],
                       "traffic": trd["bytes_per_launch"] if trd else None,
                       "peak_source": peaks["source"] + " HBM copy"}
    res["decode"] = dec

    # -------------------- the same decode step on an int8 cache --------------------
    # the 16-bit pool quantised on the device (fa_kv_quantize_int8); the step
    # then reads D + 4 bytes per cached row instead of 2 D
    kq, ksq = fa.kv_quantize_int8(kc)
    vq, vsq = fa.kv_quantize_int8(vc)
    k4, ks4 = fa.kv_quantize_int4(kc)
    v4, vs4 = fa.kv_quantize_int4(vc)
    del kc, vc
    torch.cuda.empty_cache()
    kv8 = W.decode_kv_bytes_int8(st["cache_seqlens"], cd.Hkv, cd.D)
    dec8 = {"kv_bytes": kv8, "format": "int8 codes + one float32 scale per (token, kv head) row",
            "splits": {}}
    for splits in cd.splits:
        wsd = fa.fa_kvcache_workspace_size(cd.B, 1, cd.Hq, cd.D, splits)
        wsb = torch.empty(max(wsd, 1), dtype=torch.uint8, device=dev)

        def step_dec8(splits=splits, wsb=wsb):
            fa.fwd_kvcache(dq_, kq, vq, cs, bt, k_new=kn, v_new=vn, scale=cd.scale, causal=True,
                           num_splits=splits, out=dout, lse=dlse, workspace=wsb, k_scale=ksq,
                           v_scale=vsq)

        ms_d = timed(step_dec8, max(args.steps, 20), args.warmup, dist, fa_mod=fa)
        ksplit, nsplit = fa.fa_kernel_timing_read("decode_split")
        fa.fa_kernel_timing_reset()
        gbs = kv8 / (ms_d * 1e-3) / 1e9
        entry = {"ms": ms_d, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                 "speedup_vs_16bit": dec["splits"][str(splits)]["ms"] / ms_d}
        if nsplit:
            ks = ksplit / nsplit
            entry["decode_split_kernel"] = {
                "ms_avg": ks, "gbs": kv8 / (ks * 1e-3) / 1e9,
                "frac_of_hbm": kv8 / (ks * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        dec8["splits"][str(splits)] = entry
    best8 = max(dec8["splits"].values(), key=lambda d: d["gbs"])
    dec8["best_gbs"] = best8["gbs"]
    dec8["best_frac_of_hbm"] = best8["frac_of_hbm"]
    trd8 = kernel_traffic("decode_split_int8")
    k8 = best8.get("decode_split_kernel", best8)
    dec8["roofline"] = {"kernel": "decode_split (int8 cache)", "bound": "hbm", "achieved": k8["gbs"],
                        "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": k8["gbs"] / peaks["hbm_gbs"],
                        "traffic": trd8["bytes_per_launch"] if trd8 else None,
                        "peak_source": peaks["source"] + " HBM copy"}
    res["decode_int8"] = dec8
    del kq, vq, ksq, vsq

    # -------------------- and on an int4 cache (two codes per byte) --------------------
    kv4 = W.decode_kv_bytes_int4(st["cache_seqlens"], cd.Hkv, cd.D)
    dec4 = {"kv_bytes": kv4, "format": "int4 codes two per byte + one float32 scale per (token, kv head) row",
            "splits": {}}
    try:
        for splits in cd.splits:
            wsd = fa.fa_kvcache_workspace_size(cd.B, 1, cd.Hq, cd.D, splits)
            wsb = torch.empty(max(wsd, 1), dtype=torch.uint8, device=dev)

            def step_dec4(splits=splits, wsb=wsb):
                fa.fwd_kvcache(dq_, k4, v4, cs, bt, k_new=kn, v_new=vn, scale=cd.scale, causal=True,
                               num_splits=splits, out=dout, lse=dlse, workspace=wsb, k_scale=ks4,
                               v_scale=vs4)

            ms_d = timed(step_dec4, max(args.steps, 20), args.warmup, dist, fa_mod=fa)
            ksplit, nsplit = fa.fa_kernel_timing_read("decode_split")
            fa.fa_kernel_timing_reset()
            gbs = kv4 / (ms_d * 1e-3) / 1e9
            entry = {"ms": ms_d, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                     "speedup_vs_16bit": dec["splits"][str(splits)]["ms"] / ms_d}
            if nsplit:
                ks = ksplit / nsplit
                entry["decode_split_kernel"] = {
                    "ms_avg": ks, "gbs": kv4 / (ks * 1e-3) / 1e9,
                    "frac_of_hbm": kv4 / (ks * 1e-3) / 1e9 / peaks["hbm_gbs"]}
            dec4["splits"][str(splits)] = entry
        best4 = max(dec4["splits"].values(), key=lambda d: d["gbs"])
        dec4["best_gbs"] = best4["gbs"]
        dec4["best_frac_of_hbm"] = best4["frac_of_hbm"]
        trd4 = kernel_traffic("decode_split_int4")
        k4 = best4.get("decode_split_kernel", best4)
        dec4["roofline"] = {"kernel": "decode_split (int4 cache)", "bound": "hbm",
                            "achieved": k4["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": k4["gbs"] / peaks["hbm_gbs"],
                            "traffic": trd4["bytes_per_launch"] if trd4 else None,
                            "peak_source": peaks["source"] + " HBM copy"}
    except Exception as e:  # recorded in the line; the headline measurement stands
        dec4["error"] = f"{type(e).__name__}: {e}"
    res["decode_int4"] = dec4
    del k4, v4, ks4, vs4
    torch.cuda.empty_cache()

    # -------------------- roofline of the dominant kernel --------------------
    # per-kernel averages come from CUDA events the library recorded around
    # each launch on the launching stream during the headline loop
    dominant = max(kern, key=lambda k: kern[k]["ms_avg"])
    if dominant in algorithmic:
        f_alg = algorithmic[dominant] * c.D * pairs * c.Hq
        achieved = f_alg / (kern[dominant]["ms_avg"] * 1e-3) / 1e12
        roofline = {"kernel": dominant, "bound": "tensor", "achieved": achieved,
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops"],
                    "peak_source": peaks["source"] + " burst bf16 (cuBLAS)",
                    "algorithmic": f"{f_alg:.4e} FLOP per launch ({algorithmic[dominant]}*D per "
                                   f"visible pair and query head)"}
    else:
        roofline = {"kernel": dominant, "bound": "hbm", "achieved": None, "peak": None}
    tr = kernel_traffic(dominant)
    roofline["traffic"] = tr["bytes_per_launch"] if tr else None
    roofline["traffic_unit"] = "bytes per launch (dram read + write, ncu)"
    res["kernels"] = kern

    launches_per_step = 1 + (3 if have_bwd else 0)  # fwd; bwd_pre, bwd_dkdv, bwd_dq
    line = {
        "metric": "attention fwd+bwd TFLOP/s, causal B2 H32 S8192 D128 bf16 "
                  "(decode KV GB/s and varlen fwd reported alongside)",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic N(0,1) bf16, seeded (no dataset exists for this benchmark)",
        "config": {"workload": "fwd+bwd causal B2 Hq32 Hkv32 S8192 D128 bf16" if have_bwd
                   else "fwd causal B2 Hq32 Hkv32 S8192 D128 bf16",
                   "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "S": c.S, "D": c.D, "causal": True,
                   "l2": "inputs larger than L2 (q,k,v 402 MB), no flush",
                   "parallelism": f"replicas x{dist.world}"},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "roofline": roofline,
        "peaks": peaks,
        "clocks": sampler.summary() if sampler is not None else None,
        **res,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    return line


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the headline workload
# ---------------------------------------------------------------------------
def _oracle_sample(c, inp, seconds_budget):
    """Time the oracle's forward and backward on whole heads of the causal
    S8192 workload until about `seconds_budget` seconds have passed."""
    import numpy as np

    from oracle import head_bwd, head_fwd

    done_flop = 0
    heads = 0
    t0 = time.perf_counter()
    pairs_head = W.visible_pairs(c.S, c.S, True)
    for b in range(c.B):
        for h in range(c.Hq):
            qh = inp["q"][b, :, h]
            kh = inp["k"][b, :, h]
            vh = inp["v"][b, :, h]
            doh = inp["do"][b, :, h]
            head_fwd(qh, kh, vh, c.scale, True)
            head_bwd(qh, kh, vh, doh, c.scale, True)
            heads += 1
            done_flop += W.fwd_flops(pairs_head, c.D, 1) + W.bwd_flops(pairs_head, c.D, 1)
            if time.perf_counter() - t0 > seconds_budget:
                break
        else:
            continue
        break
    dt = time.perf_counter() - t0
    del np
    return done_flop, dt, heads


def cpu_baseline(seconds):
    c = W.CONFIGS[3]
    inp = W.make_fwd_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, c.dtype, seed=1000 + c.cid, with_do=True)
    flop, dt, heads = _oracle_sample(c, inp, seconds)
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{heads} whole head(s) (b, h) of the causal B2 H32 S8192 D128 workload, "
                      f"fwd + bwd in fp64 numpy, {dt:.1f} s"}


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return None
    c = W.CONFIGS[3]
    inp = W.make_fwd_inputs(c.B, c.S, c.Hq, c.Hkv, c.D, c.dtype, seed=1000 + c.cid, with_do=True)
    per_step = []
    flop_total = 0
    heads_total = 0
    budget = max(2.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup and 1):
        _oracle_sample(c, inp, 0.0)  # one head: warm BLAS
    for _ in range(args.steps):
        flop, dt, heads = _oracle_sample(c, inp, budget)
        per_step.append(dt)
        flop_total += flop
        heads_total += heads
    t = sum(per_step)
    value = flop_total / t / 1e12
    line = {
        "impl": "reference",
        "metric": "attention fwd+bwd TFLOP/s, causal B2 H32 S8192 D128 bf16 "
                  "(decode KV GB/s and varlen fwd reported alongside)",
        "value": value, "unit": "TFLOP/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic N(0,1) bf16 inputs, seeded; each step a bounded sample of whole heads",
        "config": {"workload": "fwd+bwd causal B2 Hq32 Hkv32 S8192 D128 bf16", "B": c.B,
                   "Hq": c.Hq, "Hkv": c.Hkv, "S": c.S, "D": c.D, "causal": True},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "kind": "oracle",
                         "cores": len(os.sched_getaffinity(0)),
                         "sample": f"{heads_total} head(s) over {args.steps} step(s), fp64 numpy"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default=None, choices=["fwd", "bwd", "varlen", "decode", "fp8"],
                    help="time one kernel family only (profiling runs)")
    ap.add_argument("--splits", type=int, default=16, help="num_splits for --only decode")
    ap.add_argument("--int8", action="store_true", help="--only decode on an int8 cache")
    ap.add_argument("--int4", action="store_true", help="--only decode on an int4 cache")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="batch for --only decode (default: the B64 workload); smaller for ncu")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours" and args.only is None:
        args.warmup = 3
    dist = Dist()
    try:
        if args.impl == "reference":
            line = run_reference(args, dist)
        elif args.only is not None:
            line = run_only(args, dist)
        else:
            line = run_ours(args, dist)
        if dist.rank == 0 and line is not None:
            print(json.dumps(line))
            sys.stdout.flush()
    finally:
        dist.close()


if __name__ == "__main__":
    main()
