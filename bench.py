#!/usr/bin/env python
"""Benchmark of the exact-attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of the prefill
workload (B=4, H=16, N=2048, d=128, bf16, iid N(0,1) inputs):
  1. fa_fwd, no mask             (O, LSE)
  2. fa_fwd, causal mask         (O, LSE)
  3. fa_bwd, causal mask         (dQ, dK, dV from step 2's O and LSE and a dO)
  4. fa_decode_splitkv           (one new query token per sequence and head
                                  against the step's K/V as the cache,
                                  every cache length 2048)
The metric is attention TFLOP/s: FLOPs are 4 B H N^2 d per forward (halved
under the causal mask), 2.5x that for the backward, 4 H L d per decoded
token; `value` is the whole-job throughput over all ranks. The JSON line also
carries a per-kernel breakdown of the step with each kernel's fraction of its
roofline (tensor peak for the forward/backward, HBM bandwidth for decode; the
no-mask and causal forward launches apart), and, under `configs`, every
benchmark workload timed on its own shape after the step: prefill forward
(B=4 H=16 N=2048 d=128) without and with the causal mask, the long causal
forward (B=1 H=32 N=16384), the backward (B=2 H=16 N=4096, causal) and the
split-KV decode (B=8 H=32, cache lengths 16k-32k).

Inputs are resident in HBM when the timed region starts; L2 (126 MB) is
flushed between timed steps by writing a 256 MB buffer outside the timed
events. `e2e` repeats the measurement through the same C ABI calls with the
step's inputs copied from pinned host memory and every output copied back,
inside the timed region.

Multi-GPU (torchrun): every rank runs its own copy of the workload (weak
scaling, no collective on the data path); the timed region is bracketed by a
barrier and a device synchronise on both sides and the per-rank time is
reduced with MAX.

--impl reference times the fp64 CPU oracle (the one reference
implementation there is to time) on a bounded sample of the same workload
per step, on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("attention fwd/bwd TFLOP/s (bf16,d=128) as % of B200 tensor peak; "
          "decode HBM GB/s")
WORKLOAD_NAME = "prefill"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # single-kernel mode, for profiler captures (prints timings, no bench line)
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the FP8 forward and paged decode measured after the step")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload measurements (prefill, long causal, backward, "
                         "decode) made after the step")
    ap.add_argument("--kernel", choices=["fwd", "fwd_pair", "fwd_ex", "fwd_fp8", "fp8_prep", "bwd",
                                         "bwd_ex", "decode", "decode_paged"],
                    default=None)
    ap.add_argument("--hkv", type=int, default=8, help="KV heads of --kernel decode_paged")
    ap.add_argument("--page", type=int, default=64, help="page rows of --kernel decode_paged")
    ap.add_argument("--causal", type=int, default=0)
    ap.add_argument("--B", type=int, default=16)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--N", type=int, default=2048)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--p-drop", type=float, default=0.1, help="dropout of --kernel fwd_ex/bwd_ex")
    ap.add_argument("--bias", type=int, default=1, help="--kernel fwd_ex/bwd_ex: 1 = a bf16 bias "
                    "[1, H, N, N] (broadcast over the batch), 0 = none")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, local):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(world, x: float, op: str) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def dist_max(world, x: float) -> float:
    """Slowest rank's time: the job is done when the last rank is."""
    return _reduce(world, x, "max")


def dist_sum(world, x: float) -> float:
    """Work summed over ranks (weak scaling: every rank runs its own batch)."""
    return _reduce(world, x, "sum")


# ---------------------------------------------------------------------------
# clocks sampled during the timed region (NVML, every 1 ms)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2,
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sync_boost": 0x10,
        "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no clocks rather than fail
            self._nvml = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0}
        names = [n for n, bit in self.REASONS.items()
                 if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# peaks and recorded DRAM traffic
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "source": "measured (MEASURED_PEAKS.json, burst)"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def kernel_source_hash(name: str) -> str:
    files = {"fwd_full": "fwd_sm100.cu", "fwd_causal": "fwd_sm100.cu",
             "bwd_dkdv": "bwd_sm100.cu", "bwd_dq": "bwd_sm100.cu",
             "decode_split": "decode_sm100.cu"}
    path = os.path.join(ROOT, "exact_attention_130_b200", "csrc", files.get(name, ""))
    try:
        return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except Exception:
        return ""


# the launch of each kernel that one bench step makes, as named in
# profiles/traffic.json when a capture of exactly that launch is recorded
BENCH_LAUNCH = {
    "fwd_full": "bench step: fwd no mask B=4 H=16 N=2048 d=128",
    "fwd_causal": "bench step: fwd causal B=4 H=16 N=2048 d=128",
    "bwd_dkdv": "bench step: bwd causal B=4 H=16 N=2048 d=128",
    "bwd_dq": "bench step: bwd causal B=4 H=16 N=2048 d=128",
    "decode_split": "bench step: decode B=4 H=16 cache 2048 d=128",
}


def recorded_traffic(name: str):
    """DRAM bytes per launch from the committed ncu capture of the bench's
    own launch of this kernel, if the kernel source is unchanged since it was
    taken; else None."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
        k = rec["kernels"][name]
        if k["source_sha256_16"] != kernel_source_hash(name):
            return None
        if k.get("workload") != BENCH_LAUNCH.get(name):
            return None
        return float(k["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    import numpy as np
    import torch

    import exact_attention_130_b200 as fa
    import inputgen
    from exact_attention_130_b200 import counters as C

    dist_init(world, local)
    w = inputgen.WORKLOADS[WORKLOAD_NAME]
    B, H, N, d = w.B, w.H, w.N, w.d
    x = inputgen.make_attention_inputs(w, with_grad=True)
    host = {n: torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).pin_memory()
            for n in ("q", "k", "v", "do")}
    dev = {n: t.cuda() for n, t in host.items()}
    lens = torch.full((B,), N, dtype=torch.int32, device="cuda")
    qdec = dev["q"][:, :, -1].contiguous()
    out = {
        "o_full": torch.empty_like(dev["q"]), "lse_full": torch.empty((B, H, N), dtype=torch.float32, device="cuda"),
        "o_causal": torch.empty_like(dev["q"]), "lse_causal": torch.empty((B, H, N), dtype=torch.float32, device="cuda"),
        "dq": torch.empty_like(dev["q"]), "dk": torch.empty_like(dev["q"]), "dv": torch.empty_like(dev["q"]),
        "o_dec": torch.empty_like(qdec), "lse_dec": torch.empty((B, H), dtype=torch.float32, device="cuda"),
    }
    ws_bwd = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    ws_dec = torch.empty(fa.fa_decode_workspace_size(B, H, N, d, 0), dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def step(src, dst=None):
        dst = out if dst is None else dst
        fa.fa_fwd(src["q"], src["k"], src["v"], causal=False, o=dst["o_full"], lse=dst["lse_full"])
        fa.fa_fwd(src["q"], src["k"], src["v"], causal=True, o=dst["o_causal"], lse=dst["lse_causal"])
        fa.fa_bwd(src["q"], src["k"], src["v"], dst["o_causal"], dst["lse_causal"], src["do"],
                  causal=True, dq=dst["dq"], dk=dst["dk"], dv=dst["dv"], workspace=ws_bwd)
        fa.fa_decode_splitkv(src["qdec"], src["k"], src["v"], lens, o=dst["o_dec"],
                             lse=dst["lse_dec"], workspace=ws_dec)

    src_dev = dict(dev, qdec=qdec)
    launches_per_step = 1 + 1 + 3 + 2  # fwd, fwd, bwd (pre, dK/dV, dQ), decode (split, merge)
    # FLOPs by the measurement's convention (the headline): forward 4 B H N^2 d
    # (halved under the causal mask), backward 2.5x the causal forward
    step_flops = (C.fwd_flops(B, H, N, d, False) + C.fwd_flops(B, H, N, d, True)
                  + C.bwd_flops(B, H, N, d, True) + C.decode_flops(H, [N] * B, d))
    # tensor-core work each kernel actually performs per step (for the per-kernel
    # rates): the dK/dV kernel runs S^T, dP^T, dV, dK (2x the causal forward),
    # the dQ kernel S, dP, dQ (1.5x)
    fc = C.fwd_flops(B, H, N, d, True)
    flops = {  # per launch (each runs once per step)
        "fwd_full": C.fwd_flops(B, H, N, d, False),
        "fwd_causal": fc,
        "bwd_dkdv": 2.0 * fc,
        "bwd_dq": 1.5 * fc,
    }
    dec_bytes = C.decode_bytes(H, [N] * B, d)

    def timed(fn, k):
        """Run k steps; return summed device ms of the steps (L2 flushed in between)."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
        for i in range(k):
            flush.zero_()
            starts[i].record()
            fn()
            ends[i].record()
        torch.cuda.synchronize()
        return sum(s.elapsed_time(e) for s, e in zip(starts, ends))

    # warm-up
    for _ in range(args.warmup):
        step(src_dev)
    torch.cuda.synchronize()
    st, word = fa.fa_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} ({word:#x}) after warm-up")

    # 1. headline: device-resident inputs
    sampler = ClockSampler(local)
    dist_barrier(world)
    torch.cuda.synchronize()
    with sampler:
        ms = timed(lambda: step(src_dev), args.steps)
    torch.cuda.synchronize()
    dist_barrier(world)
    ms_max = dist_max(world, ms)
    total_flops = dist_sum(world, step_flops * args.steps)
    value = total_flops / (ms_max * 1e-3) / 1e12

    # 2. per-kernel breakdown: the same steps again, each call bracketed by
    # the library's own CUDA events around every launch (on the launching
    # stream); the two forward launches are kept apart (no mask, causal)
    peaks = load_peaks()
    calls = [
        ("fwd_full", lambda: fa.fa_fwd(src_dev["q"], src_dev["k"], src_dev["v"], causal=False,
                                       o=out["o_full"], lse=out["lse_full"])),
        ("fwd_causal", lambda: fa.fa_fwd(src_dev["q"], src_dev["k"], src_dev["v"], causal=True,
                                         o=out["o_causal"], lse=out["lse_causal"])),
        ("bwd", lambda: fa.fa_bwd(src_dev["q"], src_dev["k"], src_dev["v"], out["o_causal"],
                                  out["lse_causal"], src_dev["do"], causal=True, dq=out["dq"],
                                  dk=out["dk"], dv=out["dv"], workspace=ws_bwd)),
        ("decode", lambda: fa.fa_decode_splitkv(src_dev["qdec"], src_dev["k"], src_dev["v"], lens,
                                                o=out["o_dec"], lse=out["lse_dec"],
                                                workspace=ws_dec)),
    ]
    prof = {}
    for _ in range(args.steps):
        flush.zero_()
        for label, fn in calls:
            fa.fa_profile_begin()
            fn()
            for kname, (n, tot) in fa.fa_profile_end().items():
                key = label if kname == "fwd" else kname
                a = prof.setdefault(key, [0, 0.0])
                a[0] += n
                a[1] += tot
    kernels = {}
    for name, (n, tot) in prof.items():
        avg = tot / n
        entry = {"launches": n, "avg_ms": round(avg, 5)}
        if name in flops:
            tf = flops[name] * args.steps / (tot * 1e-3) / 1e12
            entry.update({"tflops": round(tf, 1),
                          "frac_of_tensor_peak": round(tf / peaks["bf16_tflops"], 4)})
        elif name == "decode_split":
            gbs = dec_bytes * args.steps / (tot * 1e-3) / 1e9
            entry.update({"gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)})
        kernels[name] = entry
    dominant = max(prof, key=lambda k: prof[k][1])
    dn, dtot = prof[dominant]
    if dominant in flops:
        achieved = flops[dominant] * args.steps / (dtot * 1e-3) / 1e12
        roofline = {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": round(achieved / peaks["bf16_tflops"], 4),
                    "traffic": recorded_traffic(dominant),
                    "algorithmic_per_launch": flops[dominant],
                    "peak_source": peaks["source"]}
    else:
        achieved = dec_bytes * args.steps / (dtot * 1e-3) / 1e9
        roofline = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": recorded_traffic(dominant),
                    "algorithmic_per_launch": dec_bytes, "peak_source": peaks["source"]}

    # 3. end to end through the same calls with host buffers: every step copies
    # its inputs in from pinned host memory and all its outputs back out. The
    # steps are pipelined as a host program would run them: step i+1's
    # host-to-device copies, step i's kernels and step i-1's device-to-host
    # copies run on three streams (device inputs, outputs and host outputs
    # double-buffered, ordered by events), so the two copy directions of the
    # link overlap each other and the kernels. One device-event region from
    # the first input copy to the last output copy; no L2 flush is needed, as
    # every step's 134 MB of input copies pass through L2.
    e2e = None
    if not args.no_e2e:
        host_qdec = host["q"][:, :, -1].contiguous().pin_memory()
        bufs = [dict({n: torch.empty_like(t) for n, t in dev.items()}, qdec=torch.empty_like(qdec))
                for _ in range(2)]
        outs = [{k: torch.empty_like(v) for k, v in out.items()} for _ in range(2)]
        h_out = [{k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in out.items()}
                 for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host.values()) + host_qdec.numel() * 2
        d2h = sum(t.numel() * t.element_size() for t in out.values())
        s_cmp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_run(k):
            ev = lambda: torch.cuda.Event(enable_timing=True)
            start, end = ev(), ev()
            start.record(s_cmp)
            s_in.wait_event(start)
            s_out.wait_event(start)
            done_cmp, done_out = [None] * k, [None] * k
            for i in range(k):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(done_cmp[i - 2])  # inputs of step i-2 consumed
                    for n in ("q", "k", "v", "do"):
                        bufs[b][n].copy_(host[n], non_blocking=True)
                    bufs[b]["qdec"].copy_(host_qdec, non_blocking=True)
                    ready = torch.cuda.Event()
                    ready.record(s_in)
                s_cmp.wait_event(ready)
                if i >= 2:
                    s_cmp.wait_event(done_out[i - 2])  # outputs of step i-2 read back
                step(bufs[b], outs[b])
                done_cmp[i] = torch.cuda.Event()
                done_cmp[i].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(done_cmp[i])
                    for kk, t in outs[b].items():
                        h_out[b][kk].copy_(t, non_blocking=True)
                    done_out[i] = torch.cuda.Event()
                    done_out[i].record(s_out)
            s_cmp.wait_event(done_out[k - 1])
            end.record(s_cmp)
            torch.cuda.synchronize()
            return start.elapsed_time(end)

        e2e_run(2)
        dist_barrier(world)
        e_ms = e2e_run(args.steps)
        dist_barrier(world)
        e_ms = dist_max(world, e_ms)
        e2e = {"value": round(total_flops / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_ms / args.steps, 4),
               "pipelining": "host-to-device copies of step i+1, kernels of step i and device-to-host "
                             "copies of step i-1 on three streams, double-buffered"}

    configs = None if args.no_configs else measure_configs(fa, torch, dev, flush, peaks)
    next_rows = None if args.no_next_rows else measure_next_rows(fa, torch, dev, flush, peaks)

    st, word = fa.fa_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} ({word:#x}) after timing")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(x, w)

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (iid N(0,1), seeded, bf16 round-to-nearest-even)",
        "config": {
            "workload": "prefill B=4 H=16 N=2048 d=128; step = fwd (no mask) + fwd (causal) "
                        "+ bwd (causal) + split-KV decode of one token per sequence over the "
                        "step's K/V (cache length 2048)",
            "B": B, "H": H, "N": N, "d": d, "step_gflop": round(step_flops / 1e9, 3),
            "l2": "flushed between timed steps (256 MB write outside the timed events)",
            "parallelism": f"replicas x{world} (independent heads, no collective)",
        },
        "roofline": roofline,
        "kernels": kernels,
        "configs": configs,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": sampler.summary(),
        "e2e": e2e,
        "cpu_baseline": cpu,
        "next_rows": next_rows,
        "impl": "ours",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (HGX 7.7 TB/s, DGX 8 TB/s)


def measure_configs(fa, torch, dev, flush, peaks, iters=10):
    """Every benchmark workload on its own, after the step (not part of
    `value`): median of `iters` launches with L2 flushed before each, CUDA
    events on the launching stream. Rates follow the step's conventions:
    4 B H N^2 d forward FLOPs (halved under the causal mask), backward 2.5x
    the forward (and, separately, the split backward's own GEMM count,
    3.5x the causal forward), decode bytes = every visible K and V row once
    plus q, O and LSE."""
    import numpy as np

    from exact_attention_130_b200 import counters as C

    def med_ms(fn):
        ts = []
        for _ in range(iters):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    tpk = peaks["bf16_tflops"]
    res = {}

    def fwd_entry(name, q, k, v, causal, workload):
        B, H, N, d = q.shape
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        ms = med_ms(lambda: fa.fa_fwd(q, k, v, causal=causal, o=o, lse=lse))
        tf = C.fwd_flops(B, H, N, d, causal) / (ms * 1e-3) / 1e12
        res[name] = {"workload": workload, "ms": round(ms, 4), "tflops": round(tf, 1),
                     "frac": round(tf / tpk, 4), "peak": tpk, "unit": "TFLOP/s"}
        return o, lse

    # prefill (the step's own inputs), no mask and causal apart
    wl = "prefill B=4 H=16 N=2048 d=128"
    fwd_entry("prefill_fwd_full", dev["q"], dev["k"], dev["v"], False, wl + ", no mask")
    fwd_entry("prefill_fwd_causal", dev["q"], dev["k"], dev["v"], True, wl + ", causal")

    g = torch.Generator(device="cuda").manual_seed(20262)

    def rnd(*shape):
        return torch.randn(shape, device="cuda", dtype=torch.bfloat16, generator=g)

    # long-context causal forward
    q, k, v = rnd(1, 32, 16384, 128), rnd(1, 32, 16384, 128), rnd(1, 32, 16384, 128)
    fwd_entry("long_fwd_causal", q, k, v, True, "long causal B=1 H=32 N=16384 d=128")
    del q, k, v

    # backward with recomputation, O and LSE from the forward
    q, k, v, do = (rnd(2, 16, 4096, 128) for _ in range(4))
    o, lse = fa.fa_fwd(q, k, v, causal=True)
    ws = torch.empty(fa.fa_bwd_workspace_size(2, 16, 4096, 128), dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ms = med_ms(lambda: fa.fa_bwd(q, k, v, o, lse, do, causal=True, dq=dq, dk=dk, dv=dv,
                                  workspace=ws))
    fc = C.fwd_flops(2, 16, 4096, 128, True)
    tf = C.bwd_flops(2, 16, 4096, 128, True) / (ms * 1e-3) / 1e12
    tf_own = 3.5 * fc / (ms * 1e-3) / 1e12
    res["backward_causal"] = {
        "workload": "backward B=2 H=16 N=4096 d=128, causal (preprocess + dK/dV + dQ)",
        "ms": round(ms, 4), "tflops": round(tf, 1), "frac": round(tf / tpk, 4),
        "convention": "2.5x the causal forward FLOPs",
        "tflops_own_gemms": round(tf_own, 1), "frac_own_gemms": round(tf_own / tpk, 4),
        "own_gemms": "3.5x the causal forward (S^T, dP^T, dV, dK and S, dP, dQ)",
        "peak": tpk, "unit": "TFLOP/s"}
    del q, k, v, do, o, lse, ws, dq, dk, dv

    # split-KV decode: B=8, H=32, d=128, lengths from the workload's seeded draw
    lens_np = np.random.default_rng(20264).integers(16384, 32769, size=8).astype(np.int32)
    lens = torch.from_numpy(lens_np).cuda()
    kc, vc, qd = rnd(8, 32, 32768, 128), rnd(8, 32, 32768, 128), rnd(8, 32, 128)
    ws = torch.empty(fa.fa_decode_workspace_size(8, 32, 32768, 128, 0), dtype=torch.uint8,
                     device="cuda")
    od = torch.empty_like(qd)
    ld = torch.empty((8, 32), dtype=torch.float32, device="cuda")
    ms = med_ms(lambda: fa.fa_decode_splitkv(qd, kc, vc, lens, o=od, lse=ld, workspace=ws))
    nbytes = C.decode_bytes(32, lens_np.tolist(), 128)
    gbs = nbytes / (ms * 1e-3) / 1e9
    res["decode_splitkv"] = {
        "workload": "split-KV decode B=8 H=32 d=128, cache lengths "
                    f"{lens_np.tolist()} (uniform [16384, 32768], seeded)",
        "us": round(ms * 1e3, 1), "bytes": nbytes, "gbs": round(gbs, 1),
        "frac": round(gbs / peaks["hbm_gbs"], 4), "peak": peaks["hbm_gbs"],
        "peak_kind": "measured copy rate (read + write); a read-mostly kernel can exceed it",
        "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4), "nominal_gbs": NOMINAL_HBM_GBS,
        "unit": "GB/s"}
    del kc, vc
    return res


def measure_next_rows(fa, torch, dev, flush, peaks, iters=8):
    """Rows beyond the headline step, timed on their own after it (not part
    of `value`): the FP8 forward on the prefill inputs (rotated, e4m3), and
    the paged grouped-query decode. Median of `iters` launches, L2 flushed
    before each."""
    import statistics

    def med_ms(fn):
        ts = []
        for _ in range(iters):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    B, H, N, d = dev["q"].shape
    g = torch.Generator(device="cuda").manual_seed(20264)
    signs = torch.where(torch.rand(d, device="cuda", generator=g) < 0.5, -1.0, 1.0)
    prep = fa.fa_fp8_prepare(dev["q"], dev["k"], dev["v"], signs)
    o = torch.empty_like(dev["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    rows = {"fwd_fp8": {
        "workload": f"prefill B={B} H={H} N={N} d={d}, Q and K rotated (random signs x Hadamard), "
                    "e4m3 with 128-row block scales, V e4m3 per head",
        "prep_ms": round(med_ms(lambda: fa.fa_fp8_prepare(dev["q"], dev["k"], dev["v"], signs,
                                                          out=prep)), 4),
        "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
        "peak_source": "2 x " + peaks["source"] + " (nominal fp8 / bf16 dense ratio)"}}
    for causal in (False, True):
        ms = med_ms(lambda: fa.fa_fwd_fp8(prep, causal=causal, o=o, lse=lse))
        tf = 4.0 * B * H * N * N * d / (2 if causal else 1) / (ms * 1e-3) / 1e12
        key = "causal" if causal else "full"
        rows["fwd_fp8"][f"ms_{key}"] = round(ms, 4)
        rows["fwd_fp8"][f"tflops_{key}"] = round(tf, 1)
        rows["fwd_fp8"][f"frac_{key}"] = round(tf / fp8_peak, 4)
    del prep, o, lse

    # bias (bf16 [1, H, N, N]) and dropout 0.1 on the prefill inputs:
    # forward without mask and causal, backward causal
    try:
        bias = torch.randn((1, H, N, N), device="cuda", dtype=torch.bfloat16, generator=g)
        ex = dict(bias=bias, p_drop=0.1, seed=20265, offset=0)
        oe = torch.empty_like(dev["q"])
        le = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        row = {"workload": f"prefill B={B} H={H} N={N} d={d}, bias [1, H, N, N] bf16, dropout 0.1",
               "unit": "TFLOP/s", "peak": peaks["bf16_tflops"]}
        for causal in (False, True):
            ms = med_ms(lambda: fa.fa_fwd_ex(dev["q"], dev["k"], dev["v"], causal=causal, o=oe,
                                             lse=le, **ex))
            key = "causal" if causal else "full"
            row[f"fwd_ms_{key}"] = round(ms, 4)
            row[f"fwd_tflops_{key}"] = round(4.0 * B * H * N * N * d / (2 if causal else 1)
                                             / (ms * 1e-3) / 1e12, 1)
        fa.fa_fwd_ex(dev["q"], dev["k"], dev["v"], causal=True, o=oe, lse=le, **ex)
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
        g3 = [torch.empty_like(dev["q"]) for _ in range(3)]
        ms = med_ms(lambda: fa.fa_bwd_ex(dev["q"], dev["k"], dev["v"], oe, le, dev["do"], causal=True,
                                         dq=g3[0], dk=g3[1], dv=g3[2], workspace=ws, **ex))
        row["bwd_ms_causal"] = round(ms, 4)
        row["bwd_tflops_causal"] = round(2.5 * 2.0 * B * H * N * N * d / (ms * 1e-3) / 1e12, 1)
        rows["bias_dropout"] = row
        del bias, oe, le, ws, g3
    except Exception as e:  # reported in the line, never fatal to the bench
        rows["bias_dropout"] = {"error": f"{type(e).__name__}: {e}"[:200]}

    # paged decode: B=8, Hq=32, Hkv=8, d=128, 64-row pages in a shuffled
    # order, lengths uniform in [16384, 32768]
    Bq, Hq, Hkv, page, cap = 8, 32, 8, 64, 32768
    lens = torch.randint(cap // 2, cap + 1, (Bq,), device="cuda", dtype=torch.int32, generator=g)
    max_pages = cap // page
    kp = torch.randn((Bq * max_pages, Hkv, page, d), device="cuda", dtype=torch.bfloat16, generator=g)
    vp = torch.randn((Bq * max_pages, Hkv, page, d), device="cuda", dtype=torch.bfloat16, generator=g)
    table = torch.randperm(Bq * max_pages, device="cuda", generator=g).to(torch.int32).view(Bq, max_pages)
    qd = torch.randn((Bq, Hq, d), device="cuda", dtype=torch.bfloat16, generator=g)
    ws = torch.empty(fa.fa_decode_workspace_size(Bq, Hq, cap, d, 0), dtype=torch.uint8, device="cuda")
    od = torch.empty_like(qd)
    lsed = torch.empty((Bq, Hq), dtype=torch.float32, device="cuda")
    call = lambda: fa.fa_decode_paged(qd, kp, vp, table, lens, o=od, lse=lsed, workspace=ws)  # noqa: E731
    ms = med_ms(call)
    kv_bytes = int(lens.sum().item()) * Hkv * d * 2 * 2
    gbs = kv_bytes / (ms * 1e-3) / 1e9
    # the split kernel alone: the library's CUDA events around its launch,
    # over `iters` calls, each after an L2 flush
    fa.fa_profile_begin()
    for _ in range(iters):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    prof = fa.fa_profile_end()
    n_split, t_split = prof.get("decode_split", (0, 0.0))
    n_merge, t_merge = prof.get("decode_merge", (0, 0.0))
    split_us = t_split / max(n_split, 1) * 1e3
    rows["decode_paged"] = {
        "workload": f"B={Bq} Hq={Hq} Hkv={Hkv} d={d}, {page}-row pages shuffled, lengths uniform "
                    f"[{cap // 2}, {cap}] (tensor-core kernel, keys as rows: 4 query heads per "
                    f"KV head; balanced tile split)",
        "us": round(ms * 1e3, 1), "gbs_unique_kv": round(gbs, 1), "peak": peaks["hbm_gbs"],
        "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
        "split_kernel_us": round(split_us, 1),
        "split_kernel_gbs": round(kv_bytes / (split_us * 1e-6) / 1e9, 1) if split_us > 0 else None,
        "merge_kernel_us": round(t_merge / max(n_merge, 1) * 1e3, 1)}
    del kp, vp
    return rows


def cpu_baseline(x, w, heads=16):
    """The fp64 oracle on a bounded sample: the step on `heads` heads of
    batch entry 0 (fwd no mask, fwd causal, bwd causal, decode of the last
    row), timed on the host cores."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import inputgen
    import oracle
    from exact_attention_130_b200 import counters as C

    def f64(b):
        return inputgen.bf16_bits_to_f32(b).astype(np.float64)

    q, k, v, do = (f64(x[n][0, :heads]) for n in ("q", "k", "v", "do"))
    t0 = time.perf_counter()
    oracle.attention_fwd(q, k, v, w.scale, False)
    oracle.attention_fwd(q, k, v, w.scale, True)
    oracle.attention_bwd(q, k, v, do, w.scale, True)
    oracle.decode(q[None, :, -1], k[None], v[None], np.array([w.N]), w.scale)
    dt = time.perf_counter() - t0
    fl = (C.fwd_flops(1, heads, w.N, w.d, False) + C.fwd_flops(1, heads, w.N, w.d, True)
          + C.bwd_flops(1, heads, w.N, w.d, True) + C.decode_flops(heads, [w.N], w.d))
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": round(fl / dt / 1e12, 5), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"the step on {heads} of {w.B * w.H} heads (batch entry 0), "
                      f"fp64 numpy, {dt:.1f} s"}


# ---------------------------------------------------------------------------
# reference arm: the oracle as it stands, rank 0 only
# ---------------------------------------------------------------------------
def run_reference(args, world, rank):
    if rank != 0:
        return
    import numpy as np
    from threadpoolctl import threadpool_info

    import inputgen
    import oracle
    from exact_attention_130_b200 import counters as C

    w = inputgen.WORKLOADS[WORKLOAD_NAME]
    x = inputgen.make_attention_inputs(w, with_grad=True)

    def f64(b):
        return inputgen.bf16_bits_to_f32(b).astype(np.float64)

    heads = 1  # one (batch, head) of the workload per step
    def one(i):
        b, h = divmod(i % (w.B * w.H), w.H)
        q, k, v, do = (f64(x[n][b, h:h + heads]) for n in ("q", "k", "v", "do"))
        oracle.attention_fwd(q, k, v, w.scale, False)
        oracle.attention_fwd(q, k, v, w.scale, True)
        oracle.attention_bwd(q, k, v, do, w.scale, True)
        oracle.decode(q[None, :, -1], k[None], v[None], np.array([w.N]), w.scale)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(args.warmup + i)
    dt = time.perf_counter() - t0
    fl = (C.fwd_flops(1, heads, w.N, w.d, False) + C.fwd_flops(1, heads, w.N, w.d, True)
          + C.bwd_flops(1, heads, w.N, w.d, True) + C.decode_flops(heads, [w.N], w.d))
    value = fl * args.steps / dt / 1e12
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    sample = f"one (batch, head) of the prefill workload per step, fp64 numpy oracle"
    line = {
        "metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (iid N(0,1), seeded, bf16 round-to-nearest-even)",
        "config": {"workload": "prefill B=4 H=16 N=2048 d=128; step = fwd (no mask) + fwd "
                               "(causal) + bwd (causal) + decode, on a sample of one head",
                   "B": w.B, "H": w.H, "N": w.N, "d": w.d},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_single_kernel(args):
    """Launch one entry point `iters` times on random inputs of the given
    shape (decode: N is the cache capacity, lengths drawn in [N/2, N])."""
    import torch

    import exact_attention_130_b200 as fa
    B, H, N, d = args.B, args.H, args.N, args.d
    g = torch.Generator(device="cuda").manual_seed(1)

    def rnd(*shape):
        return torch.randn(shape, device="cuda", dtype=torch.bfloat16, generator=g)

    if args.kernel == "decode_paged":
        # pages [P, Hkv, page, d] in a shuffled order; N is the cache capacity
        # per sequence, lengths drawn in [N/2, N]; H query heads share Hkv KV heads
        page, hkv = args.page, args.hkv
        lens = torch.randint(N // 2, N + 1, (B,), device="cuda", dtype=torch.int32, generator=g)
        max_pages = (N + page - 1) // page
        num_pages = B * max_pages
        kp, vp = rnd(num_pages, hkv, page, d), rnd(num_pages, hkv, page, d)
        perm = torch.randperm(num_pages, device="cuda", generator=g).to(torch.int32)
        table = perm.view(B, max_pages).contiguous()
        q = rnd(B, H, d)
        ws = torch.empty(fa.fa_decode_workspace_size(B, H, max_pages * page, d, 0),
                         dtype=torch.uint8, device="cuda")
        kv_bytes = int(lens.sum().item()) * hkv * d * 2 * 2
        fn = lambda: fa.fa_decode_paged(q, kp, vp, table, lens, workspace=ws)  # noqa: E731
    elif args.kernel in ("fwd_fp8", "fp8_prep"):
        # FP8 forward with incoherent processing: random signs, rotated and
        # block-quantised Q, K; the timed call is the forward on the codes
        # (fwd_fp8) or the preparation itself (fp8_prep)
        q, k, v = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
        signs = torch.where(torch.rand(d, device="cuda", generator=g) < 0.5, -1.0, 1.0)
        prep = fa.fa_fp8_prepare(q, k, v, signs)
        if args.kernel == "fp8_prep":
            fn = lambda: fa.fa_fp8_prepare(q, k, v, signs, out=prep)  # noqa: E731
        else:
            o, lse = fa.fa_fwd_fp8(prep, causal=bool(args.causal))
            fn = lambda: fa.fa_fwd_fp8(prep, causal=bool(args.causal), o=o, lse=lse)  # noqa: E731
    elif args.kernel == "decode":
        # lengths drawn as the split-KV decode workload draws them (seed
        # 20264, uniform [N/2, N]): B=8 H=32 N=32768 is that workload
        import numpy as np
        q, kc, vc = rnd(B, H, d), rnd(B, H, N, d), rnd(B, H, N, d)
        lens = torch.from_numpy(np.random.default_rng(20264).integers(
            N // 2, N + 1, size=B).astype(np.int32)).cuda()
        ws = torch.empty(fa.fa_decode_workspace_size(B, H, N, d, 0), dtype=torch.uint8, device="cuda")
        fn = lambda: fa.fa_decode_splitkv(q, kc, vc, lens, workspace=ws)  # noqa: E731
    elif args.kernel in ("fwd_ex", "bwd_ex"):
        q, k, v, do = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
        bias = rnd(1, H, N, N) if args.bias else None
        ex = dict(causal=bool(args.causal), bias=bias, p_drop=args.p_drop, seed=1234, offset=0)
        o, lse = fa.fa_fwd_ex(q, k, v, **ex)
        if args.kernel == "fwd_ex":
            fn = lambda: fa.fa_fwd_ex(q, k, v, o=o, lse=lse, **ex)  # noqa: E731
        else:
            ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
            dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
            fn = lambda: fa.fa_bwd_ex(q, k, v, o, lse, do, dq=dq, dk=dk, dv=dv,  # noqa: E731
                                      workspace=ws, **ex)
    else:
        q, k, v, do = rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d), rnd(B, H, N, d)
        o, lse = fa.fa_fwd(q, k, v, causal=bool(args.causal))
        if args.kernel == "fwd":
            fn = lambda: fa.fa_fwd(q, k, v, causal=bool(args.causal), o=o, lse=lse)  # noqa: E731
        elif args.kernel == "fwd_pair":
            fn = lambda: fa.fa_fwd_pair(q, k, v, causal=bool(args.causal), o=o, lse=lse)  # noqa: E731
        else:
            ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
            dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
            fn = lambda: fa.fa_bwd(q, k, v, o, lse, do, causal=bool(args.causal), dq=dq, dk=dk,  # noqa: E731
                                   dv=dv, workspace=ws)
    torch.cuda.synchronize()
    for i in range(args.iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        extra = ""
        if args.kernel == "decode_paged":
            extra = (f" Hkv={args.hkv} page={args.page}: "
                     f"{kv_bytes / (a.elapsed_time(b) * 1e-3) / 1e9:.1f} GB/s of KV pages")
        elif args.kernel in ("fwd", "fwd_pair", "fwd_fp8", "fwd_ex"):
            fl = 4.0 * B * H * N * N * d / (2 if args.causal else 1)
            extra = f": {fl / (a.elapsed_time(b) * 1e-3) / 1e12:.1f} TFLOP/s"
        print(f"{args.kernel} B={B} H={H} N={N} d={d} causal={args.causal} "
              f"iter {i}: {a.elapsed_time(b):.4f} ms{extra}", flush=True)
    st, word = fa.fa_device_status()
    if st != 0:
        raise SystemExit(f"device status {st} ({word:#x})")


def main():
    args = parse_args()
    world, rank, local = dist_setup()
    if args.kernel:
        run_single_kernel(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
