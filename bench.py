#!/usr/bin/env python
"""Throughput of exact attention forward + backward on B200, one JSON line.

One step = the whole hot path once over one batch: fa_fwd (O, lse) then
fa_bwd (dQ, dK, dV) on the 4K-token MHA workload (B=4, Hq=Hkv=32, N=4096,
d=128, causal, bf16) unless --workload names another.  FLOPs follow the
stated convention: forward 4*B*Hq*N^2*d, halved when causal; backward 2.5x
forward.  ``value`` is whole-job TFLOPS (all ranks); every rank runs its own
replica (the path has no exchange step), so scaling is weak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle arm
  python bench.py --window W | --dropout P | --block-mask KIND | --decode | --fp8   # the variants

Timing: W untimed steps, then K steps between a barrier + synchronize on both
sides, CUDA events on the launching stream, max over ranks.  The inputs
(Q, K, V, dO: 512 MiB for the default workload) are larger than L2.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_io_aware_bwd_b200 import binding  # noqa: E402
from exact_io_aware_bwd_b200.build import build  # noqa: E402
from exact_io_aware_bwd_b200.workloads import WORKLOADS  # noqa: E402

METRIC = "attention fwd+bwd TFLOPS/GPU at N=4K–64K, d=128, and % of B200 bf16 peak"
UNIT = "TFLOPS"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the backward main kernel on the default workload, from one ncu capture of
# that kernel, with a digest of the kernel sources it was taken on: reported
# only while the sources are unchanged.
PROFILED_TRAFFIC = {"workload": "mha4k", "bytes": 1295312384, "sources_sha256_16": "ad6562f226110961",
                    "sources": ("exact_io_aware_bwd_b200/csrc/fa_bwd.cuh",
                                "exact_io_aware_bwd_b200/csrc/sm100.cuh")}
# The same for the forward kernel (one launch on the default workload).
PROFILED_TRAFFIC_FWD = {"workload": "mha4k", "bytes": 516944128, "sources_sha256_16": "404444234fe2e56c",
                        "sources": ("exact_io_aware_bwd_b200/csrc/fa_fwd.cuh",
                                    "exact_io_aware_bwd_b200/csrc/sm100.cuh")}
# The same for the FP8 forward kernel (one launch on the 4K-token MHA shape).
PROFILED_TRAFFIC_FP8 = {"workload": "mha4k", "bytes": 305240832, "sources_sha256_16": "481515a16f74b0cd",
                        "sources": ("exact_io_aware_bwd_b200/csrc/fa_fwd_fp8.cuh",
                                    "exact_io_aware_bwd_b200/csrc/sm100.cuh")}
# The same for one decode step (split and merge launch) at 16K cached tokens.
PROFILED_TRAFFIC_DEC = {"workload": "decode B=32 Hq=32 Hkv=8 Nq=1 d=128 L=16384 page=64", "bytes": 2155173376,
                        "sources_sha256_16": "63499268775b3e64",
                        "sources": ("exact_io_aware_bwd_b200/csrc/fa_decode.cuh",
                                    "exact_io_aware_bwd_b200/csrc/sm100.cuh")}


def profiled_traffic(workload_name, spec=PROFILED_TRAFFIC):
    import hashlib
    h = hashlib.sha256()
    try:
        for f in spec["sources"]:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    if workload_name != spec["workload"] or h.hexdigest()[:16] != spec["sources_sha256_16"]:
        return None
    return spec["bytes"]


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def workload_desc(w, causal):
    return (f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} "
            f"{'causal' if causal else 'non-causal'} {str(w.dtype).replace('torch.', '')}")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        p = torch.cuda.get_device_properties(device)
        self.bus = f"{p.pci_bus_id:02X}:{p.pci_device_id:02X}"
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            bus = parts[0].upper()
            if self.bus not in bus and len({r[0] for r in rows} | {bus}) > 1:
                continue
            rows.append(parts)
        os.unlink(self.path)
        mine = [r for r in rows if self.bus in r[0].upper()] or rows
        if not mine:
            return None
        sm = [float(r[1]) for r in mine if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in mine if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in mine for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(mine)}


# ---------------------------------------------------------------- our arm

def max_over_ranks(x, world, device):
    """The largest value of x over the ranks (one all-reduce; x itself when alone)."""
    if world <= 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world, flops_per_replica_step, ms_per_step):
    """Whole-job throughput: every rank runs one replica of the step."""
    return world * flops_per_replica_step / (ms_per_step * 1e-3) / 1e12


def rank_seed(w, rank):
    """Seed of a rank's synthetic inputs (replicas draw different data)."""
    return w.seed + 1000 * rank


def kernel_stats(ms):
    """Mean, median and min of per-launch times (ms)."""
    return {"mean": statistics.mean(ms), "median": statistics.median(ms), "min": min(ms)}


def block_mask_for(kind, w):
    """A block mask over 128 x 128 blocks for workload w, by name:
    'local': each query block sees itself and the 2 key blocks before it,
    plus the first key block (global tokens), and the first query block sees
    all; 'random:RHO': every (head, query block, key block) visible with
    probability RHO (seeded), the diagonal always."""
    nb = -(-w.N // 128)
    if kind == "local":
        m = torch.zeros((nb, nb), dtype=torch.uint8)
        for i in range(nb):
            m[i, max(0, i - 2):i + 1] = 1
        m[:, 0] = 1
        m[0, :] = 1
        return m
    if kind.startswith("random:"):
        rho = float(kind.split(":", 1)[1])
        g = torch.Generator("cpu").manual_seed(w.seed + 13)
        m = (torch.rand((w.Hq, nb, nb), generator=g) < rho).to(torch.uint8)
        m[:, torch.arange(nb), torch.arange(nb)] = 1
        return m
    raise SystemExit(f"bench.py: unknown block mask {kind!r} (local | random:RHO)")


def visible_pairs(mask, w, causal):
    """(query, key) pairs a block mask (and the causal mask) leaves visible,
    summed over heads and batch entries."""
    nb = mask.shape[-1]
    sizes = torch.tensor([min(128, w.N - 128 * i) for i in range(nb)], dtype=torch.float64)
    pair = sizes[:, None] * sizes[None, :]
    if causal:
        # off-diagonal blocks below the diagonal are whole; a diagonal block
        # of n rows has n(n+1)/2 visible pairs
        pair = torch.tril(pair, -1) + torch.diag(sizes * (sizes + 1) / 2)
    m = mask.to(torch.float64)
    per_head = (m * pair).sum(dim=(-1, -2))
    total = per_head.sum() * (w.Hq if m.dim() == 2 else 1)
    return float(total) * w.B


def alloc_problem(w, rank, device, block_mask=False):
    """Device tensors of one replica of workload w (inputs drawn on the device)."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    g = torch.Generator(device=device).manual_seed(rank_seed(w, rank))
    mk = lambda H, s: (torch.randn((B, H, N, d), generator=g, device=device, dtype=torch.float32) * s).to(w.dtype)
    q, k, v, do = mk(Hq, w.sigma_qk), mk(Hkv, w.sigma_qk), mk(Hkv, w.sigma_vdo), mk(Hq, w.sigma_vdo)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), device=device, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = (binding.fa_bwd_blockmask_workspace_bytes if block_mask else binding.fa_bwd_workspace_bytes)(
        B, Hq, Hkv, N, d)
    ws = torch.empty(nbytes, device=device, dtype=torch.uint8)
    return dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ws=ws)


def make_step(t, w, causal, W, DR, stream, fwd_ev=None, bwd_ev=None, BM=None):
    """One pass of the hot path (fa_fwd then fa_bwd) on the tensors t; with
    events, the i-th call records around each of the two calls on `stream`."""
    q, k, v, do, o, lse, dq, dk, dv, ws = (t[n] for n in ("q", "k", "v", "do", "o", "lse", "dq", "dk", "dv", "ws"))
    scale = w.scale

    def step(i=None):
        if i is not None:
            fwd_ev[i][0].record(stream)
        if BM is not None:
            binding.fa_fwd_blockmask(q, k, v, o, lse, scale, causal, BM, stream)
        elif DR:
            binding.fa_fwd_dropout(q, k, v, o, lse, scale, causal, DR[0], DR[1], stream)
        elif W:
            binding.fa_fwd_window(q, k, v, o, lse, scale, W, stream)
        else:
            binding.fa_fwd(q, k, v, o, lse, scale, causal, stream)
        if i is not None:
            fwd_ev[i][1].record(stream)
            bwd_ev[i][0].record(stream)
        if BM is not None:
            binding.fa_bwd_blockmask(q, k, v, o, do, lse, dq, dk, dv, scale, causal, BM, ws, stream)
        elif DR:
            binding.fa_bwd_dropout(q, k, v, o, do, lse, dq, dk, dv, scale, causal, DR[0], DR[1], ws, stream)
        elif W:
            binding.fa_bwd_window(q, k, v, o, do, lse, dq, dk, dv, scale, W, ws, stream)
        else:
            binding.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, scale, causal, ws, stream)
        if i is not None:
            bwd_ev[i][1].record(stream)
    return step


def time_steps(args, w, causal, rank, world, device, steps, warmup, W=0, DR=None, clocks=None, BM=None):
    """W untimed steps, then `steps` timed ones between a barrier and a
    synchronize on both sides, with CUDA events on the launching stream
    around the whole region only (the step time of the headline value); then
    the same number of steps again with events around every fa_fwd and
    fa_bwd call and (through the library) around every launch of the forward
    kernel and of the backward main kernel, for the breakdown (those events
    add a few microseconds a call to the stream, so they stay out of the
    first region).  Returns the timings (ms; the total is the max over
    ranks)."""
    t = alloc_problem(w, rank, device, block_mask=BM is not None)
    stream = torch.cuda.current_stream(device)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    K = steps
    fwd_ev = [(ev(), ev()) for _ in range(K)]
    bwd_ev = [(ev(), ev()) for _ in range(K)]
    kf_ev = [(ev(), ev()) for _ in range(K)]
    kb_ev = [(ev(), ev()) for _ in range(K)]
    for a, b in kf_ev + kb_ev:  # materialise the handles the library records into
        a.record(stream)
        b.record(stream)
    step = make_step(t, w, causal, W, DR, stream, fwd_ev, bwd_ev, BM)
    # the clock sampler starts first (it needs a moment), then the warm-up
    # steps run right before the timed ones, so that the GPU does not idle
    # (and lower its clock) between the two
    if clocks:
        clocks.start()
        time.sleep(0.3)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    assert binding.fa_get_device_status(stream) == binding.FA_OK

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    t0, t1 = ev(), ev()
    barrier()
    torch.cuda.synchronize(device)
    t0.record(stream)
    for i in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    # a pause, so that the breakdown runs from the same power state as the
    # timed region (a loop right after it runs under the 1 kW power cap),
    # then the warm-up steps again
    time.sleep(1.0)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    barrier()
    for i in range(K):
        binding.fa_set_profile_events(binding.KERNEL_FWD, *kf_ev[i])
        binding.fa_set_profile_events(binding.KERNEL_BWD_MAIN, *kb_ev[i])
        step(i)
    torch.cuda.synchronize(device)
    barrier()
    binding.fa_set_profile_events(binding.KERNEL_FWD, None, None)
    binding.fa_set_profile_events(binding.KERNEL_BWD_MAIN, None, None)
    clk = clocks.stop() if clocks else None
    status = binding.fa_get_device_status(stream)
    assert status == binding.FA_OK, binding.fa_status_string(status)
    el = lambda pairs: [a.elapsed_time(b) for a, b in pairs]
    res = dict(ms_total=max_over_ranks(t0.elapsed_time(t1), world, device),
               fwd=kernel_stats(el(fwd_ev)), bwd=kernel_stats(el(bwd_ev)),
               fwd_kernel=kernel_stats(el(kf_ev)), bwd_main=kernel_stats(el(kb_ev)),
               clocks=clk, tensors=t)
    return res


def summarize(w, causal, res, K, peak, W=0, flops=None):
    """TFLOPS and % of peak of a timed run (medians of per-call times)."""
    f_fwd, f_bwd = flops if flops else (w.flops_fwd(causal, W), w.flops_bwd(causal, W))
    tf = lambda f, ms: f / (ms * 1e-3) / 1e12
    fwd, bwd, bm = res["fwd"]["median"], res["bwd"]["median"], res["bwd_main"]["median"]
    return {
        "workload": workload_desc(w, causal) + (f" window={W}" if W else ""),
        "ms_per_step": round(res["ms_total"] / K, 4),
        "tflops": round(tf(f_fwd + f_bwd, res["ms_total"] / K), 2),
        "pct_of_peak": round(100 * tf(f_fwd + f_bwd, res["ms_total"] / K) / peak, 2),
        "fwd_ms": round(fwd, 4), "fwd_ms_min": round(res["fwd"]["min"], 4),
        "fwd_tflops": round(tf(f_fwd, fwd), 2), "fwd_pct_of_peak": round(100 * tf(f_fwd, fwd) / peak, 2),
        "bwd_ms": round(bwd, 4), "bwd_ms_min": round(res["bwd"]["min"], 4),
        "bwd_tflops": round(tf(f_bwd, bwd), 2), "bwd_pct_of_peak": round(100 * tf(f_bwd, bwd) / peak, 2),
        "bwd_main_ms": round(bm, 4), "bwd_main_ms_min": round(res["bwd_main"]["min"], 4),
        "bwd_main_tflops": round(tf(f_bwd, bm), 2),
        "steps": K,
    }


# Configurations of the metric's range besides the headline one, timed after
# it on the same GPU and reported as sub-results of the same line.
RANGE_WORKLOADS = ("gqa16k", "long64k")


def run_ours(args, w, causal, rank, world, device):
    torch.cuda.set_device(device)
    build()
    binding.load()
    W = args.window
    DR = (args.dropout, 0x5EED0000 + rank) if args.dropout else None
    BMh = block_mask_for(args.block_mask, w) if args.block_mask else None
    BM = BMh.to(device) if BMh is not None else None
    K = args.steps
    clocks = ClockSampler(device) if rank == 0 else None
    res = time_steps(args, w, causal, rank, world, device, K, args.warmup, W, DR, clocks, BM)
    clk = res["clocks"]
    t = res.pop("tensors")
    ms_step = res["ms_total"] / K
    f_fwd, f_bwd = w.flops_fwd(causal, W), w.flops_bwd(causal, W)
    if BM is not None:
        # FLOPs over the (query, key) pairs the mask leaves visible
        f_fwd = 4.0 * w.d * visible_pairs(BMh, w, causal)
        f_bwd = 2.5 * f_fwd
    value = job_tflops(world, f_fwd + f_bwd, ms_step)
    fwd_ms, bwd_ms = res["fwd"]["median"], res["bwd"]["median"]
    fwd_kern_mean, bwd_main_mean = res["fwd_kernel"]["mean"], res["bwd_main"]["mean"]
    stream = torch.cuda.current_stream(device)

    # end to end through the C ABI with host buffers: every step copies the
    # step's inputs in from pinned host memory, runs fwd + bwd and copies all
    # results back.  Two sets of device buffers on two streams let one
    # step's copies back overlap the next step's copies in (the two
    # directions use separate copy engines) and the kernels.
    e2e = None
    if not args.no_e2e:
        ev = lambda: torch.cuda.Event(enable_timing=True)
        q, k, v, do, o, lse, dq, dk, dv, ws = (t[n] for n in ("q", "k", "v", "do", "o", "lse", "dq", "dk", "dv", "ws"))
        hin = [x.cpu().pin_memory() for x in (q, k, v, do)]
        outs_like = (o, lse, dq, dk, dv)
        sets = [dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ws=ws)]
        sets.append({n: torch.empty_like(x) for n, x in sets[0].items()})
        hout = [[torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in outs_like] for _ in sets]
        streams = [torch.cuda.Stream(device) for _ in sets]
        steps_e = [make_step(b, w, causal, W, DR, st, BM=BM) for b, st in zip(sets, streams)]
        h2d = sum(x.numel() * x.element_size() for x in hin)
        d2h = sum(x.numel() * x.element_size() for x in hout[0])

        def e2e_step(i):
            b, st, ho = sets[i % 2], streams[i % 2], hout[i % 2]
            with torch.cuda.stream(st):
                for name, src in zip(("q", "k", "v", "do"), hin):
                    b[name].copy_(src, non_blocking=True)
                steps_e[i % 2]()
                for dst, name in zip(ho, ("o", "lse", "dq", "dk", "dv")):
                    dst.copy_(b[name], non_blocking=True)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(device)
        Ke = max(4, min(K, 10))
        e0, e1 = ev(), ev()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)
        e0.record(stream)
        for st in streams:
            st.wait_event(e0)
        for i in range(Ke):
            e2e_step(i)
        for st in streams:
            done = ev()
            done.record(st)
            stream.wait_event(done)
        e1.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        status = binding.fa_get_device_status(stream)
        assert status == binding.FA_OK, binding.fa_status_string(status)
        ems = max_over_ranks(e0.elapsed_time(e1) / Ke, world, device)
        e2e = {"value": job_tflops(world, f_fwd + f_bwd, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "copies": "pinned host buffers; two device buffer sets on two streams, so a "
                         "step's copies back overlap the next step's copies in"}
        del sets, hin, hout
    del t

    pk, pk_kind = peaks()
    peak = pk["bf16_tflops"]
    head = summarize(w, causal, res, K, peak, W, (f_fwd, f_bwd))
    bwd_tflops_main = f_bwd / (bwd_main_mean * 1e-3) / 1e12
    launches_per_step = 4  # fa_fwd_kernel, fa_bwd_pre_kernel, fa_bwd_kernel, fa_bwd_post_kernel
    if BM is not None:
        launches_per_step += 1  # fa_bwd_plan_kernel
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": str(w.dtype).replace("torch.", ""),
        "data": "synthetic: seeded normals (per-rank CUDA generator) with the workload's shapes and sigmas",
        "config": {"workload": workload_desc(w, causal) + (f" window={W}" if W else "")
                   + (f" dropout={args.dropout}" if DR else "")
                   + (f" block_mask={args.block_mask} (visible fraction "
                      f"{f_fwd / w.flops_fwd(causal):.3f})" if BM is not None else ""),
                   "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
                   "seq_len": w.N, "head_dim": w.d, "causal": causal, "window": W,
                   "dropout": args.dropout,
                   "parallelism": f"replicas x{world} (no exchange)",
                   "l2": "inputs larger than L2 (no flush)",
                   "flops_per_step": f_fwd + f_bwd},
        "pct_of_peak": round(100 * value / world / peak, 2),
        "fwd_ms": head["fwd_ms"], "fwd_ms_min": head["fwd_ms_min"],
        "fwd_tflops": head["fwd_tflops"], "fwd_pct_of_peak": head["fwd_pct_of_peak"],
        "bwd_ms": head["bwd_ms"], "bwd_ms_min": head["bwd_ms_min"],
        "bwd_tflops": head["bwd_tflops"], "bwd_pct_of_peak": head["bwd_pct_of_peak"],
        "bwd_main_ms": head["bwd_main_ms"], "bwd_main_ms_min": head["bwd_main_ms_min"],
        "bwd_main_tflops": head["bwd_main_tflops"],
        "timing_stats": "fwd/bwd: median (and min) of per-call CUDA-event times on the launch stream; "
                        "roofline: mean of the kernel's per-launch times",
        "roofline": {"kernel": "fa_bwd_kernel (main backward pass)", "bound": "tensor",
                     "achieved": round(bwd_tflops_main, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(bwd_tflops_main / peak, 4), "peak_kind": f"{pk_kind} bf16 burst",
                     "traffic": (profiled_traffic(w.name)
                                 if causal and not (W or DR or BM is not None) else None),
                     "traffic_unit": "bytes per launch (ncu)",
                     "algorithmic": "2.5 x 4*B*Hq*N^2*d (/2 causal) FLOPs per launch"
                                    + (" (visible pairs under the window)" if W else "")
                                    + (" (visible pairs under the block mask)" if BM is not None else "")},
        "forward_kernel": {"kernel": "fa_fwd_kernel", "bound": "tensor",
                           "achieved": round(f_fwd / (fwd_kern_mean * 1e-3) / 1e12, 2), "peak": peak,
                           "unit": "TFLOP/s",
                           "frac": round(f_fwd / (fwd_kern_mean * 1e-3) / 1e12 / peak, 4),
                           "traffic": (profiled_traffic(w.name, PROFILED_TRAFFIC_FWD)
                                       if causal and not (W or DR or BM is not None) else None)},
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
        "e2e": e2e,
    }
    # the rest of the metric's range (N = 16K GQA, N = 64K fp16), each on
    # its own inputs, fewer steps (each step is longer)
    if not (W or DR or BM is not None or args.no_range) and w.name == "mha4k" and causal:
        subs = []
        for name in RANGE_WORKLOADS:
            ws_ = WORKLOADS[name]
            Ks = max(3, min(K, 10))
            r = time_steps(args, ws_, True, rank, world, device, Ks, 3)
            r.pop("tensors")
            torch.cuda.empty_cache()
            sub = summarize(ws_, True, r, Ks, peak)
            sub["gpu_launches"] = launches_per_step * Ks
            subs.append(sub)
        line["range"] = subs
    return line


def run_decode(args, rank, world, device):
    """Decode over a paged KV cache: B sequences of L cached tokens each, Nq
    new query tokens, pages of 64 tokens scattered through the pool.  The
    kernel pair is memory bound: value = cache bytes read per second."""
    torch.cuda.set_device(device)
    build()
    binding.load()
    B, Hq, Hkv, Nq, d, P, L = 32, 32, 8, 1, 128, 64, args.decode_len
    dt = torch.bfloat16
    npg = (L + P - 1) // P
    num_pages = B * npg
    g = torch.Generator(device=device).manual_seed(4321 + rank)
    perm = torch.randperm(num_pages, generator=g, device=device).to(torch.int32)
    table = perm.view(B, npg).contiguous()
    lens = torch.full((B,), L, dtype=torch.int32, device=device)
    kc = torch.randn((num_pages, Hkv, P, d), generator=g, device=device, dtype=torch.float32).to(dt)
    vc = torch.randn((num_pages, Hkv, P, d), generator=g, device=device, dtype=torch.float32).to(dt)
    q = torch.randn((B, Hq, Nq, d), generator=g, device=device, dtype=torch.float32).to(dt)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), device=device, dtype=torch.float32)
    ws = torch.empty(binding.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, d, npg), device=device,
                     dtype=torch.uint8)
    stream = torch.cuda.current_stream(device)
    scale = 1.0 / math.sqrt(d)
    step = lambda: binding.fa_decode_paged(q, kc, vc, table, lens, o, lse, scale, ws, stream)
    clocks = ClockSampler(device) if rank == 0 else None
    if clocks:  # started before the warm-up, which then runs right before the timed steps
        clocks.start()
        time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    assert binding.fa_get_device_status(stream) == binding.FA_OK
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop() if clocks else None
    assert binding.fa_get_device_status(stream) == binding.FA_OK
    ms = max_over_ranks(t0.elapsed_time(t1) / K, world, device)
    cache_bytes = 2 * B * L * Hkv * d * 2                      # K and V read once
    io_bytes = cache_bytes + 2 * q.numel() * 2 + lse.numel() * 4  # + q read, O and lse written
    gbs = world * io_bytes / (ms * 1e-3) / 1e9
    pk, pk_kind = peaks()
    workload = f"decode B={B} Hq={Hq} Hkv={Hkv} Nq={Nq} d={d} L={L} page=64"
    return {
        "metric": "paged-KV decode: cache bytes read per second", "value": round(gbs, 1),
        "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bfloat16",
        "data": "synthetic: seeded normals, pages of 64 tokens in a shuffled pool",
        "config": {"workload": workload,
                   "parallelism": f"replicas x{world} (no exchange)",
                   "l2": "cache larger than L2 (no flush)" if cache_bytes > 126e6 else "cache fits L2"},
        "tokens_per_s": round(world * B * Nq / (ms * 1e-3), 1),
        "roofline": {"kernel": "fa_decode_split_kernel + fa_decode_merge_kernel", "bound": "hbm",
                     "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / pk["hbm_gbs"], 4), "peak_kind": f"{pk_kind} copy",
                     "traffic": profiled_traffic(workload, PROFILED_TRAFFIC_DEC),
                     "traffic_unit": "bytes per step, split + merge (ncu)",
                     "algorithmic": "K and V cache read once, q read, O and lse written"},
        "gpu_launches": 2 * K,
        "clocks": clk,
    }


def run_fp8(args, w, causal, rank, world, device):
    """FP8 forward only: Q, K, V as E4M3 codes with per-tensor factors, O in
    bf16.  FLOPs by the forward convention; roofline against the FP8 tensor
    peak, taken as the measured bf16 peak times the nominal FP8:bf16 ratio 2."""
    from exact_io_aware_bwd_b200.workloads import make_fp8_inputs
    torch.cuda.set_device(device)
    build()
    binding.load()
    (q8, k8, v8), descale = make_fp8_inputs(w, seed=rank_seed(w, rank))
    q8, k8, v8 = (t.to(device) for t in (q8, k8, v8))
    B, Hq, N, d = q8.shape
    o = torch.empty((B, Hq, N, d), device=device, dtype=torch.bfloat16)
    lse = torch.empty((B, Hq, N), device=device, dtype=torch.float32)
    stream = torch.cuda.current_stream(device)
    step = lambda: binding.fa_fwd_fp8(q8, k8, v8, o, lse, w.scale, descale, causal, stream)
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K)]
    for e in ev:
        e.record(stream)  # creates the event handle the library records into
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(device) if rank == 0 else None
    if clocks:  # started before the warm-up, which then runs right before the timed steps
        clocks.start()
        time.sleep(0.3)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(device)
    assert binding.fa_get_device_status(stream) == binding.FA_OK
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    t0.record(stream)
    for i in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    # the same steps again with events around every kernel launch (kept out
    # of the timed region above: each event adds a little to the stream),
    # after a pause and the warm-up, from the same power state
    time.sleep(1.0)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(device)
    for i in range(K):
        binding.fa_set_profile_events(binding.KERNEL_FWD, ev[2 * i], ev[2 * i + 1])
        step()
    torch.cuda.synchronize(device)
    binding.fa_set_profile_events(binding.KERNEL_FWD)
    clk = clocks.stop() if clocks else None
    assert binding.fa_get_device_status(stream) == binding.FA_OK
    ms = max_over_ranks(t0.elapsed_time(t1) / K, world, device)
    kern_ms = statistics.mean(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K))
    flops = w.flops_fwd(causal)
    value = job_tflops(world, flops, ms)
    pk, pk_kind = peaks()
    peak8 = 2.0 * pk["bf16_tflops"]
    achieved = flops / (kern_ms * 1e-3) / 1e12
    in_bytes = q8.numel() + k8.numel() + v8.numel()
    return {
        "metric": "FP8 attention forward TFLOPS/GPU", "value": round(value, 1), "unit": "TFLOPS",
        "n_gpus": world, "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic: seeded normals quantised to E4M3 with per-tensor factors",
        "config": {"workload": workload_desc(w, causal).replace(str(w.dtype).replace("torch.", ""),
                                                                  "e4m3 in, bf16 out"),
                   "parallelism": f"replicas x{world} (no exchange)",
                   "l2": "inputs larger than L2 (no flush)" if in_bytes > 126e6 else "inputs fit L2"},
        "roofline": {"kernel": "fa_fwd_fp8_kernel", "bound": "tensor", "achieved": round(achieved, 1),
                     "peak": round(peak8, 1), "unit": "TFLOP/s", "frac": round(achieved / peak8, 4),
                     "peak_kind": f"{pk_kind} bf16 burst x 2 (nominal FP8:bf16 ratio)",
                     "traffic": profiled_traffic(w.name, PROFILED_TRAFFIC_FP8) if causal else None,
                     "algorithmic_bytes": in_bytes + o.numel() * 2 + lse.numel() * 4,
                     "kernel_ms": round(kern_ms, 4)},
        "gpu_launches": K,
        "clocks": clk,
    }


# ---------------------------------------------------------------- CPU oracle

_ORACLE_INPUTS = {}


# Share of the conventional fwd + bwd FLOPs that the oracle's row sample
# performs: the forward row (S and P V, 2 of the 7 products the convention
# counts) and the dQ row (S, dP and dQ, 3 more); the key-side products dV and
# dK are not in the sample.
ORACLE_ROW_SHARE = 5.0 / 7.0


def oracle_sample(w, causal, seconds, rows_hint=None):
    """Times the fp64 oracle (forward rows + dQ rows) on seeded query rows of
    one head of the workload; returns (TFLOPS-equivalent, rows, s, threads).
    Each row is credited the FLOPs of the products it computes: 5/7 of its
    share of the workload's conventional fwd + bwd FLOPs."""
    import oracle
    from exact_io_aware_bwd_b200.workloads import make_inputs
    g = torch.Generator().manual_seed(w.seed + 3)
    per_row = ORACLE_ROW_SHARE * (w.flops_fwd(causal) + w.flops_bwd(causal)) / (w.B * w.Hq * w.N)
    heads_max = min(w.B * w.Hq, 64)
    key = (w.name, heads_max)
    if key not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[key] = make_inputs(w, shape_override=(1, heads_max, heads_max, w.N, w.d))
    q, k, v, do = _ORACLE_INPUTS[key]

    def run(nrows):
        # nrows query rows in total: the same seeded rows in each of H heads
        H = min(heads_max, max(1, -(-nrows // w.N)))
        per_head = min(w.N, max(1, nrows // H))
        rows = torch.sort(torch.randperm(w.N, generator=g)[:per_head]).values.numpy()
        t = time.perf_counter()
        oracle.fwd_rows(q[:, :H], k[:, :H], v[:, :H], rows, w.scale, causal)
        oracle.bwd_rows(q[:, :H], k[:, :H], v[:, :H], do[:, :H], rows, w.scale, causal)
        return time.perf_counter() - t, H * per_head

    threads = oracle.num_threads()
    if rows_hint is None:
        # calibrate on a probe of at least ~1 s, then size the sample
        probe = 4 * threads
        while True:
            dt, n = run(probe)
            if dt >= 1.0 or probe >= heads_max * w.N:
                break
            probe = min(heads_max * w.N, probe * 4)
        rows_hint = max(1, min(heads_max * w.N, int(n * seconds / max(dt, 1e-6))))
    dt, n = run(rows_hint)
    return per_row * n / dt / 1e12, n, dt, threads


def oracle_sample_fp8(w, causal, seconds):
    """Times the fp64 oracle's FP8 forward (E4M3 decode + forward rows) on
    seeded query rows of the first heads of the workload; returns
    (TFLOPS-equivalent, rows, s, threads), each row counted at its share of
    the forward FLOPs."""
    import oracle
    from exact_io_aware_bwd_b200.workloads import make_fp8_inputs
    H = min(w.B * w.Hq, 8)
    (q8, k8, v8), ds = make_fp8_inputs(w, shape_override=(1, H, H, w.N, w.d))
    per_row = w.flops_fwd(causal) / (w.B * w.Hq * w.N)
    g = torch.Generator().manual_seed(w.seed + 5)

    def run(per_head):
        rows = torch.sort(torch.randperm(w.N, generator=g)[:per_head]).values.numpy()
        t = time.perf_counter()
        oracle.fwd_fp8_rows(q8, k8, v8, ds, rows, w.scale, causal)
        return time.perf_counter() - t, H * per_head

    per_head = 4
    while True:
        dt, n = run(per_head)
        if dt >= 1.0 or per_head >= w.N:
            break
        per_head = min(w.N, per_head * 4)
    per_head = max(1, min(w.N, int(per_head * seconds / max(dt, 1e-6))))
    dt, n = run(per_head)
    return per_row * n / dt / 1e12, n, dt, oracle.num_threads()


def run_reference(args, w, causal):
    """The oracle arm: each step is a bounded sample of the same workload."""
    budget = 150.0
    per_step = max(0.2, min(10.0, budget / max(1, args.steps + args.warmup)))
    _, rows, dt, threads = oracle_sample(w, causal, per_step)
    vals = []
    for i in range(args.warmup + args.steps):
        v, _, dt, _ = oracle_sample(w, causal, per_step, rows_hint=rows)
        if i >= args.warmup:
            vals.append((v, dt))
    value = statistics.mean(v for v, _ in vals)
    ms = 1e3 * statistics.mean(dt for _, dt in vals)
    sample = (f"{rows} seeded query rows per step (forward O/lse rows + dQ rows, fp64; each row "
              f"credited the 5 of 7 conventional products it computes), {workload_desc(w, causal)}")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload_desc(w, causal)},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mha4k", choices=sorted(WORKLOADS))
    ap.add_argument("--noncausal", action="store_true", help="non-causal variant of the workload")
    ap.add_argument("--decode", action="store_true",
                    help="time decode over a paged KV cache instead (B=32, Hq=32, Hkv=8, d=128)")
    ap.add_argument("--decode-len", type=int, default=16384, help="cached tokens per sequence (--decode)")
    ap.add_argument("--fp8", action="store_true",
                    help="time the FP8 forward (E4M3 Q, K, V; bf16 O) on the workload's shape")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="dropout probability on the attention probabilities (0: none)")
    ap.add_argument("--window", type=int, default=0,
                    help="causal sliding window of this many keys (0: none); FLOPs counted over visible pairs")
    ap.add_argument("--block-mask", default="",
                    help="block-sparse mask over 128 x 128 blocks: 'local' or 'random:RHO'; FLOPs "
                         "counted over visible pairs")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (small cases for profiler captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-range", action="store_true",
                    help="skip the 16K GQA and 64K fp16 sub-results of the default line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    assert args.warmup >= 0 and args.steps >= 1

    w = WORKLOADS[args.workload]
    if args.batch:
        from dataclasses import replace
        w = replace(w, B=args.batch)
    causal = (not args.noncausal) and (True in w.causal_modes)
    if sum(bool(x) for x in (args.window, args.dropout, args.block_mask)) > 1:
        raise SystemExit("bench.py: --window, --dropout and --block-mask are not combined")
    if args.window:
        assert args.window > 0 and causal, "--window needs a causal workload"
        if args.impl == "reference":
            raise SystemExit("bench.py: the reference arm times the plain workload only (no --window)")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w, causal)), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device; the product path has no CPU fallback")
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.cuda.set_device(device)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        if args.decode or args.fp8:
            line = (run_decode(args, rank, world, device) if args.decode
                    else run_fp8(args, w, causal, rank, world, device))
            if rank == 0 and args.fp8 and not args.no_cpu_baseline:
                v, rows, dt, threads = oracle_sample_fp8(w, causal, args.cpu_seconds)
                line["cpu_baseline"] = {
                    "value": round(v, 6), "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                    "sample": f"{rows} seeded query rows of the FP8 forward (E4M3 decode, fp64 rows), "
                              f"{dt:.1f} s; each row counted at its share of the forward FLOPs"}
            if rank == 0:
                print(json.dumps(line), flush=True)
            return
        line = run_ours(args, w, causal, rank, world, device)
        if rank == 0 and not args.no_cpu_baseline and not (args.window or args.dropout or args.block_mask):
            v, rows, dt, threads = oracle_sample(w, causal, args.cpu_seconds)
            line["cpu_baseline"] = {
                "value": round(v, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                "sample": f"{rows} seeded query rows, forward O/lse rows + dQ rows in fp64, "
                          f"{dt:.1f} s; each row credited the 5 of 7 conventional products it "
                          f"computes (no dK/dV)"}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
