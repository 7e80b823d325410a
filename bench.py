"""Benchmark: exact attention forward + backward on B200, attention TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path over one batch of synthetic input:
the forward (O, LSE) followed by the backward (D and the zeroed dQ
accumulator, the main dK/dV/dQ kernel, the dQ conversion), all through the C
ABI of libfa_b200.so on the caller's CUDA stream.  FLOPs follow the pages'
convention: forward 4·B·H·N²·d (halved when causal), backward 2.5× forward.

Timing: W warm-up steps, then K timed steps.  Before every step a 256 MiB
buffer is written to flush the 126 MB L2; each step is bracketed by CUDA
events on the stream the kernels run on (and each kernel by its own events,
for the per-kernel roofline).  Under torchrun every rank runs its own copy
of the workload (independent heads and sequences: weak scaling, no data-path
collective); the time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), on a
bounded sample of the same workload: the pages describe the method but ship
no code, so the oracle is the reference arm.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# NVIDIA's datasheet dense BF16 tensor figure for one B200 (its doubled figure assumes 2:4 sparsity);
# reported beside the measured cuBLAS peak, which is the denominator of every `frac_of_peak`.
NOMINAL_DENSE_BF16_TFLOPS = 2250.0
E2E_MODE = ("every step copies its inputs in from pinned host memory and its results out; two buffer slots let "
            "the next step's inputs and the previous step's results cross PCIe while a step computes")
FP8_OVER_BF16 = 2.0  # nominal dense e4m3 / bf16 tensor throughput (4.5 / 2.25 PFLOP/s)
NOMINAL_SOURCE = "NVIDIA B200 datasheet, dense BF16 (2.25 PFLOP/s; 4.5 with 2:4 sparsity)"
METRIC = "attention TFLOP/s (fwd, fwd+bwd) on 1 B200 and % of dense bf16 tensor peak"
DEFAULT_WORKLOAD = "causal_n8k_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# The source files each profiled kernel is built from: its own file and the two shared headers.
KERNEL_SOURCES = {
    "fa_fwd_kernel": ["fa_fwd.cu", "sm100.cuh", "fa_internal.h"],
    "fa_bwd_main_q128_kernel": ["fa_bwd.cu", "sm100.cuh", "fa_internal.h"],
    "fa_bwd_dropout": ["fa_bwd.cu", "sm100.cuh", "fa_internal.h"],
    "fa_decode_split_kernel": ["fa_decode.cu", "sm100.cuh", "fa_internal.h"],
    "fa_merge_kernel": ["fa_merge.cu", "sm100.cuh", "fa_internal.h"],
}


def kernel_source_hash(kernel):
    """Hash of the sources `kernel` is built from (every file under csrc/ for a kernel not listed)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_90_b200", "csrc")
    for name in sorted(KERNEL_SOURCES.get(kernel, os.listdir(csrc))):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload, dropout_p=0.0):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel source
    (entries of the dropout variant are keyed "<workload>+dropout<p>")."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload if dropout_p <= 0.0 else f"{workload}+dropout{dropout_p:g}")
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons through NVML every
    ~10 ms while the timed region runs (read-only; no setting is changed)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self.handle = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def start(self):
        try:
            import pynvml
            self.nvml = pynvml
            self.handle = self._handle()
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.handle = None
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                clk = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((float(clk), int(rs)))
            except Exception:
                pass
            time.sleep(0.01)

    def stop(self):
        if self.handle is None:
            return None
        self._stop.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return None
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": float(np.median([c for c, _ in self.samples])), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "NVML, 10 ms polling"}


# ----------------------------------------------------------------------------- distributed plumbing


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "gloo" if args.impl == "reference" else "nccl"
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(x, pg, device=None):
    if pg is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- GPU arm


def pipelined_e2e(stream, n, host_in, dev_in, dev_out, host_out, compute):
    """Time n end-to-end steps through the public API: every step copies its inputs from pinned host
    memory (host_in → dev_in[slot]), computes (``compute(slot)`` on ``stream``) and copies its results
    back (dev_out[slot] → host_out[slot]).  Two slots of buffers let step i+1's inputs stream in and
    step i−1's results stream out (PCIe is full duplex; each direction on its own stream) while step i
    computes; events keep a slot's copies and compute in order.  Returns ms per step (device events:
    the start is recorded before the first copy, the end after the last copy-out)."""
    import torch
    dev = stream.device
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_done, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    s_in.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(n):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])  # step i−2 has finished reading this slot's inputs
            for d, h in zip(dev_in[b], host_in):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])  # step i−2's results have left this slot
        compute(b)
        ev_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            for h, d in zip(host_out[b], dev_out[b]):
                h.copy_(d, non_blocking=True)
            ev_out[b].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1) / n


def run_gpu(args, world, rank, local, pg):
    import torch

    import workloads
    import exact_io_aware_90_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    wname = args.workload
    spec = workloads.WORKLOADS[wname]
    inp_h = workloads.make_workload(wname, backward=spec["backward"])
    # weak scaling: each rank gets its own seeded copy of the workload
    if rank > 0:
        inp_h = workloads.random_inputs(inp_h.H, inp_h.d, inp_h.dtype, spec["seed"] + 1000 * rank, B=inp_h.B,
                                        N=inp_h.N, seqlens=inp_h.seqlens if inp_h.cu_seqlens is not None else None,
                                        causal=inp_h.causal, backward=spec["backward"])
    backward = spec["backward"]
    B, H, N, d, T = inp_h.B, inp_h.H, inp_h.N, inp_h.d, inp_h.T
    dt = fa.dtype_code(inp_h.q)
    scale, causal = inp_h.scale, int(inp_h.causal)
    flops_fwd = 4.0 * H * d * sum(float(L) * L for L in inp_h.seqlens) * (0.5 if causal else 1.0)
    flops_bwd = 2.5 * flops_fwd if backward else 0.0

    # device buffers
    q, k, v = inp_h.q.to(dev), inp_h.k.to(dev), inp_h.v.to(dev)
    do = inp_h.do.to(dev) if backward else None
    cu = inp_h.cu_seqlens.to(dev) if inp_h.cu_seqlens is not None else None
    cu_p = cu.data_ptr() if cu is not None else None
    o = torch.empty_like(q)
    lse = torch.empty((T, H), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3)) if backward else (None, None, None)
    ws_bytes = fa.fa_bwd_workspace_bytes(T, H, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if backward else None
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def check(st, where):
        if st != fa.FA_OK:
            raise fa.FAError(st, where)

    def fwd():
        check(fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                        causal, cu_p, T, dt, sp), "fa_fwd")

    def bwd_pre():
        check(fa.fa_bwd_preprocess(o.data_ptr(), do.data_ptr(), B, H, N, d, cu_p, T, dt, ws.data_ptr(), ws_bytes, sp),
              "fa_bwd_preprocess")

    def bwd_main():
        check(fa.fa_bwd_main(q.data_ptr(), k.data_ptr(), v.data_ptr(), lse.data_ptr(), do.data_ptr(), dk.data_ptr(),
                             dv.data_ptr(), B, H, N, d, scale, causal, cu_p, T, dt, ws.data_ptr(), ws_bytes, sp),
              "fa_bwd_main")

    def bwd_post():
        check(fa.fa_bwd_postprocess(dq.data_ptr(), B, H, N, d, scale, cu_p, T, dt, ws.data_ptr(), ws_bytes, sp),
              "fa_bwd_postprocess")

    drop_p, drop_seed, drop_off = float(args.dropout), 0x5EED, 0

    def fwd_drop():
        check(fa.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d,
                                scale, causal, cu_p, T, dt, drop_p, drop_seed, drop_off, sp), "fa_fwd_dropout")

    def bwd_drop():  # one call: D = rowsum(dO∘O), the main kernel, dQ conversion (three launches)
        check(fa.fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, scale, causal, cu_p, T, dt,
                                drop_p, drop_seed, drop_off, ws.data_ptr(), ws_bytes, sp), "fa_bwd_dropout")

    if drop_p > 0.0:
        stages = [("fa_fwd_kernel", fwd_drop)]
        launches = {"fa_fwd_kernel": 1}
        if backward:
            stages += [("fa_bwd_dropout", bwd_drop)]
            launches["fa_bwd_dropout"] = 3
        flops_of = {"fa_fwd_kernel": flops_fwd, "fa_bwd_dropout": flops_bwd}
    else:
        stages = [("fa_fwd_kernel", fwd)]
        if backward:
            stages += [("fa_bwd_pre_kernel", bwd_pre), ("fa_bwd_main_q128_kernel", bwd_main),
                       ("fa_bwd_post_kernel", bwd_post)]
        launches = {name: 1 for name, _ in stages}
        flops_of = {"fa_fwd_kernel": flops_fwd, "fa_bwd_main_q128_kernel": flops_bwd}
    drop_kw = dict(dropout_p=drop_p, seed=drop_seed, offset=drop_off) if drop_p > 0.0 else {}

    def one_step(record):
        flush.fill_(1)  # outside the timed events
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
        evs[0].record(stream)
        for i, (_, fn) in enumerate(stages):
            fn()
            evs[i + 1].record(stream)
        if record is not None:
            record.append(evs)

    for _ in range(args.warmup):
        one_step(None)
    torch.cuda.synchronize(dev)
    st = fa.fa_check_device_status(sp)
    if st != fa.FA_OK:
        raise fa.FAError(st, "warm-up")

    clocks = ClockSampler(dev)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    recs = []
    for _ in range(args.steps):
        one_step(recs)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if pg is not None:
        pg.barrier()
    st = fa.fa_check_device_status(sp)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed steps")
    step_ms = [r[0].elapsed_time(r[-1]) for r in recs]
    per_kernel = {name: float(np.mean([r[i].elapsed_time(r[i + 1]) for r in recs]))
                  for i, (name, _) in enumerate(stages)}
    total_ms = max_over_ranks(float(np.sum(step_ms)), pg, dev)
    ms_per_step = total_ms / args.steps
    flops_step = flops_fwd + flops_bwd
    value = world * flops_step / (ms_per_step * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region,
    # pipelined across steps over two buffer slots (see pipelined_e2e)
    pin = lambda t: None if t is None else t.pin_memory()
    host_in = [pin(t) for t in (inp_h.q, inp_h.k, inp_h.v, inp_h.do) if t is not None]
    mk_out = lambda: [o, lse] + ([dq, dk, dv] if backward else [])
    dev_out = [mk_out(), [torch.empty_like(t) for t in mk_out()]]
    dev_in = [[q, k, v] + ([do] if backward else []), [torch.empty_like(t, device=dev) for t in host_in]]
    host_out = [[torch.empty_like(t, device="cpu").pin_memory() for t in dev_out[0]] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])

    def e2e_compute(b):
        qi, ki, vi = dev_in[b][:3]
        oo, ll = dev_out[b][:2]
        fa.attention_forward(qi, ki, vi, causal=bool(causal), scale=scale, cu_seqlens=cu,
                             max_seqlen=N if cu is not None else None, batch=B, out=oo, lse=ll, stream=sp, **drop_kw)
        if backward:
            g = dev_out[b][2:]
            fa.attention_backward(qi, ki, vi, oo, ll, dev_in[b][3], causal=bool(causal), scale=scale, cu_seqlens=cu,
                                  max_seqlen=N if cu is not None else None, batch=B, dq=g[0], dk=g[1], dv=g[2],
                                  workspace=ws, stream=sp, **drop_kw)

    e2e_steps = max(2, min(args.steps, 6))
    pipelined_e2e(stream, 2, host_in, dev_in, dev_out, host_out, e2e_compute)  # warm-up
    e2e_ms = max_over_ranks(pipelined_e2e(stream, e2e_steps, host_in, dev_in, dev_out, host_out, e2e_compute),
                            pg, dev)
    st = fa.fa_check_device_status(sp)
    if st != fa.FA_OK:
        raise fa.FAError(st, "e2e steps")
    # the forward is deterministic: the last step's O, copied out, is the other slot's O
    if not torch.equal(host_out[(e2e_steps - 1) % 2][0], dev_out[e2e_steps % 2][0].cpu()):
        raise RuntimeError("the end-to-end steps' output differs between buffer slots")

    # ---- the forward alone (inference use): same workload, same L2 flush, back-to-back steps
    fwd_only = None
    if backward:
        fwd_fn = stages[0][1]
        for _ in range(args.warmup):
            flush.fill_(1)
            fwd_fn()
        torch.cuda.synchronize(dev)
        fo_clocks = ClockSampler(dev)
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize(dev)
        fo_clocks.start()
        fo = []
        for _ in range(args.steps):
            flush.fill_(1)  # outside the timed events
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fwd_fn()
            b.record(stream)
            fo.append((a, b))
        torch.cuda.synchronize(dev)
        fo_clk = fo_clocks.stop()
        st = fa.fa_check_device_status(sp)
        if st != fa.FA_OK:
            raise fa.FAError(st, "forward-only steps")
        fo_ms = max_over_ranks(float(np.mean([x.elapsed_time(y) for x, y in fo])), pg, dev)
        fwd_only = {"ms": round(fo_ms, 4), "tflops": round(flops_fwd / (fo_ms * 1e-3) / 1e12, 1), "clocks": fo_clk}

    # ---- roofline of the dominant kernel
    peaks = load_peaks()
    dom = max(per_kernel, key=per_kernel.get)
    dom_ms = per_kernel[dom]
    if dom in flops_of:
        achieved = flops_of[dom] / (dom_ms * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "frac_of_sustained": round(achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4),
                "peak_source": peaks["source"] + " (burst bf16; kernels timed one launch at a time)",
                "traffic": load_traffic(dom, wname, drop_p), "launch_ms": round(dom_ms, 4)}
        if dom == "fa_bwd_dropout":
            roof["note"] = "time of the whole dropout backward call (D = rowsum(dO∘O), main kernel, dQ conversion)"
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": None, "traffic": load_traffic(dom, wname, drop_p)}
    kernels = {}
    for name, ms in per_kernel.items():
        e = {"ms": round(ms, 4)}
        if name in flops_of:
            e["tflops"] = round(flops_of[name] / (ms * 1e-3) / 1e12, 1)
            e["frac_of_peak"] = round(e["tflops"] / peaks["bf16_tflops"], 4)
        kernels[name] = e

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": inp_h.dtype,
        "data": "synthetic: i.i.d. N(0,1) q, k, v, dO from a seeded CPU generator, rounded to the dtype",
        "config": {"workload": wname, "B": B, "H": H, "N": N, "d": d, "causal": bool(causal),
                   "varlen": inp_h.cu_seqlens is not None, "tokens": T, "step": "fwd+bwd" if backward else "fwd",
                   "flops_per_step": flops_step, "l2": "flushed before every step (256 MiB write, outside the events)",
                   "parallelism": f"replicas x{world} (independent workloads per GPU)",
                   "dropout_p": drop_p},
        "fwd_tflops": round(flops_fwd / (per_kernel["fa_fwd_kernel"] * 1e-3) / 1e12, 1),
        "fwd_frac_of_peak": round(flops_fwd / (per_kernel["fa_fwd_kernel"] * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
        "pct_of_peak": round(100.0 * value / world / peaks["bf16_tflops"], 2),
        # the forward kernel timed in a forward-only loop (inference use; the fwd+bwd step above times it right
        # after the previous step's backward)
        "fwd_only": (None if fwd_only is None else
                     dict(fwd_only, frac_of_peak=round(fwd_only["tflops"] / peaks["bf16_tflops"], 4),
                          frac_of_sustained=round(fwd_only["tflops"] / peaks.get("bf16_tflops_sustained",
                                                                                 peaks["bf16_tflops"]), 4),
                          frac_of_nominal=round(fwd_only["tflops"] / NOMINAL_DENSE_BF16_TFLOPS, 4))),
        "nominal_peak": {"tflops": NOMINAL_DENSE_BF16_TFLOPS, "source": NOMINAL_SOURCE},
        "kernels": kernels,
        "roofline": roof,
        "e2e": {"value": round(world * flops_step / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": E2E_MODE},
        "gpu_launches": sum(launches.values()) * args.steps,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = (cpu_baseline_dropout(inp_h, drop_p, budget_s=args.cpu_budget) if drop_p > 0.0 else
                               cpu_baseline(inp_h, budget_s=args.cpu_budget))
    return out


# ----------------------------------------------------------------------------- CPU oracle (baseline / reference arm)


def run_gpu_decode(args, world, rank, local, pg):
    """Decode workloads: one query per sequence over a device-resident K/V cache (HBM-bound)."""
    import torch

    import workloads
    import exact_io_aware_90_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    wname = args.workload
    spec = workloads.DECODE_WORKLOADS[wname]
    inp_h = workloads.make_decode_workload(wname)
    if rank > 0:  # weak scaling: each rank its own seeded copy
        inp_h = workloads.decode_inputs(inp_h.H, inp_h.d, inp_h.dtype, spec["seed"] + 1000 * rank, B=inp_h.B,
                                        Nk=inp_h.Nk, seqlens=inp_h.seqlens if inp_h.cu_seqlens_k is not None else None)
    B, H, Nk, d, Tk = inp_h.B, inp_h.H, inp_h.Nk, inp_h.d, inp_h.Tk
    dt = fa.dtype_code(inp_h.q)
    flops = 4.0 * H * d * float(sum(inp_h.seqlens))  # q·Kᵀ and p·V, 2 FLOP per multiply-add
    elt = 2
    algo_bytes = 2 * Tk * H * d * elt + 2 * B * H * d * elt + B * H * 4  # K, V once; q, o; lse
    q, k, v = inp_h.q.to(dev), inp_h.k.to(dev), inp_h.v.to(dev)
    cu = inp_h.cu_seqlens_k.to(dev) if inp_h.cu_seqlens_k is not None else None
    o = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    ws_bytes = fa.fa_decode_workspace_bytes(B, H, Nk, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        st = fa.fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Nk, d,
                          inp_h.scale, cu.data_ptr() if cu is not None else None, Tk, dt, ws.data_ptr(), ws_bytes, sp)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_decode")

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1)  # outside the timed events: the cache is read from HBM every step
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    st = fa.fa_check_device_status(sp)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed steps")
    ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])), pg, dev)
    value = world * flops / (ms * 1e-3) / 1e12
    # end to end through the public API: the new query in from pinned host memory, the output back (the cache
    # stays resident on the device, as it does while generating)
    hq = inp_h.q.pin_memory()
    ho = torch.empty_like(hq).pin_memory()
    hl = torch.empty((B, H), dtype=torch.float32).pin_memory()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        fa.attention_decode(q, k, v, scale=inp_h.scale, cu_seqlens_k=cu, max_seqlen_k=Nk if cu is not None else None,
                            out=o, lse=lse, workspace=ws, stream=sp)
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, min(args.steps, 10))
    a.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, pg, dev)
    peaks = load_peaks()
    gbs = algo_bytes / (ms * 1e-3) / 1e9
    out = {
        "metric": METRIC + " (decode: one query per sequence)",
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": inp_h.dtype,
        "data": "synthetic: i.i.d. N(0,1) q, k, v from a seeded CPU generator, rounded to the dtype",
        "config": {"workload": wname, "B": B, "H": H, "Nk": Nk, "d": d, "varlen": cu is not None, "keys": Tk,
                   "step": "decode", "flops_per_step": flops,
                   "l2": "flushed before every step (256 MiB write, outside the events)",
                   "parallelism": f"replicas x{world} (independent workloads per GPU)"},
        "roofline": {"kernel": "fa_decode_split_kernel + fa_decode_merge_kernel", "bound": "hbm",
                     "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": load_traffic("fa_decode_split_kernel", wname),  # the split kernel: the K/V stream
                     "algorithmic_bytes": algo_bytes, "peak_source": peaks["source"]},
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(hq.numel() * hq.element_size()),
                "d2h_bytes_per_step": int(ho.numel() * ho.element_size() + hl.numel() * 4)},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_decode(inp_h, budget_s=args.cpu_budget)
    return out


MERGE_WORKLOADS = {"ring_merge_t32k_h16_d128": dict(T=32768, H=16, d=128, dtype="bf16", seed=1009)}


def run_gpu_merge(args, world, rank, local, pg):
    """The ring path's elementwise kernels (HBM-bound) at the headline's token count: the merge of a
    normalised block result into the fp32 running (O, LSE), the last merge straight into the output dtype,
    and the fp32 accumulation of a dK/dV block part.  GB/s of algorithmic bytes against the HBM peak."""
    import torch

    import exact_io_aware_90_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    w = MERGE_WORKLOADS[args.workload]
    T, H, d = w["T"], w["H"], w["d"]
    g = torch.Generator().manual_seed(w["seed"] + 1000 * rank)
    tdt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float16
    part_o = torch.randn(T, H, d, generator=g).to(tdt).to(dev)
    part_lse = torch.randn(T, H, generator=g).to(dev)
    acc_o = torch.randn(T, H, d, generator=g).to(dev)
    acc_lse = torch.randn(T, H, generator=g).to(dev)
    out_o = torch.empty_like(part_o)
    acc = torch.randn(T * H * d, generator=g).to(dev)
    dt = fa.dtype_code(part_o)
    n, rows = T * H * d, T * H
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def merge(first_out):
        st = fa.fa_attn_merge(acc_o.data_ptr(), acc_lse.data_ptr(), part_o.data_ptr(), part_lse.data_ptr(),
                              out_o.data_ptr() if first_out else None, T, H, d, dt, 0, sp)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_attn_merge")

    def accumulate():
        st = fa.fa_accumulate(acc.data_ptr(), part_o.data_ptr(), None, n, dt, 0, sp)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_accumulate")

    # algorithmic bytes per launch: a running merge reads the part (2 B) and the fp32 accumulator and writes
    # it back (4 + 4 B) per element, and per row reads the part LSE and reads and writes the running LSE;
    # the last merge writes the output dtype (2 B) instead of the accumulator; the accumulation reads the
    # fp32 accumulator and the part and writes the accumulator back
    kernels = [("fa_merge_kernel (running)", lambda: merge(False), n * 10 + rows * 12),
               ("fa_merge_kernel (last)", lambda: merge(True), n * 8 + rows * 12),
               ("fa_accum_kernel", accumulate, n * 10)]
    for _ in range(args.warmup):
        for _, fn, _ in kernels:
            flush.fill_(1)
            fn()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    times = {name: [] for name, _, _ in kernels}
    for _ in range(args.steps):
        for name, fn, _ in kernels:
            flush.fill_(1)  # outside the timed events
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            times[name].append((a, b))
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    st = fa.fa_check_device_status(sp)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed steps")
    peaks = load_peaks()
    per = {}
    for name, _, nbytes in kernels:
        ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in times[name]])), pg, dev)
        gbs = nbytes / (ms * 1e-3) / 1e9
        per[name] = {"ms": round(ms, 4), "bytes": nbytes, "gbs": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4)}
    step_ms = sum(v["ms"] for v in per.values())
    step_bytes = sum(nb for _, _, nb in kernels)
    value = world * step_bytes / (step_ms * 1e-3) / 1e9
    dom = max(per, key=lambda k: per[k]["ms"])
    return {
        "metric": "ring-merge kernels: algorithmic HBM GB/s", "value": round(value, 1), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"],
        "data": "synthetic: N(0,1) partial O and running O/LSE from a seeded CPU generator",
        "config": {"workload": args.workload, "T": T, "H": H, "d": d, "step": "merge (running) + merge (last) + "
                   "accumulate", "l2": "flushed before every launch (256 MiB write, outside the events)",
                   "parallelism": f"replicas x{world} (independent workloads per GPU)"},
        "kernels": per,
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": per[dom]["gbs"], "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": per[dom]["frac"], "traffic": load_traffic("fa_merge_kernel", args.workload),
                     "peak_source": peaks["source"]},
        "e2e": None,
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }


def real_inputs(inp):
    """e4m3 inputs as the float64 values they stand for (NumPy, so the oracle widens nothing through
    float32: e4m3 × an fp32 descale needs up to 28 significand bits)."""
    import workloads
    ds = inp.extra["descale"]
    return workloads.AttnInputs(workloads.real_values(inp.q, ds["q"]), workloads.real_values(inp.k, ds["k"]),
                                workloads.real_values(inp.v, ds["v"]), None, inp.cu_seqlens, list(inp.seqlens),
                                inp.B, inp.H, inp.N, inp.d, inp.scale, inp.causal, "f64", inp.name)


def run_gpu_fp8(args, world, rank, local, pg):
    """The forward with e4m3 inputs (per-tensor descales, bf16 output): TFLOP/s by the same FLOP
    convention, against the e4m3 tensor peak."""
    import torch

    import workloads
    import exact_io_aware_90_b200 as fa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    wname = args.workload
    spec = workloads.WORKLOADS[wname]
    inp_h = workloads.make_workload(wname)
    if rank > 0:  # weak scaling: each rank its own seeded copy
        inp_h = workloads.random_inputs(inp_h.H, inp_h.d, "e4m3", spec["seed"] + 1000 * rank, B=inp_h.B, N=inp_h.N,
                                        causal=inp_h.causal, backward=False)
    B, H, N, d, T = inp_h.B, inp_h.H, inp_h.N, inp_h.d, inp_h.T
    ds = inp_h.extra["descale"]
    scale, causal = inp_h.scale, int(inp_h.causal)
    flops = 4.0 * H * d * sum(float(L) * L for L in inp_h.seqlens) * (0.5 if causal else 1.0)
    q, k, v = inp_h.q.to(dev), inp_h.k.to(dev), inp_h.v.to(dev)
    o = torch.empty((T, H, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, H), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def fwd():
        st = fa.fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d, scale,
                           causal, None, T, ds["q"], ds["k"], ds["v"], sp)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_fwd_fp8")

    for _ in range(args.warmup):
        flush.fill_(1)
        fwd()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    evs = []
    for _ in range(args.steps):
        flush.fill_(1)  # outside the timed events
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fwd()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if pg is not None:
        pg.barrier()
    st = fa.fa_check_device_status(sp)
    if st != fa.FA_OK:
        raise fa.FAError(st, "timed steps")
    ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])), pg, dev)
    value = world * flops / (ms * 1e-3) / 1e12
    # the same forward with one descale per (128-token block, head) (fa_fwd_fp8_per_block): the inputs'
    # per-tensor descales repeated into [num_blocks, H] arrays, so the output is the same computation
    nb = B * ((N + 127) // 128)
    blk = {n: torch.full((nb, H), float(ds[n]), dtype=torch.float32, device=dev) for n in ("q", "k", "v")}

    def fwd_block():
        st = fa.fa_fwd_fp8_per_block(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N,
                                     d, scale, causal, None, T, blk["q"].data_ptr(), blk["k"].data_ptr(),
                                     blk["v"].data_ptr(), nb, sp)
        if st != fa.FA_OK:
            raise fa.FAError(st, "fa_fwd_fp8_per_block")

    for _ in range(args.warmup):
        flush.fill_(1)
        fwd_block()
    evb = []
    for _ in range(args.steps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fwd_block()
        b.record(stream)
        evb.append((a, b))
    torch.cuda.synchronize(dev)
    st = fa.fa_check_device_status(sp)
    if st != fa.FA_OK:
        raise fa.FAError(st, "per-block steps")
    ms_blk = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evb])), pg, dev)
    # end to end through the public API: e4m3 inputs from pinned host memory, O and LSE back, pipelined
    # across steps over two buffer slots (see pipelined_e2e)
    host_in = [inp_h.q.pin_memory(), inp_h.k.pin_memory(), inp_h.v.pin_memory()]
    dev_in = [[q, k, v], [torch.empty_like(t) for t in (q, k, v)]]
    dev_out = [[o, lse], [torch.empty_like(o), torch.empty_like(lse)]]
    host_out = [[torch.empty_like(t, device="cpu").pin_memory() for t in (o, lse)] for _ in range(2)]

    def e2e_compute(b):
        qi, ki, vi = dev_in[b]
        fa.attention_forward_fp8(qi, ki, vi, ds["q"], ds["k"], ds["v"], causal=bool(causal), scale=scale, batch=B,
                                 out=dev_out[b][0], lse=dev_out[b][1], stream=sp)

    pipelined_e2e(stream, 2, host_in, dev_in, dev_out, host_out, e2e_compute)  # warm-up
    n_e2e = max(2, min(args.steps, 6))
    e2e_ms = max_over_ranks(pipelined_e2e(stream, n_e2e, host_in, dev_in, dev_out, host_out, e2e_compute), pg, dev)
    if not torch.equal(host_out[(n_e2e - 1) % 2][0], dev_out[n_e2e % 2][0].cpu()):
        raise RuntimeError("the end-to-end steps' output differs between buffer slots")
    peaks = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    out = {
        "metric": METRIC + " (e4m3 inputs, forward)",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic: i.i.d. N(0,1) q, k, v from a seeded CPU generator, divided by amax/448 per tensor and "
                "rounded to e4m3",
        "config": {"workload": wname, "B": B, "H": H, "N": N, "d": d, "causal": bool(causal), "tokens": T,
                   "step": "fwd", "flops_per_step": flops, "output": "bf16",
                   "l2": "flushed before every step (256 MiB write, outside the events)",
                   "parallelism": f"replicas x{world} (independent workloads per GPU)"},
        "roofline": {"kernel": "fa_fwd_kernel (e4m3)", "bound": "tensor", "achieved": round(value / world, 1),
                     "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(value / world / fp8_peak, 4),
                     "frac_of_bf16_peak": round(value / world / peaks["bf16_tflops"], 4),
                     "peak_source": peaks["source"] + f" (burst bf16) x {FP8_OVER_BF16:g}, the nominal e4m3/bf16 "
                                                      "dense ratio (4.5 / 2.25 PFLOP/s)",
                     "traffic": load_traffic("fa_fwd_kernel", wname), "launch_ms": round(ms, 4)},
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": 3 * T * H * d, "mode": E2E_MODE,
                "d2h_bytes_per_step": T * H * d * 2 + T * H * 4},
        "gpu_launches": args.steps,
        "clocks": clk,
        "per_block_descales": {"ms": round(ms_blk, 4), "tflops": round(flops / (ms_blk * 1e-3) / 1e12, 1),
                               "frac": round(flops / (ms_blk * 1e-3) / 1e12 / fp8_peak, 4),
                               "note": "fa_fwd_fp8_per_block on the same inputs, one descale per (128-token block, "
                                       "head); timed after the per-tensor steps, outside the headline value"},
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(real_inputs(inp_h), budget_s=args.cpu_budget)
        out["cpu_baseline"]["sample"] += " (the real values of the e4m3 inputs)"
    return out


def decode_oracle_seq(inp, n):
    """fp64 oracle decode of sequence n (all heads).  Returns (seconds, flops credited)."""
    import oracle
    lo = int(sum(inp.seqlens[:n]))
    L = int(inp.seqlens[n])
    t0 = time.perf_counter()
    oracle.decode_forward(inp.q[n:n + 1], inp.k[lo:lo + L], inp.v[lo:lo + L], inp.scale, cu_seqlens_k=[0, L])
    return time.perf_counter() - t0, 4.0 * inp.H * inp.d * L


def cpu_baseline_decode(inp, budget_s=15.0):
    """Whole sequences (all heads) through the oracle until about `budget_s` seconds of CPU work."""
    tot_t, tot_f, n = 0.0, 0.0, 0
    while n < inp.B and tot_t < budget_s:
        dt, f = decode_oracle_seq(inp, n)
        tot_t, tot_f, n = tot_t + dt, tot_f + f, n + 1
    return {"value": round(tot_f / max(tot_t, 1e-9) / 1e12, 6), "unit": "TFLOP/s", **host_threads(),
            "kind": "oracle", "sample": f"fp64 NumPy oracle decode of {n} whole sequence(s), all heads, {tot_t:.2f} s"}


def run_reference_decode(args):
    import workloads
    inp = workloads.make_decode_workload(args.workload)
    for _ in range(args.warmup):
        decode_oracle_seq(inp, 0)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, f = decode_oracle_seq(inp, 0)
        times.append(dt)
        flops = f
    ms = 1e3 * float(np.mean(times))
    value = flops / (ms * 1e-3) / 1e12
    return {
        "impl": "reference", "metric": METRIC + " (decode: one query per sequence)", "value": round(value, 6),
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "B": inp.B, "H": inp.H, "Nk": inp.Nk, "d": inp.d, "sample": "sequence 0"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", **host_threads(), "kind": "oracle",
                         "sample": "fp64 NumPy oracle decode of sequence 0 (all heads) per step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(n[0])
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def host_threads():
    """The oracle's thread counts: `cores` = the threads its work ran on (NumPy's BLAS pool; the rest of
    the oracle is single-threaded), beside the cores this process may run on and the BLAS pool size."""
    n = blas_threads()
    return {"cores": n, "cores_available": len(os.sched_getaffinity(0)), "blas_threads": n}


def oracle_sample(inp, rows, head=0):
    """fp64 oracle forward+backward on one head of the first sequence, query rows [L-rows, L).

    Returns (seconds, flops credited by the same convention as the GPU arm)."""
    import oracle
    L = inp.seqlens[0]
    lo = max(0, L - rows)
    sl = slice(0, L)
    t0 = time.perf_counter()
    oracle.attention_fwd_bwd_rows(inp.q[sl], inp.k[sl], inp.v[sl],
                                  inp.do[sl] if inp.do is not None else inp.q[sl], lo, L, inp.scale, inp.causal,
                                  head=head)
    dt = time.perf_counter() - t0
    # visible (query, key) pairs of the sampled rows, times 4·d, times 3.5 for fwd+bwd
    pairs = sum((i + 1) if inp.causal else L for i in range(lo, L))
    f = 4.0 * inp.d * pairs * (3.5 if inp.do is not None else 1.0)
    return dt, f


def cpu_baseline(inp, budget_s=15.0):
    """Whole heads of sequence 0 through the oracle until about `budget_s` seconds of CPU work."""
    L = inp.seqlens[0]
    tot_t, tot_f, heads = 0.0, 0.0, 0
    for h in range(inp.H):
        dt, f = oracle_sample(inp, L, head=h)
        tot_t += dt
        tot_f += f
        heads += 1
        if tot_t >= budget_s:
            break
    return {"value": round(tot_f / tot_t / 1e12, 6), "unit": "TFLOP/s", **host_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle, {'fwd+bwd' if inp.do is not None else 'fwd'} of {heads} whole head(s) of "
                      f"sequence 0 ({L} query rows x all visible keys each), {tot_t:.2f} s"}


def oracle_sample_dropout(inp, rows, p, head=0):
    """fp64 dropout oracle forward+backward on one head of the first `rows` tokens of sequence 0 (a
    sequence of that length).  Returns (seconds, flops by the GPU arm's convention)."""
    import oracle
    R = min(rows, inp.seqlens[0])
    sl = (slice(0, R), slice(head, head + 1))
    q, k, v = inp.q[sl], inp.k[sl], inp.v[sl]
    t0 = time.perf_counter()
    oracle.attention_forward_dropout(q, k, v, inp.scale, inp.causal, p, 0x5EED, 0, B=1, N=R)
    if inp.do is not None:
        oracle.attention_backward_dropout(q, k, v, inp.do[sl], inp.scale, inp.causal, p, 0x5EED, 0, B=1, N=R)
    dt = time.perf_counter() - t0
    pairs = R * (R + 1) / 2 if inp.causal else R * R
    return dt, 4.0 * inp.d * pairs * (3.5 if inp.do is not None else 1.0)


def dropout_sample_rows(inp, p, budget_s):
    """Largest power-of-two prefix (from 256) whose dropout oracle run stays within about budget_s."""
    R = 256
    dt, _ = oracle_sample_dropout(inp, R, p)
    while 2 * R <= inp.seqlens[0] and dt * 4 < budget_s:
        R *= 2
        dt, _ = oracle_sample_dropout(inp, R, p)
    return R


def cpu_baseline_dropout(inp, p, budget_s=15.0):
    R = dropout_sample_rows(inp, p, budget_s / 2)
    dt, f = oracle_sample_dropout(inp, R, p)
    return {"value": round(f / dt / 1e12, 6), "unit": "TFLOP/s", **host_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy dropout oracle (p = {p}), {'fwd+bwd' if inp.do is not None else 'fwd'} of one head "
                      f"of the first {R} tokens of sequence 0 as a sequence of that length, {dt:.2f} s"}


def run_reference_merge(args):
    """The oracle's merge of two normalised partials on a bounded sample of (token, head) rows per step."""
    import torch

    import oracle
    w = MERGE_WORKLOADS[args.workload]
    rows, d = 65536, w["d"]  # 1/8 of the workload's 524 288 rows per step
    g = torch.Generator().manual_seed(w["seed"])
    a_o, b_o = (torch.randn(rows, d, generator=g).double().numpy() for _ in range(2))
    a_l, b_l = (torch.randn(rows, generator=g).double().numpy() for _ in range(2))
    for _ in range(args.warmup):
        oracle.merge_attention_partials([(a_o, a_l), (b_o, b_l)])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.merge_attention_partials([(a_o, a_l), (b_o, b_l)])
        times.append(time.perf_counter() - t0)
    ms = 1e3 * float(np.mean(times))
    nbytes = rows * d * 10 + rows * 12  # the GPU arm's count for a running merge of as many rows
    value = nbytes / (ms * 1e-3) / 1e9
    return {
        "impl": "reference", "metric": "ring-merge kernels: algorithmic HBM GB/s", "value": round(value, 3),
        "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "sample_rows": rows, "d": d},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", **host_threads(), "kind": "oracle",
                         "sample": f"fp64 NumPy oracle merge of two normalised partials over {rows} rows per step"},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, rank):
    import workloads
    if args.workload in workloads.DECODE_WORKLOADS:
        return run_reference_decode(args)
    if args.workload in MERGE_WORKLOADS:
        return run_reference_merge(args)
    spec = workloads.WORKLOADS[args.workload]
    inp = workloads.make_workload(args.workload, backward=spec["backward"])
    metric = METRIC
    if inp.dtype == "e4m3":
        inp = real_inputs(inp)
        metric = METRIC + " (e4m3 inputs, forward)"
    if args.dropout > 0.0:
        return run_reference_dropout(args, inp)
    L = inp.seqlens[0]
    # size each step so the whole run stays within ~3 minutes
    dt0, _ = oracle_sample(inp, 128)
    per_step = 180.0 / max(1, args.steps + args.warmup)
    rows = 128
    while rows < L and dt0 * (2 * rows / 128) < per_step:
        rows *= 2
    rows = min(rows, L)
    for _ in range(args.warmup):
        oracle_sample(inp, rows)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, f = oracle_sample(inp, rows)
        times.append(dt)
        flops = f
    ms = 1e3 * float(np.mean(times))
    value = flops / (ms * 1e-3) / 1e12
    sample = (f"fp64 NumPy oracle {'fwd+bwd' if inp.do is not None else 'fwd'} of query rows [{L - rows}, {L}) of "
              f"one head of sequence 0 per step")
    return {
        "impl": "reference", "metric": metric, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "B": inp.B, "H": inp.H, "N": inp.N, "d": inp.d,
                   "causal": inp.causal, "sample_rows": rows},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", **host_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference_dropout(args, inp):
    p = float(args.dropout)
    R = dropout_sample_rows(inp, p, 180.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample_dropout(inp, R, p)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, flops = oracle_sample_dropout(inp, R, p)
        times.append(dt)
    ms = 1e3 * float(np.mean(times))
    value = flops / (ms * 1e-3) / 1e12
    sample = (f"fp64 NumPy dropout oracle (p = {p}) {'fwd+bwd' if inp.do is not None else 'fwd'} of one head of the "
              f"first {R} tokens of sequence 0 per step")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "B": inp.B, "H": inp.H, "N": inp.N, "d": inp.d,
                   "causal": inp.causal, "dropout_p": p, "sample_tokens": R},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", **host_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# The five workloads the headline metric is quoted on (the default workload is the headline itself); each
# is measured by the same step as the headline, with fewer steps, and summarised in the `configs` object.
CONFIG_WORKLOADS = ["tiny_d64", "mha_n4k_d64", "causal_n8k_d128", "varlen_causal_d128", "long_n128k_d128"]


def config_summary(r):
    """Compact per-workload entry: step time, TFLOP/s and fraction of the measured peak, per kernel."""
    peaks = load_peaks()
    e = {"workload": r["config"]["workload"], "step": r["config"]["step"], "dtype": r["dtype"],
         "ms_per_step": r["ms_per_step"], "tflops": round(r["value"] / r["n_gpus"], 1),
         "frac_of_peak": round(r["value"] / r["n_gpus"] / peaks["bf16_tflops"], 4),
         "kernels": r.get("kernels"), "clocks": r.get("clocks")}
    if r["config"].get("dropout_p"):
        e["dropout_p"] = r["config"]["dropout_p"]
    if r["config"]["workload"] == "tiny_d64":
        e["us_per_step"] = round(1e3 * r["ms_per_step"], 1)  # launch-latency bound: no roofline claim
    return e


def run_configs(args, world, rank, local, pg, headline):
    """The other measured workloads (fp16 d = 64, varlen, 128k, the tiny call) and the dropout step,
    measured after the headline."""
    import copy
    out = {}
    for name in CONFIG_WORKLOADS + ["causal_n8k_d128+dropout0.1"]:
        if name == headline["config"]["workload"] and not headline["config"].get("dropout_p"):
            out[name] = config_summary(headline)
            continue
        a = copy.copy(args)
        a.workload, a.dropout = (name.split("+")[0], 0.1) if "+dropout" in name else (name, 0.0)
        a.steps = min(args.steps, 5)
        a.no_cpu_baseline = True
        try:
            out[name] = config_summary(run_gpu(a, world, rank, local, pg))
        except Exception as exc:  # a failed extra config must not lose the headline line
            out[name] = {"workload": name, "error": f"{type(exc).__name__}: {exc}"}
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        for name, e in out.items():
            if "error" not in e and name != headline["config"]["workload"]:
                e["cpu_baseline"] = config_cpu_baseline(name)
    return out


def config_cpu_baseline(name, budget_s=4.0):
    """The oracle on a short sample of one extra workload (the headline has its own cpu_baseline): the
    last `rows` query rows of head 0 of sequence 0 (the rows with the most visible keys), `rows` doubled
    from 64 until the run takes about a quarter of `budget_s`, then timed once."""
    import workloads
    wl, p = (name.split("+")[0], 0.1) if "+dropout" in name else (name, 0.0)
    inp = workloads.make_workload(wl)
    L = inp.seqlens[0]
    if p > 0.0:
        R = dropout_sample_rows(inp, p, budget_s / 2)
        dt, f = oracle_sample_dropout(inp, R, p)
        sample = f"fp64 NumPy dropout oracle (p = {p}), one head of the first {R} tokens of sequence 0"
    else:
        rows = min(64, L)
        dt, f = oracle_sample(inp, rows)
        while rows < L and dt * 4 < budget_s:
            rows = min(2 * rows, L)
            dt, f = oracle_sample(inp, rows)
        reps = max(1, int(0.25 * budget_s / max(dt, 1e-6)))  # a tiny sample is repeated to a measurable time
        if reps > 1:
            dt = sum(oracle_sample(inp, rows)[0] for _ in range(reps)) / reps
        sample = (f"fp64 NumPy oracle, {'fwd+bwd' if inp.do is not None else 'fwd'} of the last {rows} query rows "
                  f"of head 0 of sequence 0 ({L} tokens), {dt:.4f} s per run, {reps} run(s)")
    return {"value": round(f / dt / 1e12, 6), "unit": "TFLOP/s", **host_threads(), "kind": "oracle",
            "sample": sample}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="dropout probability on P (attention workloads; 0 = the plain step)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' summary (the `configs` object of the default line)")
    args = ap.parse_args()
    if not (0.0 <= args.dropout < 1.0):
        ap.error("--dropout must be in [0, 1)")
    if args.dropout > 0.0:
        import workloads
        spec = workloads.WORKLOADS.get(args.workload)
        if spec is None or spec["dtype"] == "e4m3":
            ap.error("--dropout applies to the 16-bit attention workloads only (not decode or e4m3)")
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    args.steps = max(1, args.steps)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank)), flush=True)
        return 0
    world, rank, local, pg = dist_setup(args)
    try:
        import workloads
        if args.workload in workloads.DECODE_WORKLOADS:
            out = run_gpu_decode(args, world, rank, local, pg)
        elif args.workload in MERGE_WORKLOADS:
            out = run_gpu_merge(args, world, rank, local, pg)
        elif workloads.WORKLOADS[args.workload]["dtype"] == "e4m3":
            out = run_gpu_fp8(args, world, rank, local, pg)
        else:
            out = run_gpu(args, world, rank, local, pg)
            if args.workload == DEFAULT_WORKLOAD and args.dropout == 0.0 and not args.no_configs:
                out["configs"] = run_configs(args, world, rank, local, pg, out)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if pg is not None:
            pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
