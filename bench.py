#!/usr/bin/env python
"""KDA prefill throughput on B200 through the library's C ABI.

Default workload: bf16 q/k/v, fp32 g/beta/state, B=2, H=8, T=4096,
d_k = d_v = 128, nonzero initial state (seeded synthetic inputs).  A step is one
full prefill (both kernels of the tensor-core path: the intra-chunk transform and
the state pass) over one batch.  With --gpus N > 1 (launched by torchrun) every
rank runs its own independent batch (weak scaling, no collective on the data
path); the reported time is the max over ranks.

Prints ONE JSON line (rank 0).  --impl reference times the fp64 CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s at d=128; achieved TFLOP/s and HBM GB/s vs B200 peak"
L2_FLUSH_BYTES = 256 << 20          # > 126 MB L2
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled from a thread)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, torch_dev, period=0.005):
        self.samples = []
        self.period = period
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            props = __import__("torch").cuda.get_device_properties(torch_dev)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:  # noqa: BLE001
                self.h = pynvml.nvmlDeviceGetHandleByIndex(torch_dev.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        inside = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples
        reasons = set()
        for _, _, rs in inside:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside)}


# ---------------------------------------------------------------------------
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x, world, device):
    """The maximum of a per-rank float over all ranks (the job's time is its slowest
    rank's); a no-op for one rank."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def workload_inputs(name, device, seed_offset=0):
    from kimi_delta_attention_28_b200 import workloads as W
    w = {"prefill": W.PREFILL, "long": W.LONG, "varlen": W.VARLEN,
         "few_chains": W.FEW_CHAINS}[name]
    import dataclasses
    w = dataclasses.replace(w, seed=w.seed + seed_offset)
    return w, W.make_workload(w, device)


def record_bytes():
    """Bytes of one (64-token chunk, head) record of the tensor-core path (its
    affine map on the state, as documented in include/kda.h)."""
    return 98816


def algorithmic(w, inp):
    """Units and algorithmic byte / flop counts of one prefill step."""
    ntok = inp["q"].shape[0] * inp["q"].shape[1]          # tokens (each with H heads)
    units = ntok * w.H                                       # token-heads
    nseq = inp["h0"].shape[0] if inp["h0"] is not None else inp["q"].shape[0]
    chains = nseq * w.H
    state_bytes = w.dk * w.dv * 4
    io = 2 if w.dtype.itemsize == 2 else 4
    per_unit_in = 3 * w.dk * io + w.dk * 4 + 4               # q, k, v, g, beta
    per_unit_out = w.dv * io                                 # o
    compulsory = units * (per_unit_in + per_unit_out) + chains * state_bytes * (
        2 if inp["h0"] is not None else 1)
    rec_per_unit = record_bytes() / 64                       # intra-chunk record bytes per token-head
    intra_bytes = units * (per_unit_in + rec_per_unit)
    inter_bytes = units * (rec_per_unit + per_unit_out) + chains * state_bytes * (
        2 if inp["h0"] is not None else 1)
    flops_recurrence = units * 7 * w.dk * w.dv
    return dict(ntok=ntok, units=units, chains=chains, compulsory=compulsory,
                intra_bytes=intra_bytes, inter_bytes=inter_bytes, flops=flops_recurrence)


def run_ours(args, world, rank, local):
    import torch
    import kimi_delta_attention_28_b200 as kda
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.load_library()
    w, inp = workload_inputs(args.workload, dev, seed_offset=rank)
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    cu = inp["cu_seqlens"]
    nseq = 0 if cu is None else cu.numel() - 1
    N = B if cu is None else nseq
    ws = torch.empty(kda.workspace_size(B, T, H, dk, dv, nseq, w.dtype), dtype=torch.uint8,
                     device=dev)
    o = torch.empty(B, T, H, dv, dtype=w.dtype, device=dev)
    hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # --ckpt-every N: every step also stores the state after each N tokens of every
    # sequence (kda_fwd_checkpointed, prefix caching) into a preallocated buffer
    ck = None
    if args.ckpt_every > 0:
        ck = torch.empty(kda.checkpoint_count(T, args.ckpt_every, B, cu), H, dk, dv,
                         dtype=torch.float32, device=dev)

    def step():
        # one kda_fwd call: the prep kernel, then the state pass
        if ck is not None:
            kda.kda_fwd_checkpointed(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                     inp["h0"], cu, ckpt_every=args.ckpt_every, ckpts=ck, o=o,
                                     hT=hT, workspace=ws)
        else:
            kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], cu, o=o,
                        hT=hT, workspace=ws)

    def step_split(ev):
        # the two phases as separate calls, an event between them: per-kernel times
        ev[0].record(stream)
        kda.kda_fwd_intra(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], cu, workspace=ws)
        ev[1].record(stream)
        kda.kda_fwd_inter(inp["h0"], cu, o, hT, B=B, T=T, H=H, dk=dk, dv=dv, dtype=w.dtype,
                          workspace=ws)
        ev[2].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.02)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        ev = events[i]
        ev[0].record(stream)
        step()
        ev[2].record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    clocks.stop()
    total_ms = sum(e[0].elapsed_time(e[2]) for e in events)
    # per-kernel split, outside the timed region
    split = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
             for _ in range(min(args.steps, 20))]
    for ev in split:
        flush.zero_()
        step_split(ev)
    torch.cuda.synchronize(dev)
    intra = [e[0].elapsed_time(e[1]) for e in split]
    inter = [e[1].elapsed_time(e[2]) for e in split]
    nseg = kda.plan_segments(B, T, H, dk, dv, nseq, w.dtype)
    launches_per_step = (2 if cu is not None else 1) + (1 if nseg <= 1 else 3)
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    A = algorithmic(w, inp)

    # end to end: pinned host inputs -> device, kda_fwd through the C ABI, results -> host.
    # Every step copies its inputs in and its outputs (o, hT) out; consecutive steps
    # are pipelined on three streams with two buffer sets, so step i+1's inputs go
    # up while step i computes and step i-1's results come down.
    e2e = None
    if not args.no_e2e and ck is None:
        host = {k_: (v_.cpu().pin_memory() if v_ is not None else None) for k_, v_ in inp.items()}
        o_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hT_h = [torch.empty(hT.shape, dtype=hT.dtype).pin_memory() for _ in range(2)]
        dev_in = [{k_: (torch.empty_like(v_, device=dev) if v_ is not None else None)
                   for k_, v_ in host.items()} for _ in range(2)]
        o_d = [o, torch.empty_like(o)]
        hT_d = [hT, torch.empty_like(hT)]
        h2d = sum(v_.numel() * v_.element_size() for v_ in host.values() if v_ is not None)
        d2h = o_h[0].numel() * o_h[0].element_size() + hT_h[0].numel() * hT_h[0].element_size()
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_up = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_down = [torch.cuda.Event() for _ in range(2)]
        for b_ in range(2):   # all buffers free at the start
            ev_comp[b_].record(stream)
            ev_down[b_].record(stream)

        def e2e_step(i):
            b_ = i & 1
            with torch.cuda.stream(s_up):
                s_up.wait_event(ev_comp[b_])           # step i-2 has read these inputs
                for k_, v_ in host.items():
                    if v_ is not None:
                        dev_in[b_][k_].copy_(v_, non_blocking=True)
                ev_up[b_].record(s_up)
            stream.wait_event(ev_up[b_])
            stream.wait_event(ev_down[b_])            # step i-2's results are down
            d = dev_in[b_]
            kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], d["cu_seqlens"],
                        o=o_d[b_], hT=hT_d[b_], workspace=ws)
            ev_comp[b_].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_comp[b_])
                o_h[b_].copy_(o_d[b_], non_blocking=True)
                hT_h[b_].copy_(hT_d[b_], non_blocking=True)
                ev_down[b_].record(s_down)

        for i in range(max(3, args.warmup // 4)):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 50))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        e0.record(s_up)
        for i in range(n_e2e):
            e2e_step(i)
        for b_ in range(2):                           # everything down before the stop
            s_down.wait_event(ev_down[b_])
        e1.record(s_down)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
        e2e = {"value": world * A["ntok"] / (e2e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms,
               "note": "inputs up and outputs down every step; steps pipelined on 3 streams"}

    if rank != 0:
        return None
    hbm_peak, tf_peak, peak_src = load_peaks()
    intra_ms = statistics.mean(intra)
    inter_ms = statistics.mean(inter)
    dom = "intra" if intra_ms >= inter_ms else "inter"
    dom_ms = max(intra_ms, inter_ms)
    dom_bytes = A["intra_bytes"] if dom == "intra" else A["inter_bytes"]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    traffic = load_traffic(dom)
    path_gbs = A["compulsory"] / (ms_per_step * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": world * A["ntok"] / (ms_per_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype.itemsize == 2 else "f32",
        "data": "synthetic (seeded; q,k L2-normalised, g=-5*sigmoid(N(-3,1)), beta=sigmoid(N(0,1)))",
        "config": prefill_config(w, inp, world),
        "roofline": {"bound": "hbm", "kernel": "kda_tc_prep_kernel" if dom == "intra"
                     else "kda_tc_state_kernel", "achieved": achieved, "peak": hbm_peak,
                     "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                     "algorithmic_bytes_per_launch": dom_bytes},
        "path": {"compulsory_bytes_per_step": A["compulsory"], "hbm_gbs": path_gbs,
                 "hbm_frac": path_gbs / hbm_peak,
                 "tflops_recurrence": A["flops"] / (ms_per_step * 1e-3) / 1e12,
                 "tensor_frac": A["flops"] / (ms_per_step * 1e-3) / 1e12 / tf_peak},
        "kernels_ms": {"kda_tc_prep_kernel": intra_ms,
                       ("kda_tc_state_kernel" if nseg <= 1 else
                        f"state pass split in {nseg} segments (map, combine, output)"): inter_ms},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(t_wall0, t_wall1),
        "e2e": e2e,
    }
    if ck is not None:
        out["config"]["ckpt_every"] = args.ckpt_every
        out["config"]["checkpoints_per_head"] = int(ck.shape[0])
        out["kernels_ms_note"] = ("per-kernel split measured through kda_fwd_intra / "
                                  "kda_fwd_inter, which store no checkpoints")
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, inp, budget_s=args.cpu_seconds)
    return out


def run_ours_decode(args, world, rank, local):
    """Decode workload: 256 sequences x 96 heads x d=128, fp32 state updated in
    place; each step consumes fresh pre-generated inputs (the state, 1.6 GB, is
    larger than L2, so no flush is needed)."""
    import torch
    import kimi_delta_attention_28_b200 as kda
    from kimi_delta_attention_28_b200 import workloads as W
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.load_library()
    w = W.DECODE
    nsteps = args.warmup + args.steps
    inp = W.make_decode_inputs(w.B, w.H, w.dk, w.dv, nsteps, w.dtype, w.seed + rank, dev)
    S = inp["S"]
    o = torch.empty(w.B, w.H, w.dv, dtype=w.dtype, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(t):
        kda.kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t], inp["beta"][t],
                            S, o)

    for t in range(args.warmup):
        step(t)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.02)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.perf_counter()
    ev[0].record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    clocks.stop()
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = max_over_ranks(total_ms, world, dev)
    if rank != 0:
        return None
    ms = total_ms / args.steps
    units = w.B * w.H
    per_unit = 2 * w.dk * w.dv * 4 + 3 * w.dk * 2 + w.dk * 4 + 4 + w.dv * 2
    bytes_step = units * per_unit
    hbm_peak, _, peak_src = load_peaks()
    gbs = bytes_step / (ms * 1e-3) / 1e9
    return {
        "metric": "KDA decode steps/s (256 sequences x 96 heads, d=128, fp32 state in place)",
        "value": world * 1e3 / ms, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "N": w.B, "H": w.H, "dk": w.dk, "dv": w.dv,
                   "l2": "state (1.6 GB) larger than L2; no flush"},
        "roofline": {"bound": "hbm", "kernel": "kda_decode_kernel", "achieved": gbs,
                     "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                     "traffic": load_traffic("decode"),
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                     "algorithmic_bytes_per_launch": bytes_step},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(t_wall0, t_wall1),
    }


def _strip_comments(text):
    """C/C++ source without comments and blank lines (string literals are kept)."""
    import re
    pat = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)
    text = pat.sub(lambda m: m.group(0) if m.group(0).startswith('"') else "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def kernel_source_sha(src=None):
    """sha256 over the CUDA sources of the library with comments removed (identifies
    the kernel code; an edit of comments alone keeps it)."""
    import hashlib
    src = src or os.path.join(ROOT, "kimi_delta_attention_28_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(src)):
        if f.endswith((".cu", ".cuh")):
            with open(os.path.join(src, f), encoding="utf-8") as fh:
                h.update(f.encode() + b"\0" + _strip_comments(fh.read()).encode())
    return h.hexdigest()


def load_traffic(which):
    """DRAM bytes (read + write) per launch of kernel `which`, from the committed
    ncu summary profiles/traffic.json -- only if it was taken on the current
    kernel sources (same sha256), else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("kernel_source_sha256") != kernel_source_sha():
            return None
        return d["per_launch_dram_bytes"].get(which)
    except Exception:  # noqa: BLE001
        return None


def host_f64(inp):
    import numpy as np
    out = {}
    for k_, v_ in inp.items():
        if v_ is None:
            out[k_] = None
        elif k_ == "cu_seqlens":
            out[k_] = v_.cpu().numpy().astype(np.int64)
        else:
            out[k_] = np.ascontiguousarray(v_.detach().cpu().double().numpy())
    return out


def cpu_baseline(w, inp, budget_s=10.0, chains_per_step=None):
    """Time the fp64 oracle (as it stands) on the host cores on whole chains of
    this workload: tokens/s in the same unit as the GPU number."""
    import oracle
    h = host_f64(inp)
    B, T, H, dk = h["q"].shape
    q, k, v, g, beta = (h[n].reshape(B * T, H, -1) if n != "beta" else h[n].reshape(B * T, H)
                        for n in ("q", "k", "v", "g", "beta"))
    cu = h["cu_seqlens"] if h["cu_seqlens"] is not None else (
        __import__("numpy").arange(B + 1) * T)
    reps, elapsed, used = 0, 0.0, 1
    while elapsed < budget_s and reps < 50:
        t0 = time.perf_counter()
        _, _, used = oracle.kda_fwd_packed(q, k, v, g, beta, h["h0"], cu)
        elapsed += time.perf_counter() - t0
        reps += 1
    ntok = B * T
    return {"value": ntok * reps / elapsed, "unit": "tokens/s", "cores": int(used),
            "kind": "oracle",
            "sample": f"whole workload ({B}x{T} tokens x {H} heads) x {reps} runs, "
                      f"{elapsed:.1f} s; fp64 token-by-token C, OpenMP over (sequence, head)"}


def prefill_config(w, inp, world):
    """The `config` object of a prefill workload (shared by both arms)."""
    B, T, H, dk = inp["q"].shape
    nseq = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    return {"workload": w.name, "B": B, "T": T, "H": H, "dk": dk, "dv": inp["v"].shape[-1],
            "h0": "N(0, 0.1^2)" if inp["h0"] is not None else "zeros",
            "varlen_seqs": nseq, "l2": "flushed between steps (256 MiB write)",
            "parallelism": f"replicas x{world} (independent batches)"}


def run_reference(args, world, rank):
    """The oracle on a bounded sample of the workload, timed per step."""
    import numpy as np
    import torch
    import oracle
    from kimi_delta_attention_28_b200 import workloads as W
    w = {"prefill": W.PREFILL, "long": W.LONG, "varlen": W.VARLEN,
         "few_chains": W.FEW_CHAINS}[args.workload]
    inp = W.make_workload(w, "cpu")
    h = host_f64(inp)
    B, T, H, dk = h["q"].shape
    dv = h["v"].shape[-1]
    # sample: whole (sequence, head) chains over the first Ts tokens of sequence 0,
    # sized so warmup + steps finish in about args.ref_seconds
    Ts = min(T, 4096)
    one = lambda n: np.ascontiguousarray(h[n][0, :Ts, :1])  # noqa: E731
    t0 = time.perf_counter()
    oracle.kda_fwd_packed(one("q"), one("k"), one("v"), one("g"), one("beta"), None,
                          np.array([0, Ts]))
    t_chain = max(time.perf_counter() - t0, 1e-4)
    nthreads = oracle.threads_available()
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    chains = int(max(1, min(H, per_step / t_chain * min(nthreads, H) * 0.8)))
    if t_chain > per_step:
        Ts = max(64, int(Ts * per_step / t_chain))
    sl = lambda n: np.ascontiguousarray(h[n][0, :Ts, :chains])  # noqa: E731
    args_ = (sl("q"), sl("k"), sl("v"), sl("g"), sl("beta"),
             None if h["h0"] is None else np.ascontiguousarray(h["h0"][:1, :chains]),
             np.array([0, Ts]))
    for _ in range(args.warmup):
        oracle.kda_fwd_packed(*args_)
    times, used = [], 1
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _, _, used = oracle.kda_fwd_packed(*args_)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    tokens = Ts * chains / H          # tokens-with-H-heads equivalent of the sample
    value = tokens / (ms * 1e-3)
    sample = (f"{chains} of {H} heads x {Ts} tokens of sequence 0 per step "
              f"(fp64 token-by-token C oracle)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded), same generator as the GPU arm",
            "config": prefill_config(w, inp, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": int(used),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 1000 for the bench workload, whose step is "
                         "~0.1 ms, so the timed region spans many clock samples; 300 otherwise)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "long", "varlen", "decode", "few_chains"],
                    default="prefill")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ckpt-every", type=int, default=0,
                    help="prefill workloads: also store the state every N tokens (multiple of 64)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 1000 if (args.impl == "ours" and args.workload == "prefill") else 300
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference" and args.workload == "decode":
        ap.error("the reference arm covers the prefill workloads")
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    try:
        if args.workload == "decode":
            out = run_ours_decode(args, world, rank, local)
        else:
            out = run_ours(args, world, rank, local)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
