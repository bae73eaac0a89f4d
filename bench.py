#!/usr/bin/env python
"""KDA prefill throughput on B200 through the library's C ABI.

Default (headline) workload: the 1M-token prefill -- bf16 q/k/v, fp32 g/beta/state,
B=1, H=16, T=1,048,576, d_k = d_v = 128, zero initial state, seeded synthetic
inputs (about 26 GB of inputs and outputs, far larger than L2).  A step is one
full ``kda_fwd`` call over the whole batch: for this shape one overlapped launch in
which the state pass consumes the intra-chunk records as they are written
(``--two-launch`` times the intra-chunk kernel, then the state pass, instead).  On one GPU the same JSON line also carries, under ``workloads``, the other
measured workloads with their own roofline and sampled parity: the B=2, H=8,
T=4,096 prefill, the packed varlen prefill (16 sequences, H=32) and the decode
step (256 sequences x 96 heads, fp32 state in place).

With --gpus N > 1 (launched by torchrun) every rank runs its own independent batch
of the headline workload (weak scaling, no collective on the data path); the
reported time is the max over ranks.

Prints ONE JSON line (rank 0).  --impl reference times the fp64 CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import datetime
import gc
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
L2_BYTES = 126 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
HEADLINE = "long"
WORKLOAD_KEYS = ("prefill", "long", "varlen", "few_chains", "decode", "profile", "speculative",
                 "backward")


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


def workload_of(name):
    from kimi_delta_attention_28_b200 import workloads as W
    return {"prefill": W.PREFILL, "long": W.LONG, "varlen": W.VARLEN,
            "few_chains": W.FEW_CHAINS, "decode": W.DECODE, "profile": W.PROFILE}[name]


def workload_inputs(name, device, seed_offset=0):
    from kimi_delta_attention_28_b200 import workloads as W
    import dataclasses
    w = dataclasses.replace(workload_of(name), seed=workload_of(name).seed + seed_offset)
    return w, W.make_workload(w, device)


def record_bytes():
    """Bytes of one (64-token chunk, head) record of the tensor-core path (its
    affine map on the state, as documented in include/kda.h)."""
    return 98816


def algorithmic(w, inp):
    """Units and the compulsory byte / flop counts of one prefill step.

    Compulsory bytes are the method's own traffic: per token-head q, k, v
    (3 d_k elements), g (fp32 d_k), beta (fp32) in and o out -- 1,540 B at
    d = 128 in bf16 -- plus each (sequence, head) state read once (if given)
    and written once.  The records the tensor-core path writes and reads back
    are this implementation's intermediate and are reported separately."""
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    ntok = B * T                                             # tokens (each with H heads)
    units = ntok * H                                         # token-heads
    nseq = inp["cu_seqlens"].numel() - 1 if inp["cu_seqlens"] is not None else B
    chains = nseq * H
    state_bytes = dk * dv * 4
    io = inp["q"].element_size()
    per_unit_in = 3 * dk * io + dk * 4 + 4                   # q, k, v, g, beta
    per_unit_out = dv * io                                   # o
    states = chains * state_bytes * (2 if inp["h0"] is not None else 1)
    compulsory = units * (per_unit_in + per_unit_out) + states
    rec_per_unit = record_bytes() / 64                       # records per token-head
    flops_recurrence = units * 7 * dk * dv
    return dict(ntok=ntok, units=units, chains=chains, compulsory=compulsory,
                per_unit_compulsory=per_unit_in + per_unit_out,
                prep_compulsory=units * per_unit_in,
                state_compulsory=units * per_unit_out + states,
                intermediate=2 * units * rec_per_unit, flops=flops_recurrence)


# ---------------------------------------------------------------------------
# committed DRAM traffic (ncu) per unit, valid only for the kernel sources it was taken on
# ---------------------------------------------------------------------------
def _strip_comments(text):
    """C/C++ source without comments and blank lines (string literals are kept)."""
    import re
    pat = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)
    text = pat.sub(lambda m: m.group(0) if m.group(0).startswith('"') else "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


# The device-code headers each kernel is compiled from (its own and the shared one).
KERNEL_SOURCES = {
    "kda_tc_fused_kernel": ("kda_prefill_tc.cuh", "kda_common.cuh"),
    "kda_tc_prep_kernel": ("kda_prefill_tc.cuh", "kda_common.cuh"),
    "kda_tc_state_kernel": ("kda_prefill_tc.cuh", "kda_common.cuh"),
    "kda_decode_kernel": ("kda_decode.cuh", "kda_common.cuh"),
    "kda_decode_multi_kernel": ("kda_decode.cuh", "kda_common.cuh"),
    "kda_bwd_slice_kernel": ("kda_bwd.cuh", "kda_common.cuh"),
}


def kernel_source_sha(kernel=None, src=None):
    """sha256 over the device-code headers `kernel` is compiled from (all of csrc/*.cuh
    when kernel is None or unknown) with comments removed: it identifies that kernel's
    code.  An edit of comments alone, of the host-side launch and policy code
    (csrc/*.cu), or of another kernel's header keeps it."""
    import hashlib
    src = src or os.path.join(ROOT, "kimi_delta_attention_28_b200", "csrc")
    files = KERNEL_SOURCES.get(kernel)
    h = hashlib.sha256()
    for f in sorted(os.listdir(src)):
        if f.endswith(".cuh") and (files is None or f in files):
            with open(os.path.join(src, f), encoding="utf-8") as fh:
                h.update(f.encode() + b"\0" + _strip_comments(fh.read()).encode())
    return h.hexdigest()


def load_traffic(kernel, units):
    """DRAM bytes (read + write) of `kernel` for `units` units (token-heads for the
    prefill kernels, (sequence, head) chains for decode): the per-unit figure of the
    committed ncu summary profiles/traffic.json scaled by the units -- only if that
    figure was taken on the kernel's current code (same sha256 of its headers), else
    None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("source_sha256", {}).get(kernel) != kernel_source_sha(kernel):
            return None
        per = d["dram_bytes_per_unit"].get(kernel)
        return None if per is None else float(per) * units
    except Exception:  # noqa: BLE001
        return None


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------
def prefill_config(w, inp, world):
    """The `config` object of a prefill workload (shared by both arms)."""
    B, T, H, dk = inp["q"].shape
    nseq = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    big = _input_bytes(inp) > 4 * L2_BYTES
    return {"workload": w.name, "B": B, "T": T, "H": H, "dk": dk, "dv": inp["v"].shape[-1],
            "h0": "N(0, 0.1^2)" if inp["h0"] is not None else "zeros",
            "varlen_seqs": nseq,
            "l2": ("inputs (%.1f GB) far larger than L2; no flush" % (_input_bytes(inp) / 1e9))
            if big else "flushed between steps (256 MiB write)",
            "parallelism": f"replicas x{world} (independent batches)"}


def _input_bytes(inp):
    return sum(v.numel() * v.element_size() for v in inp.values() if v is not None)


def measure_prefill(name, steps, warmup, world=1, rank=0, local=0, e2e=True, cpu=True,
                    cpu_seconds=10.0, ckpt_every=0, two_launch=False):
    """Time `steps` kda_fwd calls on workload `name`; returns the JSON object (rank 0).
    two_launch: time kda_fwd_segmented with one segment instead (the prep kernel, then
    the state pass) whatever schedule kda_fwd would pick."""
    import torch
    import kimi_delta_attention_28_b200 as kda
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.load_library()
    w, inp = workload_inputs(name, dev, seed_offset=rank)
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    cu = inp["cu_seqlens"]
    nseq = 0 if cu is None else cu.numel() - 1
    N = B if cu is None else nseq
    ws = torch.empty(kda.workspace_size(B, T, H, dk, dv, nseq, w.dtype), dtype=torch.uint8,
                     device=dev)
    o = torch.empty(B, T, H, dv, dtype=w.dtype, device=dev)
    hT = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    big = _input_bytes(inp) > 4 * L2_BYTES
    flush = None if big else torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # ckpt_every > 0: every step also stores the state after each ckpt_every tokens
    # of every sequence (kda_fwd_checkpointed, prefix caching)
    ck = None
    if ckpt_every > 0:
        ck = torch.empty(kda.checkpoint_count(T, ckpt_every, B, cu), H, dk, dv,
                         dtype=torch.float32, device=dev)

    def step():
        if ck is not None:
            kda.kda_fwd_checkpointed(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                     inp["h0"], cu, ckpt_every=ckpt_every, ckpts=ck, o=o,
                                     hT=hT, workspace=ws)
        elif two_launch:
            kda.kda_fwd_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                  inp["h0"], cu, num_segments=1, o=o, hT=hT, workspace=ws)
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

    def flush_l2():
        if flush is not None:
            flush.zero_()

    for _ in range(warmup):
        flush_l2()
        step()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.02)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.perf_counter()
    for i in range(steps):
        flush_l2()
        events[i][0].record(stream)
        step()
        events[i][1].record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    clocks.stop()
    total_ms = sum(e[0].elapsed_time(e[1]) for e in events)
    # per-kernel split, outside the timed region
    nsplit = min(steps, 20 if not big else 5)
    split = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nsplit)]
    for ev in split:
        flush_l2()
        step_split(ev)
    torch.cuda.synchronize(dev)
    intra_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in split)
    inter_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in split)
    nseg = kda.plan_segments(B, T, H, dk, dv, nseq, w.dtype)
    # kda_fwd's schedule: one overlapped launch, or the prep kernel then the state pass
    overlap = kda.plan_overlap(B, T, H, dk, dv, nseq, w.dtype) and not two_launch
    if two_launch:
        nseg = 1
    launches_per_step = 1 if overlap else (2 if cu is not None else 1) + (1 if nseg <= 1 else 3)
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / steps
    A = algorithmic(w, inp)
    # the outputs of the timed steps, for the parity sample of the CPU leg
    o_host = o.cpu() if rank == 0 and cpu and world == 1 else None
    hT_host = hT.cpu() if o_host is not None else None

    e2e_obj = None
    if e2e and ck is None:
        e2e_obj = measure_e2e(kda, w, inp, o, hT, ws, dev, stream, world, A["ntok"],
                              n_steps=3 if big else max(3, min(steps, 50)))
    if rank != 0:
        return None

    hbm_peak, tf_peak, peak_src = load_peaks()
    call_gbs = A["compulsory"] / (ms_per_step * 1e-3) / 1e9
    t_prep = load_traffic("kda_tc_prep_kernel", A["units"])
    t_state = load_traffic("kda_tc_state_kernel", A["units"]) if nseg <= 1 else None
    traffic = (t_prep + t_state) if (t_prep is not None and t_state is not None) else None
    state_name = ("kda_tc_state_kernel" if nseg <= 1 else
                  f"state pass split in {nseg} segments (map, combine, output)")
    call_name = "kda_fwd call (kda_tc_prep_kernel + %s)" % state_name
    if overlap:
        traffic = load_traffic("kda_tc_fused_kernel", A["units"])
        call_name = ("kda_fwd call: kda_tc_fused_kernel (records and state pass overlapped "
                     "in one launch)")
    out = {
        "metric": METRIC,
        "value": world * A["ntok"] / (ms_per_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype.itemsize == 2 else "f32",
        "data": "synthetic (seeded; q,k L2-normalised, g=-5*sigmoid(N(-3,1)), beta=sigmoid(N(0,1)))",
        "config": prefill_config(w, inp, world),
        # the whole kda_fwd call (its two kernels run back to back on one stream) against
        # the method's compulsory bytes: 1,540 B per token-head plus the states
        "roofline": {
            "bound": "hbm",
            "kernel": call_name,
            "achieved": call_gbs, "peak": hbm_peak, "unit": "GB/s",
            "frac": call_gbs / hbm_peak,
            "traffic": traffic,
            "algorithmic_bytes_per_launch": A["compulsory"],
            "algorithmic_bytes_rule": "compulsory: %d B per token-head (q,k,v,g,beta in; o out) "
                                      "x %d token-heads + states %d B" % (
                                          A["per_unit_compulsory"], A["units"],
                                          A["compulsory"] - A["units"] * A["per_unit_compulsory"]),
            "intermediate_bytes": A["intermediate"],
            "intermediate_rule": "records (%d B per 64-token chunk and head) written by the "
                                 "prep kernel and read back by the state pass" % record_bytes(),
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
            # the two-launch schedule of the same call, timed through kda_fwd_intra /
            # kda_fwd_inter outside the timed region (with the overlapped schedule it is
            # a comparison, not a part of the step)
            "per_kernel" if not overlap else "two_launch_schedule": {
                "kda_tc_prep_kernel": {
                    "ms": intra_ms,
                    "compulsory_bytes": A["prep_compulsory"],
                    "frac": A["prep_compulsory"] / (intra_ms * 1e-3) / 1e9 / hbm_peak,
                    "dram_bytes": t_prep},
                state_name: {
                    "ms": inter_ms,
                    "compulsory_bytes": A["state_compulsory"],
                    "frac": A["state_compulsory"] / (inter_ms * 1e-3) / 1e9 / hbm_peak,
                    "dram_bytes": t_state},
                "dominant": "kda_tc_prep_kernel" if intra_ms >= inter_ms else state_name,
                "dominant_frac_all_compulsory_over_its_time":
                    A["compulsory"] / (max(intra_ms, inter_ms) * 1e-3) / 1e9 / hbm_peak,
            },
        },
        "path": {"compulsory_bytes_per_step": A["compulsory"], "hbm_gbs": call_gbs,
                 "hbm_frac": call_gbs / hbm_peak,
                 "tflops_recurrence": A["flops"] / (ms_per_step * 1e-3) / 1e12,
                 "tensor_frac": A["flops"] / (ms_per_step * 1e-3) / 1e12 / tf_peak},
        "kernels_ms": ({"kda_tc_fused_kernel": ms_per_step} if overlap else
                       {"kda_tc_prep_kernel": intra_ms, state_name: inter_ms}),
        "gpu_launches": launches_per_step * steps,
        "clocks": clocks.summary(t_wall0, t_wall1),
        "e2e": e2e_obj,
    }
    out["config"]["schedule"] = ("one overlapped launch (kda_tc_fused_kernel)" if overlap else
                                 "two launches (prep kernel, then state pass)" +
                                 (" (forced)" if two_launch else ""))
    if ck is not None:
        out["config"]["ckpt_every"] = ckpt_every
        out["config"]["checkpoints_per_head"] = int(ck.shape[0])
        out["kernels_ms_note"] = ("per-kernel split measured through kda_fwd_intra / "
                                  "kda_fwd_inter, which store no checkpoints")
    if o_host is not None:
        del o, hT, ws
        out["cpu_baseline"] = cpu_baseline(w, inp, o_host, hT_host, budget_s=cpu_seconds)
    return out


def measure_e2e(kda, w, inp, o, hT, ws, dev, stream, world, ntok, n_steps):
    """End to end through the C ABI with host buffers: every step copies its inputs up
    from pinned host memory, runs kda_fwd and copies o and hT down.  Consecutive steps
    are pipelined on three streams with two device buffer sets (step i+1's inputs go
    up while step i computes and step i-1's results come down)."""
    import torch
    host = {k_: (torch.empty(v_.shape, dtype=v_.dtype, pin_memory=True).copy_(v_)
                 if v_ is not None else None) for k_, v_ in inp.items()}
    o_h = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
    hT_h = [torch.empty(hT.shape, dtype=hT.dtype, pin_memory=True) for _ in range(2)]
    dev_in = [inp, {k_: (torch.empty_like(v_) if v_ is not None else None)
                    for k_, v_ in inp.items()}]
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

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0.record(s_up)
    for i in range(n_steps):
        e2e_step(i)
    for b_ in range(2):                           # everything down before the stop
        s_down.wait_event(ev_down[b_])
    e1.record(s_down)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / n_steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    del dev_in[1], o_d[1], hT_d[1]
    return {"value": world * ntok / (e2e_ms * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": e2e_ms, "steps": n_steps,
            "note": "inputs up from pinned host memory and o, hT down every step; steps "
                    "pipelined on 3 streams with 2 device buffer sets"}


def workload_shapes(w):
    """The prefill inputs of workload `w` as meta tensors: shapes and dtypes, no data."""
    import torch
    from kimi_delta_attention_28_b200 import workloads as W
    meta = torch.device("meta")
    if w.varlen_seqs:
        lengths = W.varlen_lengths(w.varlen_seqs, *w.varlen_range, seed=w.seed)
        B, T, N = 1, int(sum(lengths)), len(lengths)
    else:
        B, T, N = w.B, w.T, w.B
    mk = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device=meta)  # noqa: E731
    return {"q": mk(B, T, w.H, w.dk, dt=w.dtype), "k": mk(B, T, w.H, w.dk, dt=w.dtype),
            "v": mk(B, T, w.H, w.dv, dt=w.dtype), "g": mk(B, T, w.H, w.dk),
            "beta": mk(B, T, w.H), "h0": mk(N, w.H, w.dk, w.dv) if w.h0 else None,
            "cu_seqlens": mk(N + 1, dt=torch.int32) if w.varlen_seqs else None}


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


def _err(got, ref):
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return {"rel_l2": float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)),
            "max_abs": float(np.abs(got - ref).max()) if got.size else 0.0}


PARITY_TOL = {"bf16": "rel-L2 <= 1e-2 and max-abs <= 5e-2", "f32": "rel-L2 <= 1e-4"}


def cpu_baseline(w, inp, o_gpu, hT_gpu, budget_s=10.0):
    """The fp64 oracle (as it stands) on the host cores, on whole (sequence, head) chains
    of this workload from their true initial states: tokens/s in the GPU number's unit
    (tokens that carry all H heads).  The oracle's outputs for the sample are also
    compared with the GPU's outputs of the timed steps (o_gpu, hT_gpu, on the host)."""
    import numpy as np
    import oracle
    h = {k_: v_ for k_, v_ in inp.items()}
    B, T, H, dk = h["q"].shape
    cu = h["cu_seqlens"]
    # only the sampled slices of o are converted (the whole o in fp64 is 17 GB at T = 1M)
    o_at = lambda *ix: o_gpu[ix].double().numpy()  # noqa: E731
    hT_g = hT_gpu.double().numpy()
    parity = {"tolerance": PARITY_TOL["bf16" if w.dtype.itemsize == 2 else "f32"]}
    if cu is not None:
        # packed: one head (0) of every sequence, whole sequences
        hh = 0
        sl = lambda x: np.ascontiguousarray(x[0, :, hh:hh + 1].detach().cpu().double().numpy())  # noqa: E731
        args_ = (sl(h["q"]), sl(h["k"]), sl(h["v"]), sl(h["g"]),
                 np.ascontiguousarray(h["beta"][0, :, hh:hh + 1].cpu().double().numpy()),
                 None if h["h0"] is None else
                 np.ascontiguousarray(h["h0"][:, hh:hh + 1].cpu().double().numpy()),
                 cu.cpu().numpy().astype(np.int64))
        t0 = time.perf_counter()
        o_ref, hT_ref, used = oracle.kda_fwd_packed(*args_)
        el = time.perf_counter() - t0
        ntok_equiv = T / H
        parity["o"] = _err(o_at(0, slice(None), slice(hh, hh + 1)), o_ref)
        parity["hT"] = _err(hT_g[:, hh:hh + 1], hT_ref)
        parity["sample"] = f"head {hh} of all {cu.numel() - 1} packed sequences, whole"
        sample = (f"head {hh} of all {cu.numel() - 1} packed sequences ({T} tokens), "
                  f"{el:.1f} s; fp64 token-by-token C, OpenMP over sequences")
        return {"value": ntok_equiv / el, "unit": "tokens/s", "cores": int(used),
                "kind": "oracle", "sample": sample, "parity": parity}
    # fixed length: all heads of sequence 0 over its first Ts tokens (exact: the chains
    # start from h0 at token 0), Ts sized to about budget_s of oracle time
    Ts = min(T, 1024)
    while True:
        sl = lambda x, n=Ts: np.ascontiguousarray(x[0, :n].detach().cpu().double().numpy())  # noqa: E731
        h0 = None if h["h0"] is None else np.ascontiguousarray(h["h0"][:1].cpu().double().numpy())
        t0 = time.perf_counter()
        o_ref, hT_ref, used = oracle.kda_fwd_packed(sl(h["q"]), sl(h["k"]), sl(h["v"]),
                                                    sl(h["g"]), sl(h["beta"]), h0,
                                                    np.array([0, Ts]))
        el = time.perf_counter() - t0
        if Ts >= T or el * 3 > budget_s:
            break
        Ts = min(T, int(Ts * min(8.0, max(2.0, budget_s / max(el, 1e-3) / 2))))
    parity["o"] = _err(o_at(0, slice(0, Ts)), o_ref)
    parity["sample"] = f"all {H} heads of sequence 0, tokens [0, {Ts})"
    if Ts >= T:
        parity["hT"] = _err(hT_g[:1], hT_ref)
    else:
        # the final block and final state by a window restarted from zero L tokens
        # earlier: every transition has operator norm <= max_c exp(g_tc), so the
        # truncation error is at most exp(sum of per-token max g) times the state norm
        L, blk = 4096, 64
        a, s = T - blk - L, T - blk
        gmax = inp["g"][0, a:s].amax(dim=-1).double().sum(dim=0).max().item()
        snorm = T * float(inp["v"].abs().max()) * math.sqrt(w.dv)
        slw = lambda x: np.ascontiguousarray(x[0, a:T].detach().cpu().double().numpy())  # noqa: E731
        ow, hw, _ = oracle.kda_fwd_packed(slw(inp["q"]), slw(inp["k"]), slw(inp["v"]),
                                          slw(inp["g"]), slw(inp["beta"]), None,
                                          np.array([0, T - a]))
        parity["o_last_block"] = _err(o_at(0, slice(s, T)), ow[L:])
        if h["h0"] is None or B == 1:
            parity["hT"] = _err(hT_g[:1], hw)
        parity["window_truncation_bound"] = math.exp(gmax) * snorm
        parity["sample"] += (f"; tokens [{s}, {T}) and the final states by a {L}-token "
                             "window restarted from zero (truncation bound above)")
    sample = (f"all {H} heads of sequence 0 over tokens [0, {Ts}) from h0, {el:.1f} s; "
              "fp64 token-by-token C, OpenMP over heads")
    return {"value": Ts / el, "unit": "tokens/s", "cores": int(used), "kind": "oracle",
            "sample": sample, "parity": parity}


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------
def measure_decode(steps, warmup, world=1, rank=0, local=0, cpu=True):
    """Decode workload: 256 sequences x 96 heads x d=128, fp32 state updated in
    place; each step consumes fresh pre-generated inputs (the state, 1.6 GB, is
    larger than L2, so no flush is needed)."""
    import numpy as np
    import torch
    import kimi_delta_attention_28_b200 as kda
    from kimi_delta_attention_28_b200 import workloads as W
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.load_library()
    w = W.DECODE
    nsteps = warmup + steps
    inp = W.make_decode_inputs(w.B, w.H, w.dk, w.dv, nsteps, w.dtype, w.seed + rank, dev)
    S = inp["S"].clone()
    o = torch.empty(w.B, w.H, w.dv, dtype=w.dtype, device=dev)
    stream = torch.cuda.current_stream(dev)
    rng = np.random.default_rng(1)
    pairs = rng.choice(w.B * w.H, size=64, replace=False)
    n_idx = torch.tensor(pairs // w.H, device=dev)
    h_idx = torch.tensor(pairs % w.H, device=dev)
    o_last = None

    def step(t):
        kda.kda_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["g"][t], inp["beta"][t],
                            S, o)

    for t in range(warmup):
        step(t)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.02)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.perf_counter()
    ev[0].record(stream)
    for i in range(steps):
        step(warmup + i)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    clocks.stop()
    o_last = o[n_idx, h_idx].cpu()
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = max_over_ranks(total_ms, world, dev)
    if rank != 0:
        return None
    ms = total_ms / steps
    units = w.B * w.H
    per_unit = 2 * w.dk * w.dv * 4 + 3 * w.dk * 2 + w.dk * 4 + 4 + w.dv * 2
    bytes_step = units * per_unit
    hbm_peak, _, peak_src = load_peaks()
    gbs = bytes_step / (ms * 1e-3) / 1e9
    out = {
        "metric": "KDA decode steps/s (256 sequences x 96 heads, d=128, fp32 state in place)",
        "value": world * 1e3 / ms, "unit": "steps/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "N": w.B, "H": w.H, "dk": w.dk, "dv": w.dv,
                   "l2": "state (1.6 GB) larger than L2; no flush"},
        "roofline": {"bound": "hbm", "kernel": "kda_decode_kernel", "achieved": gbs,
                     "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                     "traffic": load_traffic("kda_decode_kernel", units),
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
                     "algorithmic_bytes_per_launch": bytes_step,
                     "algorithmic_bytes_rule": "per (sequence, head): state read + write "
                                               "2 x 64 KiB, q,k,v bf16, g fp32, beta, o bf16"},
        "gpu_launches": steps,
        "clocks": clocks.summary(t_wall0, t_wall1),
    }
    if cpu and world == 1:
        out["cpu_baseline"] = decode_cpu_baseline(w, inp, S, o_last, pairs, nsteps)
    return out


def decode_cpu_baseline(w, inp, S_gpu, o_last, pairs, nsteps, budget_s=10.0):
    """The oracle on 64 sampled (sequence, head) chains over every step the GPU ran
    (chains are independent, so the check is exact for them): steps/s scaled to the
    whole batch, and the parity of the final outputs and states of those chains."""
    import oracle
    n_idx = pairs // w.H
    h_idx = pairs % w.H
    pick = lambda x: x[:, n_idx, h_idx].unsqueeze(2).transpose(0, 1).contiguous()  # noqa: E731
    q, k, v, g = (pick(inp[n]).cpu() for n in ("q", "k", "v", "g"))
    beta = inp["beta"][:, n_idx, h_idx].transpose(0, 1).unsqueeze(2).contiguous().cpu()
    S0 = inp["S"][n_idx, h_idx].unsqueeze(1).contiguous().cpu()
    o_ref, S_ref = oracle.kda_fwd(q, k, v, g, beta, S0)
    # the timed sample: every step over the first `nt` (sequence, head) chains (whole
    # sequences, all heads), sized to a few seconds of oracle time
    nt, el = w.H, 0.0
    while True:
        ns = max(1, nt // w.H)
        sel = lambda x: x[:, :ns].reshape(x.shape[0], ns * w.H, *x.shape[3:])  # noqa: E731
        qs, ks, vs, gs = (sel(inp[n]).transpose(0, 1).unsqueeze(2).contiguous().cpu()
                          for n in ("q", "k", "v", "g"))
        bs = sel(inp["beta"].unsqueeze(-1)).transpose(0, 1).contiguous().cpu()
        Ss = inp["S"][:ns].reshape(ns * w.H, 1, w.dk, w.dv).contiguous().cpu()
        t0 = time.perf_counter()
        oracle.kda_fwd(qs, ks, vs, gs, bs, Ss)
        el = time.perf_counter() - t0
        if el > budget_s / 4 or ns >= w.B:
            break
        nt = min(w.B * w.H, nt * 4)
    used = min(ns * w.H, oracle.threads_available())
    S_g = S_gpu[n_idx, h_idx].unsqueeze(1).cpu()
    parity = {"tolerance": PARITY_TOL["bf16"],
              "o_last_step": _err(o_last.double().numpy(), o_ref[:, -1, 0]),
              "S": _err(S_g.double().numpy(), S_ref),
              "sample": f"{len(pairs)} sampled (sequence, head) chains over all {nsteps} steps"}
    steps_per_s = nsteps / el * (ns * w.H) / (w.B * w.H)
    return {"value": steps_per_s, "unit": "steps/s", "cores": int(used), "kind": "oracle",
            "sample": f"{ns * w.H} of {w.B * w.H} (sequence, head) chains (sequences 0..{ns - 1}, "
                      f"all heads) x {nsteps} steps, {el:.1f} s, scaled to the whole batch",
            "parity": parity}


def measure_speculative(steps, warmup, K=4, cpu=True):
    """Speculative decoding on the decode workload's shapes (256 sequences x 96 heads,
    d = 128, fp32 states): every step verifies K drafted tokens per sequence
    (kda_decode_verify, the state only read) and commits a seeded accepted count in
    [0, K] per sequence (kda_decode_commit, the state advanced in place)."""
    import torch
    import kimi_delta_attention_28_b200 as kda
    from kimi_delta_attention_28_b200 import workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    kda.load_library()
    w = W.DECODE
    nsteps = warmup + steps
    drafts = [W.make_prefill_inputs(w.B, K, w.H, w.dk, w.dv, w.dtype, i == 0,
                                    seed=w.seed + 100 + i, device=dev) for i in range(4)]
    S0 = drafts[0]["h0"]
    S = S0.clone()
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    accs = torch.randint(0, K + 1, (nsteps, w.B), generator=gen, dtype=torch.int32).to(dev)
    o = torch.empty(w.B, K, w.H, w.dv, dtype=w.dtype, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(t):
        d = drafts[t % len(drafts)]
        kda.kda_decode_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], S, o)
        kda.kda_decode_commit(d["k"], d["v"], d["g"], d["beta"], accs[t], S)

    for t in range(warmup):
        step(t)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.02)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.perf_counter()
    e0.record(stream)
    for i in range(steps):
        step(warmup + i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.perf_counter()
    clocks.stop()
    assert kda.device_error() == 0
    ms = e0.elapsed_time(e1) / steps
    units = w.B * w.H
    mean_acc = float(accs[warmup:].float().mean())
    tok_in = 3 * w.dk * 2 + w.dk * 4 + 4           # q, k, v bf16, g fp32, beta
    per_unit = (3 * w.dk * w.dv * 4                 # state: verify read, commit read + write
                + K * (tok_in + w.dv * 2)           # verify: K drafted tokens in, K outputs out
                + mean_acc * (tok_in - w.dk * 2))   # commit: k, v, g, beta of accepted tokens
    bytes_step = units * per_unit
    hbm_peak, _, peak_src = load_peaks()
    gbs = bytes_step / (ms * 1e-3) / 1e9
    out = {
        "metric": f"KDA speculative decode rounds/s (verify {K} drafted tokens + commit the "
                  "accepted prefix; 256 sequences x 96 heads, d=128)",
        "value": 1e3 / ms, "unit": "rounds/s", "ms_per_step": ms, "steps": steps,
        "warmup": warmup, "accepted_tokens_per_sequence_mean": mean_acc,
        "config": {"workload": f"speculative_bf16_N{w.B}_H{w.H}_d{w.dk}_K{K}", "N": w.B,
                   "H": w.H, "K": K, "accepted": "uniform in [0, K] per sequence (seeded)"},
        "roofline": {"bound": "hbm", "kernel": "kda_decode_multi_kernel (verify + commit)",
                     "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                     # mean DRAM bytes of a verify and a commit launch (ncu capture)
                     "traffic": load_traffic("kda_decode_multi_kernel", units),
                     "algorithmic_bytes_per_launch": bytes_step / 2,
                     "algorithmic_bytes_rule": "per (sequence, head): state read (verify) + read "
                                               "and write (commit), drafted inputs and outputs",
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)"},
        "vs_single_token_steps": "K single decode steps would move K x 2 x 64 KiB of state "
                                 "per (sequence, head); verify + commit move 3 x 64 KiB",
        "gpu_launches": 2 * steps,
        "clocks": clocks.summary(t_wall0, t_wall1),
    }
    if cpu:
        out["cpu_baseline"] = speculative_cpu_baseline(w, drafts, accs, S0, S, o, K, nsteps)
    return out


def measure_backward(name, steps, warmup, cpu=True, cpu_seconds=10.0):
    """The backward pass (kda_bwd) on a prefill workload: per step one call with
    seeded upstream gradients do (dtype of q) and dhT; inputs already on the device."""
    import torch
    import kimi_delta_attention_28_b200 as kda
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    kda.load_library()
    w, inp = workload_inputs(name, dev)
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    cu = inp["cu_seqlens"]
    N = B if cu is None else cu.numel() - 1
    nseq = 0 if cu is None else N
    gen = torch.Generator(device=dev).manual_seed(w.seed + 7)
    do = torch.randn(B, T, H, dv, generator=gen, device=dev).to(w.dtype)
    dhT = 0.1 * torch.randn(N, H, dk, dv, generator=gen, device=dev)
    ws = torch.empty(kda.bwd_workspace_size(B, T, H, dk, dv, nseq, w.dtype), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = None
    for _ in range(warmup):
        res = kda.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], cu, do,
                          dhT, workspace=ws)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.02)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    t_wall0 = time.perf_counter()
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        res = kda.kda_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], cu, do,
                          dhT, workspace=ws)
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.perf_counter()
    clocks.stop()
    assert kda.device_error() == 0
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    units = B * T * H
    nseg = kda.bwd_plan_segments(B, T, H, dk, dv, nseq, w.dtype)
    # fp32 work per token-head of the slice kernel as executed: the reverse step (~10 d^2)
    # and the forward recurrence (~4 d^2 a walk) for the recompute of a chunk's 8-token
    # states, the recompute of a piece's states and the checkpoint walk, which covers
    # every chunk of a chain (or segment) but its last
    if nseg >= 2:
        sc = -(-T // 64) // nseg                       # chunks per segment
        walk = (sc - 1) / sc
        schedule = f"segmented: {nseg} segments of {sc} chunk(s) per sequence"
        launches = 5    # prep, state pass, reversed records, state pass (gradient), slices
    else:
        walk = 1.0
        schedule = "per chain"
        launches = 1 + (1 if cu is not None else 0)
    fpt = 18.0 + 4.0 * walk
    flops = units * fpt * dk * dv
    peak_fp32 = 148 * 128 * 2 * 1.965e9 / 1e12    # CUDA-core fp32 FMA peak, TFLOP/s
    tf = flops / (ms * 1e-3) / 1e12
    out = {"metric": "KDA backward tokens/s (gradients of q, k, v, g, beta, h0)",
           "value": B * T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
           "warmup": warmup, "config": prefill_config(w, inp, 1),
           "roofline": {"bound": "alu", "kernel": "kda_bwd_slice_kernel",
                        "achieved": tf, "peak": peak_fp32, "unit": "TFLOP/s",
                        "frac": tf / peak_fp32,
                        "traffic": load_traffic("kda_bwd_slice_kernel", units),
                        "algorithmic_flops_per_launch": flops,
                        "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz "
                                       "(CUDA-core fp32, nominal clock)",
                        "flops_rule": f"{fpt:.1f} d_k d_v per token-head: the reverse step "
                                      "(10), two recompute levels (4 each) and the checkpoint "
                                      "walk over all chunks but a unit's last (4 x that share)",
                        "duration": "the whole kda_bwd call (the slice kernel's share of it: "
                                    "profiles/ launch list)"},
           "gpu_launches": steps * launches,
           "clocks": clocks.summary(t_wall0, t_wall1)}
    out["config"]["schedule"] = schedule
    if cpu:
        import numpy as np
        import oracle
        # whole sequence 0, all heads (a gradient depends on every later token)
        s0 = lambda x: x[:1].contiguous()  # noqa: E731
        t0 = time.perf_counter()
        ref = oracle.kda_bwd(s0(inp["q"]), s0(inp["k"]), s0(inp["v"]), s0(inp["g"]),
                             s0(inp["beta"]), None if inp["h0"] is None else s0(inp["h0"]),
                             s0(do), s0(dhT))
        el = time.perf_counter() - t0
        par = {"tolerance": ("every gradient rel-L2 <= 1e-2 (segmented: states and gradients "
                             "at segment bounds from the bf16 tensor-core records)")
               if nseg >= 2 else "fp32-stored gradients rel-L2 <= 1e-4; bf16-stored rel-L2 <= 1e-2",
               "sample": "all heads of sequence 0, every token"}
        for nm, got, r in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), res, ref):
            if got is not None:
                par[nm] = _err(got[:1].double().cpu().numpy(), r.reshape(got[:1].shape))
        out["cpu_baseline"] = {"value": T / el, "unit": "tokens/s",
                               "cores": min(H, oracle.threads_available()), "kind": "oracle",
                               "sample": f"sequence 0 ({T} tokens x {H} heads), {el:.1f} s; "
                                         "fp64 reverse accumulation, OpenMP over heads",
                               "parity": par}
        del np
    return out


def speculative_cpu_baseline(w, drafts, accs, S0, S_gpu, o_last, K, nsteps, nchains=64):
    """The oracle on 64 sampled (sequence, head) chains over every round the GPU ran,
    from the initial states: each chain's accepted tokens, round after round, then the
    last round's verify from the oracle's own state before it.  Chains are
    independent, so the check is exact for them; the time is scaled to the batch."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(2)
    pairs = rng.choice(w.B * w.H, size=nchains, replace=False)
    n_idx, h_idx = pairs // w.H, pairs % w.H
    acc = accs.cpu().numpy()
    host = [{k_: drafts[i][k_].cpu() for k_ in ("q", "k", "v", "g", "beta")}
            for i in range(len(drafts))]

    def packed(rounds):
        """The accepted tokens of rounds [0, rounds) of every sampled chain, packed."""
        cols = {k_: [] for k_ in ("k", "v", "g", "beta")}
        cu = [0]
        for n, h in zip(n_idx, h_idx):
            for t in range(rounds):
                a = int(acc[t, n])
                d = host[t % len(host)]
                for k_ in cols:
                    x = d[k_][n, :a, h]
                    cols[k_].append(x.double().numpy().reshape(a, 1, x.shape[-1])
                                    if k_ != "beta" else x.double().numpy().reshape(a, 1))
            cu.append(cu[-1] + sum(int(acc[t, n]) for t in range(rounds)))
        arr = {k_: np.ascontiguousarray(np.concatenate(v_, axis=0)) for k_, v_ in cols.items()}
        return arr, np.array(cu, dtype=np.int64)

    S0s = S0[n_idx, h_idx].unsqueeze(1).double().cpu().numpy()
    t0 = time.perf_counter()
    arr, cu = packed(nsteps - 1)
    _, S_before, used = oracle.kda_fwd_packed(np.zeros_like(arr["k"]), arr["k"], arr["v"],
                                              arr["g"], arr["beta"], S0s, cu)
    last = host[(nsteps - 1) % len(host)]
    pick = lambda x: x[n_idx, :, h_idx].unsqueeze(2)  # noqa: E731  [64, K, 1, d]
    o_ref = oracle.kda_decode_verify(pick(last["q"]), pick(last["k"]), pick(last["v"]),
                                     pick(last["g"]), last["beta"][n_idx, :, h_idx].unsqueeze(2),
                                     S_before)
    S_ref = oracle.kda_decode_commit(pick(last["k"]), pick(last["v"]), pick(last["g"]),
                                     last["beta"][n_idx, :, h_idx].unsqueeze(2),
                                     acc[nsteps - 1, n_idx], S_before)
    el = time.perf_counter() - t0
    o_g = o_last[n_idx, :, h_idx].unsqueeze(2).double().cpu().numpy()
    S_g = S_gpu[n_idx, h_idx].unsqueeze(1).double().cpu().numpy()
    return {"value": nsteps / el * nchains / (w.B * w.H), "unit": "rounds/s",
            "cores": int(min(used, nchains)), "kind": "oracle",
            "sample": f"{nchains} sampled (sequence, head) chains over all {nsteps} rounds, "
                      f"{el:.1f} s (tokens gathered in Python), scaled to the whole batch",
            "parity": {"tolerance": PARITY_TOL["bf16"], "o_last_round": _err(o_g, o_ref),
                       "S": _err(S_g, S_ref),
                       "sample": f"{nchains} sampled chains, every round, from the initial states"}}


# ---------------------------------------------------------------------------
# reference arm: the oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------
def run_reference(args, world, rank):
    """The oracle on a bounded sample of the workload, timed per step."""
    import numpy as np
    import oracle
    from kimi_delta_attention_28_b200 import workloads as W
    w = workload_of(args.workload)
    # The sample only: whole (sequence, head) chains over Ts tokens of one sequence,
    # drawn by the workload's generator at that size (the whole workload, converted to
    # fp64 on the host, would take about 90 GB at T = 1M), sized below so that warmup +
    # steps finish in about args.ref_seconds.  The config reports the whole workload.
    shapes = workload_shapes(w)
    B, T, H, dk = shapes["q"].shape
    Ts = min(T if w.varlen_seqs == 0 else
             W.varlen_lengths(w.varlen_seqs, *w.varlen_range, seed=w.seed)[0], 4096)
    h = host_f64(W.make_prefill_inputs(1, Ts, H, dk, w.dv, w.dtype, w.h0, w.seed, "cpu"))
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
    sample = (f"{chains} of {H} heads x {Ts} tokens of one sequence per step "
              f"(fp64 token-by-token C oracle)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded), same generator as the GPU arm",
            "config": prefill_config(w, shapes, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": int(used),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _free_device_memory():
    import torch
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def default_steps(workload):
    """Timed steps when --steps is not given (about a second of timed work or less)."""
    return {"long": 10, "few_chains": 100, "varlen": 100, "prefill": 1000, "decode": 300,
            "profile": 100, "speculative": 200, "backward": 5}[workload]


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about a second of timed work for the workload)")
    ap.add_argument("--warmup", type=int, default=None, help="untimed warm-up steps (>= 3)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOAD_KEYS), default=HEADLINE)
    ap.add_argument("--no-nested", action="store_true",
                    help="skip the other workloads nested under `workloads` (one GPU only)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ckpt-every", type=int, default=0,
                    help="prefill workloads: also store the state every N tokens (multiple of 64)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--two-launch", action="store_true",
                    help="prefill workloads: time the two-launch schedule (prep kernel, then "
                         "state pass) even where kda_fwd would overlap them in one launch")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    args = ap.parse_args()
    if args.steps is None:
        args.steps = default_steps(args.workload) if args.impl == "ours" else 3
    if args.warmup is None:
        args.warmup = 3 if args.workload == "long" else 20
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference" and args.workload in ("decode", "speculative", "backward"):
        ap.error("the reference arm covers the prefill workloads")
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    cpu = not args.no_cpu_baseline
    try:
        if args.workload == "decode":
            out = measure_decode(args.steps, args.warmup, world, rank, local, cpu=cpu)
        elif args.workload == "speculative":
            out = measure_speculative(args.steps, args.warmup, cpu=cpu) if rank == 0 else None
        elif args.workload == "backward":
            out = measure_backward("prefill", args.steps, args.warmup, cpu=cpu) if rank == 0 else None
        else:
            out = measure_prefill(args.workload, args.steps, args.warmup, world, rank, local,
                                  e2e=not args.no_e2e, cpu=cpu, cpu_seconds=args.cpu_seconds,
                                  ckpt_every=args.ckpt_every, two_launch=args.two_launch)
        if world == 1 and not args.no_nested and args.workload == HEADLINE and out is not None:
            # the other workloads, each with its own roofline and parity sample
            nested = {}
            for name in ("prefill", "varlen"):
                _free_device_memory()
                r = measure_prefill(name, default_steps(name), 20, e2e=False, cpu=cpu,
                                    cpu_seconds=min(args.cpu_seconds, 5.0))
                nested[name] = {k_: r[k_] for k_ in ("value", "unit", "ms_per_step", "steps",
                                                      "warmup", "config", "roofline", "path",
                                                      "kernels_ms", "gpu_launches", "clocks",
                                                      "cpu_baseline") if k_ in r}
            _free_device_memory()
            r = measure_decode(200, 20, cpu=cpu)
            nested["decode"] = {k_: r[k_] for k_ in ("metric", "value", "unit", "ms_per_step",
                                                      "steps", "warmup", "config", "roofline",
                                                      "gpu_launches", "clocks", "cpu_baseline")
                                if k_ in r}
            _free_device_memory()
            r = measure_speculative(200, 20, cpu=cpu)
            nested["speculative"] = r
            _free_device_memory()
            nested["backward"] = measure_backward("prefill", 5, 3, cpu=cpu)
            out["workloads"] = nested
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
