"""Seeded synthetic inputs for the KDA recurrence.

This module only draws random inputs; it holds none of the recurrence's
arithmetic, so both the CUDA path and the CPU oracle can consume what it makes.

Distributions (one set for every workload):
  * q, k ~ N(0, 1), L2-normalised over the key dimension for every
    (token, head); q additionally scaled by 1/sqrt(d_k);
  * v ~ N(0, 1);
  * g = -5 * sigmoid(z), z ~ N(-3, 1), so g lies in (-5, 0): the decay bound
    stated in the "Kimi K3" open-weights field notes, panel "g ∈ (-5, 0)";
  * beta = sigmoid(N(0, 1)) per (token, head);
  * initial states (where a workload has them) ~ N(0, 0.1^2), i.e. std 0.1.

q/k/v are drawn in fp32 and rounded to the workload's dtype; g, beta and the
state are fp32.  Large tensors are drawn in token slices so peak temporary
memory stays bounded; the values depend only on (seed, device, shape).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int                      # per-sequence length (fixed-length) or total (varlen)
    dk: int
    dv: int
    dtype: torch.dtype          # dtype of q, k, v and o
    h0: bool                    # nonzero initial state?
    varlen_seqs: int = 0        # >0: packed varlen with this many sequences
    varlen_range: tuple = (0, 0)
    decode_steps: int = 0       # >0: decode workload (B = sequences)
    seed: int = 0
    note: str = ""


TINY = Workload("tiny_f32_B1_H2_T64_d32", B=1, H=2, T=64, dk=32, dv=32,
                dtype=torch.float32, h0=False, seed=1000,
                note="fp32 everywhere, zero initial state")
PREFILL = Workload("prefill_bf16_B2_H8_T4096_d128", B=2, H=8, T=4096, dk=128, dv=128,
                   dtype=torch.bfloat16, h0=True, seed=1001,
                   note="bf16 q/k/v, fp32 g/beta/state, h0 ~ N(0, 0.1^2)")
LONG = Workload("long_bf16_B1_H16_T1048576_d128", B=1, H=16, T=1 << 20, dk=128, dv=128,
                dtype=torch.bfloat16, h0=False, seed=1002,
                note="1M-token context, zero initial state")
VARLEN = Workload("varlen_bf16_N16_H32_d128", B=1, H=32, T=0, dk=128, dv=128,
                  dtype=torch.bfloat16, h0=True, varlen_seqs=16,
                  varlen_range=(1024, 32768), seed=1003,
                  note="16 packed sequences, lengths log-uniform in [1024, 32768]")
DECODE = Workload("decode_bf16_N256_H96_d128", B=256, H=96, T=1, dk=128, dv=128,
                  dtype=torch.bfloat16, h0=True, decode_steps=1000, seed=1004,
                  note="one token per sequence per step, fp32 state updated in place")

FEW_CHAINS = Workload("few_chains_bf16_B1_H2_T262144_d128", B=1, H=2, T=1 << 18, dk=128,
                      dv=128, dtype=torch.bfloat16, h0=True, seed=1005,
                      note="two (sequence, head) chains of 4,096 chunks: too few to fill "
                           "the GPU, so the state pass is split in time")

PROFILE = Workload("profile_bf16_B1_H16_T16384_d128", B=1, H=16, T=1 << 14, dk=128, dv=128,
                   dtype=torch.bfloat16, h0=False, seed=1006,
                   note="the 1M-token workload's shape at 1/64 of its length: inputs and "
                        "records (about 0.7 GB) far larger than L2 but small enough for "
                        "profiler captures; DRAM bytes per token-head measured here scale "
                        "to the full workload")

ALL = (TINY, PREFILL, LONG, VARLEN, DECODE, FEW_CHAINS, PROFILE)
BY_NAME = {w.name: w for w in ALL}


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> list:
    """Sequence lengths floor(exp(U(ln lo, ln hi))) clamped to [lo, hi], drawn
    on the CPU so every device sees the same lengths."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    u = torch.rand(n, generator=gen, dtype=torch.float64)
    lens = torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
    return [int(min(max(x, lo), hi)) for x in lens.tolist()]


def cu_from_lengths(lengths, device="cpu") -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def _fill_qk(out: torch.Tensor, gen, scale: float, slice_tokens: int):
    """out: [..., T, H, d] view whose token dim is -3; filled slice by slice."""
    T = out.shape[-3]
    for t0 in range(0, T, slice_tokens):
        t1 = min(T, t0 + slice_tokens)
        shape = out[..., t0:t1, :, :].shape
        x = torch.randn(shape, generator=gen, device=out.device, dtype=torch.float32)
        x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        if scale != 1.0:
            x = x * scale
        out[..., t0:t1, :, :].copy_(x)


def _fill_normal(out: torch.Tensor, gen, mean: float, std: float, slice_tokens: int):
    T = out.shape[-3] if out.dim() >= 3 else out.shape[0]
    for t0 in range(0, T, slice_tokens):
        t1 = min(T, t0 + slice_tokens)
        view = out[..., t0:t1, :, :] if out.dim() >= 3 else out[t0:t1]
        x = torch.randn(view.shape, generator=gen, device=out.device, dtype=torch.float32)
        view.copy_(x * std + mean)


def _fill_g(out: torch.Tensor, gen, slice_tokens: int):
    T = out.shape[-3]
    for t0 in range(0, T, slice_tokens):
        t1 = min(T, t0 + slice_tokens)
        view = out[..., t0:t1, :, :]
        z = torch.randn(view.shape, generator=gen, device=out.device, dtype=torch.float32) - 3.0
        view.copy_(-5.0 * torch.sigmoid(z))


def _fill_beta(out: torch.Tensor, gen, slice_tokens: int):
    T = out.shape[-2]
    for t0 in range(0, T, slice_tokens):
        t1 = min(T, t0 + slice_tokens)
        view = out[..., t0:t1, :]
        view.copy_(torch.sigmoid(torch.randn(view.shape, generator=gen, device=out.device,
                                             dtype=torch.float32)))


def make_prefill_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                        h0: bool = False, seed: int = 0, device="cpu", lengths=None,
                        slice_tokens: int = 1 << 16) -> dict:
    """Inputs of a prefill call.

    Fixed-length: q, k, g [B, T, H, dk]; v [B, T, H, dv]; beta [B, T, H];
    h0 [B, H, dk, dv] or None; cu_seqlens None.
    Varlen (``lengths`` given): B must be 1, T = sum(lengths), and h0 is
    [len(lengths), H, dk, dv]; cu_seqlens is int32 [N+1] on ``device``.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device).manual_seed(seed)
    if lengths is not None:
        assert B == 1
        T = int(sum(lengths))
        N = len(lengths)
    else:
        N = B
    q = torch.empty(B, T, H, dk, dtype=dtype, device=device)
    k = torch.empty(B, T, H, dk, dtype=dtype, device=device)
    v = torch.empty(B, T, H, dv, dtype=dtype, device=device)
    g = torch.empty(B, T, H, dk, dtype=torch.float32, device=device)
    beta = torch.empty(B, T, H, dtype=torch.float32, device=device)
    _fill_qk(q, gen, 1.0 / math.sqrt(dk), slice_tokens)
    _fill_qk(k, gen, 1.0, slice_tokens)
    _fill_normal(v, gen, 0.0, 1.0, slice_tokens)
    _fill_g(g, gen, slice_tokens)
    _fill_beta(beta, gen, slice_tokens)
    state = None
    if h0:
        state = torch.randn(N, H, dk, dv, generator=gen, device=device,
                            dtype=torch.float32) * 0.1
    cu = cu_from_lengths(lengths, device) if lengths is not None else None
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=state, cu_seqlens=cu)


def make_decode_inputs(N: int, H: int, dk: int, dv: int, steps: int, dtype=torch.bfloat16,
                       seed: int = 0, device="cpu") -> dict:
    """Inputs of ``steps`` chained decode steps: q, k, g [steps, N, H, dk];
    v [steps, N, H, dv]; beta [steps, N, H]; initial state S [N, H, dk, dv]."""
    device = torch.device(device)
    gen = torch.Generator(device=device).manual_seed(seed)
    S = torch.randn(N, H, dk, dv, generator=gen, device=device, dtype=torch.float32) * 0.1
    # The step index plays the role of the token axis for the slice-wise fills.
    q = torch.empty(steps, N, H, dk, dtype=dtype, device=device)
    k = torch.empty(steps, N, H, dk, dtype=dtype, device=device)
    v = torch.empty(steps, N, H, dv, dtype=dtype, device=device)
    g = torch.empty(steps, N, H, dk, dtype=torch.float32, device=device)
    beta = torch.empty(steps, N, H, dtype=torch.float32, device=device)
    sl = 64
    _fill_qk(q, gen, 1.0 / math.sqrt(dk), sl)
    _fill_qk(k, gen, 1.0, sl)
    _fill_normal(v, gen, 0.0, 1.0, sl)
    _fill_g(g, gen, sl)
    _fill_beta(beta, gen, sl)
    return dict(q=q, k=k, v=v, g=g, beta=beta, S=S)


def make_workload(w: Workload, device="cpu", steps: int | None = None) -> dict:
    if w.decode_steps:
        return make_decode_inputs(w.B, w.H, w.dk, w.dv, steps or w.decode_steps, w.dtype,
                                  w.seed, device)
    lengths = None
    if w.varlen_seqs:
        lengths = varlen_lengths(w.varlen_seqs, *w.varlen_range, seed=w.seed)
    return make_prefill_inputs(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.h0, w.seed, device,
                               lengths)
