"""Seeded synthetic inputs for the gated delta rule (shared by tests, smoke and bench).

This module draws random numbers and lays them out; it computes none of the
rule's arithmetic.  The gate tensors ``g`` and ``beta`` that the library takes
as inputs are drawn through the layer's own parametrisation so that their value
distribution matches the pages' workloads ("手撕Qwen3-Next" walkthrough,
section 一(一)1 initialisation and 4 "形状调整"):

    beta = sigmoid(b),   g = -exp(A_log) * softplus(a + dt_bias),
    A ~ U(0, 16) per v-head,  A_log = log(A),  dt_bias = 1,   a, b ~ N(0, 1).

That parametrisation is upstream of the library's boundary (the library takes
``g`` and ``beta``); it is evaluated here once, in fp32 on the host, and both
the CUDA path and the oracle consume the same stored fp32 tensors.

Draw order for one workload (torch CPU ``Generator`` seeded with ``seed``):
lengths (varlen only), q, k, v, b, a, A, initial state.  fp32 normal draws are
cast to bf16 where the workload stores bf16 (round to nearest even).

Named workloads (``WORKLOADS``) carry the sizes of the five configurations the
method is measured on; tests also build smaller cases with :func:`make_prefill`.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int
    seq_len: Optional[int]          # None => varlen (lengths drawn in [len_lo, len_hi])
    nqk: int
    nv: int
    d: int
    chunk: int
    io: str                         # "f32" or "bf16" (dtype of q, k, v, out)
    init_state: bool
    len_lo: int = 0
    len_hi: int = 0
    steps: int = 0                  # decode workloads: tokens per sequence

    @property
    def dtype(self):
        return torch.float32 if self.io == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_f32_d64": Workload("tiny_f32_d64", 1, 256, 1, 1, 64, 64, "f32", False),
    "batch_f32_d128": Workload("batch_f32_d128", 4, 4096, 4, 8, 128, 128, "f32", True),
    "long_bf16_nv32": Workload("long_bf16_nv32", 2, 32768, 16, 32, 128, 64, "bf16", False),
    "varlen_bf16_nv32": Workload("varlen_bf16_nv32", 32, None, 16, 32, 128, 64, "bf16", True,
                                 len_lo=100, len_hi=16384),
    "decode_bf16_nv32": Workload("decode_bf16_nv32", 256, None, 16, 32, 128, 0, "bf16", True,
                                 steps=1024),
}
# index order of the five measured configurations
WORKLOAD_ORDER = ["tiny_f32_d64", "batch_f32_d128", "long_bf16_nv32", "varlen_bf16_nv32",
                  "decode_bf16_nv32"]


def varlen_lengths(num_seqs: int, lo: int, hi: int, gen: torch.Generator, chunk: int = 64):
    """Lengths ~ U{lo..hi}; at least one length is 1 mod ``chunk`` (a one-row tail chunk)."""
    lens = torch.randint(lo, hi + 1, (num_seqs,), generator=gen, dtype=torch.int64)
    if not bool(((lens % chunk) == 1).any()):
        lens[0] = ((int(lens[0]) // chunk) * chunk + 1) if int(lens[0]) > chunk else chunk + 1
    return lens


def cu_from_lengths(lens) -> torch.Tensor:
    lens = torch.as_tensor(lens, dtype=torch.int64)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens, 0)
    return cu.to(torch.int32)


def draw_gates(b: torch.Tensor, a: torch.Tensor, A: torch.Tensor, dt_bias: float = 1.0):
    """beta = sigmoid(b), g = -exp(log A) * softplus(a + dt_bias), in fp32.

    ``b``, ``a`` are [..., Nv]; ``A`` is [Nv].  This is the distribution recipe
    of the layer's gate parametrisation, used to shape the synthetic inputs.
    """
    A_log = torch.log(A.float())
    beta = torch.sigmoid(b.float())
    g = -torch.exp(A_log) * torch.nn.functional.softplus(a.float() + dt_bias)
    return g.contiguous(), beta.contiguous()


def make_prefill(num_seqs: int = 1, seq_len: Optional[int] = 256, nqk: int = 1, nv: int = 1,
                 d: int = 64, dv: Optional[int] = None, io: str = "f32", init_state: bool = False,
                 seed: int = 0, lengths=None, len_lo: int = 100, len_hi: int = 16384,
                 gate: str = "layer", A_hi: float = 16.0, state_std: float = 0.1,
                 chunk: int = 64, device: str = "cpu"):
    """Draw one packed prefill batch.

    gate: "layer" (the layer parametrisation above, A ~ U(0, A_hi)), "zero"
    (g = 0), "beta1" (layer g, beta = 1), "zero_beta1" (g = 0, beta = 1) or
    "beta0" (layer g, beta = 0).

    Returns a dict with q, k [T,Nqk,Dk], v [T,Nv,Dv] (``io`` dtype), g, beta
    [T,Nv] fp32, initial_state [N,Nv,Dk,Dv] fp32 or None, cu_seqlens int32
    [N+1], the integer sizes, and the raw gate inputs they were drawn from:
    a, b [T,Nv] fp32, A_log = log A [Nv] and dt_bias [Nv] (= 1) fp32 (the
    "gate" overrides above apply to g and beta only).
    """
    dv = d if dv is None else dv
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    if lengths is None:
        if seq_len is None:
            lengths = varlen_lengths(num_seqs, len_lo, len_hi, gen, chunk)
        else:
            lengths = torch.full((num_seqs,), int(seq_len), dtype=torch.int64)
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    cu = cu_from_lengths(lengths)
    T = int(cu[-1])
    dtype = torch.float32 if io == "f32" else torch.bfloat16
    q = torch.randn(T, nqk, d, generator=gen).to(dtype)
    k = torch.randn(T, nqk, d, generator=gen).to(dtype)
    v = torch.randn(T, nv, dv, generator=gen).to(dtype)
    b = torch.randn(T, nv, generator=gen)
    a = torch.randn(T, nv, generator=gen)
    A = torch.rand(nv, generator=gen) * A_hi
    A = torch.clamp(A, min=1e-12)
    s0 = (torch.randn(len(lengths), nv, d, dv, generator=gen) * state_std) if init_state else None
    g, beta = draw_gates(b, a, A)
    if gate in ("zero", "zero_beta1"):
        g = torch.zeros_like(g)
    if gate in ("beta1", "zero_beta1"):
        beta = torch.ones_like(beta)
    if gate == "beta0":
        beta = torch.zeros_like(beta)
    out = dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=s0, cu_seqlens=cu,
               T=T, num_seqs=len(lengths), nqk=nqk, nv=nv, dk=d, dv=dv, io=io,
               a=a.contiguous(), b=b.contiguous(), A_log=torch.log(A.float()).contiguous(),
               dt_bias=torch.full((nv,), 1.0))
    if device != "cpu":
        for key in ("q", "k", "v", "g", "beta", "initial_state", "cu_seqlens", "a", "b", "A_log",
                    "dt_bias"):
            if out[key] is not None:
                out[key] = out[key].to(device)
    return out


def make_workload(name: str, seed: int, device: str = "cpu", **overrides):
    """Draw the named prefill workload (see ``WORKLOADS``)."""
    w = WORKLOADS[name]
    kw = dict(num_seqs=w.num_seqs, seq_len=w.seq_len, nqk=w.nqk, nv=w.nv, d=w.d, io=w.io,
              init_state=w.init_state, seed=seed, len_lo=w.len_lo, len_hi=w.len_hi,
              chunk=w.chunk or 64, device=device)
    kw.update(overrides)
    out = make_prefill(**kw)
    out["chunk"] = w.chunk
    return out


def make_decode(num_seqs: int = 256, steps: int = 8, nqk: int = 16, nv: int = 32, d: int = 128,
                io: str = "bf16", seed: int = 4, state_std: float = 0.1, A_hi: float = 16.0,
                device: str = "cpu"):
    """Draw a decode run: ``steps`` fresh tokens for each of ``num_seqs`` sequences.

    Returns q, k [steps,N,Nqk,D], v [steps,N,Nv,D] (``io`` dtype), g, beta
    [steps,N,Nv] fp32, the initial state [N,Nv,D,D] fp32, and the raw gate
    inputs a, b [steps,N,Nv], A_log [Nv], dt_bias [Nv] (= 1) fp32.  Drawn on
    ``device`` with a generator of that device (CPU and CUDA streams differ).
    """
    gen = torch.Generator(device=device).manual_seed(int(seed))
    dtype = torch.float32 if io == "f32" else torch.bfloat16
    kw = dict(generator=gen, device=device)
    q = torch.randn(steps, num_seqs, nqk, d, **kw).to(dtype)
    k = torch.randn(steps, num_seqs, nqk, d, **kw).to(dtype)
    v = torch.randn(steps, num_seqs, nv, d, **kw).to(dtype)
    b = torch.randn(steps, num_seqs, nv, **kw)
    a = torch.randn(steps, num_seqs, nv, **kw)
    A = torch.clamp(torch.rand(nv, **kw) * A_hi, min=1e-12)
    s0 = torch.randn(num_seqs, nv, d, d, **kw) * state_std
    g, beta = draw_gates(b, a, A)
    return dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=s0, num_seqs=num_seqs,
                steps=steps, nqk=nqk, nv=nv, dk=d, dv=d, io=io,
                a=a.contiguous(), b=b.contiguous(), A_log=torch.log(A.float()).contiguous(),
                dt_bias=torch.full((nv,), 1.0, device=device))


def make_norm_inputs(shape, io: str = "bf16", seed: int = 0, device: str = "cpu"):
    """Inputs of the gated RMSNorm epilogue for outputs of ``shape`` [..., Dv].

    z ~ N(0, 1) in the io dtype (the layer's z projection of unit-scale hidden
    states) and a per-column gain ~ U(0.5, 1.5) fp32 (initialised to 1 in the
    layer; spread here so that a wrong column shows).
    """
    gen = torch.Generator(device=device).manual_seed(int(seed) + 7919)
    dtype = torch.float32 if io == "f32" else torch.bfloat16
    z = torch.randn(*shape, generator=gen, device=device).to(dtype).contiguous()
    w = (torch.rand(shape[-1], generator=gen, device=device) + 0.5).contiguous()
    return z, w


def make_conv_inputs(rows: int, nqk: int, nv: int, dk: int, dv: int, ksize: int = 4, io: str = "bf16",
                     seed: int = 0, num_states: int = 0, bias: bool = True, device: str = "cpu"):
    """Inputs of the causal conv1d + SiLU over packed [q | k | v] channels.

    mixed_qkv [rows, C] ~ N(0, 1) (the layer's projection of unit-scale hidden
    states), C = 2 nqk dk + nv dv; weight [C, K] ~ U(-1/sqrt(K), 1/sqrt(K)) and
    bias [C] likewise (torch's default Conv1d init for a depthwise conv, fan-in
    K); conv states [num_states, C, K] ~ N(0, 1) in the io dtype (cached
    pre-convolution inputs), or None.
    """
    gen = torch.Generator(device=device).manual_seed(int(seed) + 104729)
    dtype = torch.float32 if io == "f32" else torch.bfloat16
    C = 2 * nqk * dk + nv * dv
    bound = 1.0 / float(ksize) ** 0.5
    x = torch.randn(rows, C, generator=gen, device=device).to(dtype).contiguous()
    w = ((torch.rand(C, ksize, generator=gen, device=device) * 2 - 1) * bound).contiguous()
    b = ((torch.rand(C, generator=gen, device=device) * 2 - 1) * bound).contiguous() if bias else None
    st = (torch.randn(num_states, C, ksize, generator=gen, device=device).to(dtype).contiguous()
          if num_states else None)
    return dict(x=x, weight=w, bias=b, state=st, C=C)
