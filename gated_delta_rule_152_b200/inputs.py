"""Seeded synthetic inputs for the KDA layer workloads.

This module only draws random numbers and shapes them; it holds none of the
layer's arithmetic (no normalisation, decay or state update).  Both the CUDA
path and the fp64 CPU oracle take their inputs from here, always generated on
the CPU with a ``torch.Generator`` so the same seed gives the same tensors on
any machine.

Distributions (per workload, all drawn in fp32 or fp64 and then rounded to the
storage dtype):

* q, k, v ~ N(0, 1) (q and k are L2-normalised inside the layer, not here);
* g = log(alpha) per channel:
    - ``logsigmoid``: g = log(sigmoid(x)) with x ~ N(3, 1) (alpha = sigmoid(x));
    - ``neg_softplus``: g = -softplus(x) with x ~ N(-3, 1);
  both evaluated in fp64 from the fp32 draw, then rounded to fp32;
* beta = sigmoid(N(0, 1)) per token and head, fp32;
* initial state S0 ~ N(0, 0.02^2) (std 0.02) fp32, or absent (zeros).

Layouts: q, k, v, g are ``[total_T, H, d]`` (token-major, then head, then
channel); beta is ``[total_T, H]``; cu_seqlens is int32 ``[N + 1]``; states are
``[N, H, d, d]`` with rows = key channels and columns = value channels.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

D = 128


@dataclasses.dataclass(frozen=True)
class PrefillSpec:
    name: str
    seed: int
    n_seqs: int
    heads: int
    dtype: torch.dtype
    decay: str                       # "logsigmoid" | "neg_softplus"
    seq_len: Optional[int] = None    # fixed length (n_seqs == 1 here)
    len_range: Optional[tuple] = None  # (lo, hi) inclusive, uniform integers
    init_state_std: float = 0.0      # 0 -> no initial state
    final_state: bool = False
    d: int = D


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    name: str
    seed: int
    n_seqs: int
    layers: int
    heads: int
    dtype: torch.dtype
    decay: str = "neg_softplus"
    state_std: float = 0.02
    d: int = D


# The five workloads: a tiny fp32 forward, a single-layer 8K prefill, a 128K
# long-context prefill, a 16-sequence varlen pack and a 256-sequence x 34-layer
# decode step.
TINY_FP32 = PrefillSpec("tiny_fp32_T256_H2", 1000, 1, 2, torch.float32, "logsigmoid", seq_len=256,
                        final_state=True)
PREFILL_8K = PrefillSpec("prefill_bf16_T8192_H32", 1001, 1, 32, torch.bfloat16, "neg_softplus",
                         seq_len=8192, final_state=True)
PREFILL_128K = PrefillSpec("prefill_bf16_T131072_H32", 1002, 1, 32, torch.bfloat16, "neg_softplus",
                           seq_len=131072, init_state_std=0.02, final_state=True)
VARLEN_16 = PrefillSpec("varlen_bf16_16seq_512to16384_H32", 1003, 16, 32, torch.bfloat16,
                        "neg_softplus", len_range=(512, 16384), init_state_std=0.02,
                        final_state=True)
DECODE_256x34 = DecodeSpec("decode_bf16_256seq_34layer_H32", 1004, 256, 34, 32, torch.bfloat16)

PREFILL_WORKLOADS = {s.name: s for s in (TINY_FP32, PREFILL_8K, PREFILL_128K, VARLEN_16)}


@dataclasses.dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    cu_seqlens: torch.Tensor
    initial_state: Optional[torch.Tensor]
    spec: Optional[PrefillSpec] = None

    @property
    def total_T(self) -> int:
        return int(self.q.shape[0])

    @property
    def n_seqs(self) -> int:
        return int(self.cu_seqlens.numel() - 1)

    @property
    def heads(self) -> int:
        return int(self.q.shape[1])

    def to(self, device) -> "PrefillInputs":
        mv = lambda t: None if t is None else t.to(device)
        return PrefillInputs(mv(self.q), mv(self.k), mv(self.v), mv(self.g), mv(self.beta),
                             mv(self.cu_seqlens), mv(self.initial_state), self.spec)


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor      # [N, H, d]
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor      # [N, H, d] fp32
    beta: torch.Tensor   # [N, H] fp32

    def to(self, device) -> "DecodeInputs":
        return DecodeInputs(*(t.to(device) for t in (self.q, self.k, self.v, self.g, self.beta)))


def _gen(seed: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(int(seed))


def _decay(x32: torch.Tensor, kind: str) -> torch.Tensor:
    """g from its fp32 source draw, evaluated in fp64 and rounded to fp32, in
    place and in slices so large workloads do not need an fp64 copy."""
    if kind not in ("logsigmoid", "neg_softplus"):
        raise ValueError(f"unknown decay distribution {kind!r}")
    flat = x32.view(-1)
    step = 1 << 24
    for s in range(0, flat.numel(), step):
        x = flat[s:s + step].double()
        g = torch.nn.functional.logsigmoid(x) if kind == "logsigmoid" else -torch.nn.functional.softplus(x)
        flat[s:s + step] = g.float()
    return x32


def _decay_source(shape, kind: str, gen: torch.Generator) -> torch.Tensor:
    mean = 3.0 if kind == "logsigmoid" else -3.0
    return torch.randn(shape, generator=gen, dtype=torch.float32) + mean


def seq_lengths(spec: PrefillSpec) -> list:
    if spec.seq_len is not None:
        return [int(spec.seq_len)] * spec.n_seqs
    lo, hi = spec.len_range
    gen = _gen(spec.seed * 7 + 1)
    return [int(x) for x in torch.randint(lo, hi + 1, (spec.n_seqs,), generator=gen)]


def make_prefill(spec: PrefillSpec, heads: Optional[int] = None,
                 lengths: Optional[list] = None) -> PrefillInputs:
    """Draw one workload on the CPU.  ``heads``/``lengths`` override the spec
    (used by tests to build smaller cases with the same distributions)."""
    H = spec.heads if heads is None else int(heads)
    lens = seq_lengths(spec) if lengths is None else [int(x) for x in lengths]
    d = spec.d
    gen = _gen(spec.seed)
    total = sum(lens)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    if lens:
        cu[1:] = torch.tensor(lens, dtype=torch.int64).cumsum(0).to(torch.int32)
    q = torch.randn((total, H, d), generator=gen, dtype=torch.float32).to(spec.dtype)
    k = torch.randn((total, H, d), generator=gen, dtype=torch.float32).to(spec.dtype)
    v = torch.randn((total, H, d), generator=gen, dtype=torch.float32).to(spec.dtype)
    g = _decay(_decay_source((total, H, d), spec.decay, gen), spec.decay)
    beta = torch.sigmoid(torch.randn((total, H), generator=gen, dtype=torch.float32).double()).float()
    s0 = None
    if spec.init_state_std > 0:
        s0 = torch.randn((len(lens), H, d, d), generator=gen, dtype=torch.float32) * spec.init_state_std
    return PrefillInputs(q, k, v, g, beta, cu, s0, spec)


def make_custom_prefill(seed: int, lengths, heads: int, dtype=torch.bfloat16,
                        decay: str = "neg_softplus", init_state_std: float = 0.0,
                        d: int = D) -> PrefillInputs:
    spec = PrefillSpec(f"custom_{seed}", seed, len(lengths), heads, dtype, decay,
                       len_range=(0, 0), init_state_std=init_state_std, d=d)
    return make_prefill(spec, heads=heads, lengths=list(lengths))


def make_decode_tokens(spec: DecodeSpec, layer: int, n_seqs: Optional[int] = None) -> DecodeInputs:
    """The one new token per sequence for one layer's decode step."""
    N = spec.n_seqs if n_seqs is None else int(n_seqs)
    H, d = spec.heads, spec.d
    gen = _gen(spec.seed * 1000 + 2 * layer + 1)
    q = torch.randn((N, H, d), generator=gen, dtype=torch.float32).to(spec.dtype)
    k = torch.randn((N, H, d), generator=gen, dtype=torch.float32).to(spec.dtype)
    v = torch.randn((N, H, d), generator=gen, dtype=torch.float32).to(spec.dtype)
    g = _decay(_decay_source((N, H, d), spec.decay, gen), spec.decay)
    beta = torch.sigmoid(torch.randn((N, H), generator=gen, dtype=torch.float32).double()).float()
    return DecodeInputs(q, k, v, g, beta)


def make_decode_state(spec: DecodeSpec, layer: int, n_seqs: Optional[int] = None,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One layer's state slab ``[N, H, d, d]`` fp32, S ~ N(0, std^2).

    Each layer has its own seed, so a test can regenerate any single layer
    without drawing the other 33."""
    N = spec.n_seqs if n_seqs is None else int(n_seqs)
    H, d = spec.heads, spec.d
    gen = _gen(spec.seed * 1000 + 2 * layer)
    shape = (N, H, d, d)
    if out is None:
        out = torch.empty(shape, dtype=torch.float32)
    out.normal_(0.0, spec.state_std, generator=gen)
    return out
