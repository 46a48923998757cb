"""Seeded synthetic workloads for one MoE layer forward.

This module holds only workload shapes and seeded random inputs.  It contains none of
the layer's arithmetic (no routing, no capacity, no FFN), so both the CUDA path and the
CPU oracle can be fed from it without sharing any of the method's code.

The five named workloads follow the load profiles the "Expert parallelism for MoE,
measurements before launch" page (airouter.kz) asks for: a short decode, a production
prefill, a long/skewed prefill and a mixed stress batch, with the model shapes of
Mixtral-8x7B, Mixtral-8x22B and DeepSeek-V3.

Input recipe (all seeded):
  x ~ N(0, 1); W_router ~ N(0, 1/d) in fp32; W_gate, W_up ~ N(0, 1/d); W_down ~ N(0, 1/f).
  bf16 workloads round x and the expert weights to bf16 (round-to-nearest-even); the
  router weight and the logit bias stay fp32.
  "zipf" bias: per-expert b[pi(r)] = beta * ln(E * p_r), p_r proportional to r^-1.1,
  pi a seeded permutation, beta chosen so the routed max/mean load is about 3.
  "chunks" bias: 64 single-token decode chunks, then prefill chunks of length
  round(exp(U[ln 128, ln 4096])) until T tokens (last chunk truncated); every chunk draws
  one bias vector N(0, 0.5^2) over the experts, shared by its tokens; passed as [T, E].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

SOFTMAX = 0
SIGMOID = 1
LAYOUT_COMPACT = 0
LAYOUT_PADDED = 1
F32 = 0
BF16 = 1


@dataclasses.dataclass(frozen=True)
class MoEShape:
    name: str
    T: int
    d_model: int
    d_ff: int
    E: int
    k: int
    gating: int              # SOFTMAX or SIGMOID
    capacity_factor: float   # <= 0: dropless
    dtype: int               # F32 or BF16
    bias: str = "none"       # "none" | "zipf" | "chunks"
    layout: int = LAYOUT_COMPACT
    seed: int = 1234
    zipf_s: float = 1.1
    zipf_beta: float = 0.11  # fitted: routed max/mean 2.96 on the 16384-token DeepSeek-shaped prefill
    chunk_bias_std: float = 0.5
    n_decode_tokens: int = 64
    n_groups: int = 0          # group-limited routing (0: off)
    topk_groups: int = 0
    bias_mode: int = 0         # 0: bias in score and weights; 1: selection only
    drop_policy: int = 0       # 0: token order; 1: pick rank first; 2: score priority

    def replace(self, **kw) -> "MoEShape":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16

    @property
    def assignments(self) -> int:
        return self.T * self.k


# The five workloads, by what they are.
TINY_FP32 = MoEShape("tiny_fp32_T64_d128_f256_E8_k2", 64, 128, 256, 8, 2, SOFTMAX, 1.25, F32,
                     seed=1235)
MIXTRAL_8X7B = MoEShape("mixtral8x7b_prefill_T4096", 4096, 4096, 14336, 8, 2, SOFTMAX, 0.0, BF16,
                        seed=1236)
DSV3_DECODE = MoEShape("dsv3_decode_T128", 128, 7168, 2048, 256, 8, SIGMOID, 0.0, BF16,
                       seed=1237)
DSV3_PREFILL_ZIPF = MoEShape("dsv3_prefill_zipf_T16384", 16384, 7168, 2048, 256, 8, SIGMOID, 1.0,
                             BF16, bias="zipf", seed=1238)
MIXTRAL_8X22B_MIXED = MoEShape("mixtral8x22b_mixed_T8192", 8192, 6144, 16384, 8, 2, SOFTMAX, 1.25,
                               BF16, bias="chunks", seed=1239)

WORKLOADS = {w.name: w for w in (TINY_FP32, MIXTRAL_8X7B, DSV3_DECODE, DSV3_PREFILL_ZIPF,
                                 MIXTRAL_8X22B_MIXED)}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def zipf_bias(E: int, s: float, beta: float, seed: int) -> torch.Tensor:
    """Per-expert additive logit bias whose popularity ranks follow Zipf(s)."""
    g = _gen(seed, "cpu")
    perm = torch.randperm(E, generator=g)
    r = torch.arange(1, E + 1, dtype=torch.float64)
    p = r.pow(-s)
    p = p / p.sum()
    b = torch.empty(E, dtype=torch.float64)
    b[perm] = beta * torch.log(E * p)
    return b.to(torch.float32)


def mixed_chunks(T: int, n_decode: int, seed: int) -> list[int]:
    """Chunk lengths of a mixed batch: n_decode single tokens, then log-uniform prefill
    chunks in [128, 4096], the last one truncated so the lengths sum to T."""
    g = _gen(seed, "cpu")
    lens = [1] * min(n_decode, T)
    total = sum(lens)
    lo, hi = math.log(128.0), math.log(4096.0)
    while total < T:
        u = torch.rand((), generator=g, dtype=torch.float64).item()
        L = int(round(math.exp(lo + (hi - lo) * u)))
        L = min(L, T - total)
        lens.append(L)
        total += L
    return lens


def chunk_bias(T: int, E: int, std: float, n_decode: int, seed: int) -> torch.Tensor:
    lens = mixed_chunks(T, n_decode, seed)
    g = _gen(seed + 7919, "cpu")
    rows = []
    for L in lens:
        b = torch.randn(E, generator=g, dtype=torch.float32) * std
        rows.append(b.expand(L, E))
    return torch.cat(rows, 0).contiguous()


@dataclasses.dataclass
class MoEInputs:
    shape: MoEShape
    x: torch.Tensor              # [T, d] fp32 or bf16
    w_router: torch.Tensor       # [d, E] fp32
    logit_bias: Optional[torch.Tensor]  # None, [E] or [T, E] fp32
    w_gate: torch.Tensor         # [E, f, d]
    w_up: torch.Tensor           # [E, f, d]
    w_down: torch.Tensor         # [E, d, f]

    @property
    def bias_row_stride(self) -> int:
        if self.logit_bias is None or self.logit_bias.dim() == 1:
            return 0
        return self.logit_bias.shape[1]


def expert_weights(shape: MoEShape, e: int, device="cpu"):
    """(W_g[e] [f, d], W_u[e] [f, d], W_d[e] [d, f]) of expert e.  Every expert draws from
    its own seeded stream, so one expert's weights can be made without the others'."""
    dev = torch.device(device)
    g = _gen(shape.seed * 65537 + 3 + e, dev)
    d, f, dt = shape.d_model, shape.d_ff, shape.torch_dtype
    wg = _randn((f, d), 1.0 / math.sqrt(d), g, dev).to(dt)
    wu = _randn((f, d), 1.0 / math.sqrt(d), g, dev).to(dt)
    wd = _randn((d, f), 1.0 / math.sqrt(f), g, dev).to(dt)
    return wg, wu, wd


def make_inputs(shape: MoEShape, device="cpu", weights: bool = True) -> MoEInputs:
    """Seeded inputs for `shape` on `device`.  Expert weights are drawn one expert at a time
    (expert_weights) so that the fp32 staging buffer stays small for the 22 GB
    DeepSeek-shaped layers."""
    dev = torch.device(device)
    g = _gen(shape.seed, dev)
    T, d, f, E = shape.T, shape.d_model, shape.d_ff, shape.E
    dt = shape.torch_dtype
    x = _randn((T, d), 1.0, g, dev).to(dt)
    w_router = _randn((d, E), 1.0 / math.sqrt(d), g, dev)
    if shape.bias == "none":
        bias = None
    elif shape.bias == "zipf":
        bias = zipf_bias(E, shape.zipf_s, shape.zipf_beta, shape.seed + 1).to(dev)
    elif shape.bias == "chunks":
        bias = chunk_bias(T, E, shape.chunk_bias_std, shape.n_decode_tokens,
                          shape.seed + 2).to(dev)
    else:
        raise ValueError(shape.bias)
    if weights:
        w_gate = torch.empty((E, f, d), dtype=dt, device=dev)
        w_up = torch.empty((E, f, d), dtype=dt, device=dev)
        w_down = torch.empty((E, d, f), dtype=dt, device=dev)
        for e in range(E):
            w_gate[e], w_up[e], w_down[e] = expert_weights(shape, e, dev)
    else:
        w_gate = w_up = w_down = None
    return MoEInputs(shape, x, w_router, bias, w_gate, w_up, w_down)


def reduced(shape: MoEShape, T: int, d: int, f: int, **kw) -> MoEShape:
    """Same routing regime (E, k, gating, capacity factor, dtype, bias kind) at a size the
    oracle finishes in seconds."""
    return shape.replace(name=f"{shape.name}_reduced_T{T}_d{d}_f{f}", T=T, d_model=d, d_ff=f,
                         **kw)
