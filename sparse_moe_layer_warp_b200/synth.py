"""Seeded synthetic inputs for the sparse-MoE layer (shapes and distributions only).

This module holds none of the layer's arithmetic: it draws random tensors of the right
shapes and distributions and is the one module that both the CUDA path's callers and the
CPU oracle's callers share.

Workloads (all synthetic; no dataset or trained weights are involved):

=================  =====  =====  ===  ==  =====  ======================================
name               T      d      E    k   f      notes
=================  =====  =====  ===  ==  =====  ======================================
tiny_fp32          64     256    16   2   64     fp32 everything
decode_t16         16     4096   288  8   1280   bf16; 4 sequences x 4 MTP-3 positions
decode_t256        256    4096   288  8   1280   bf16; batched decode
prefill_t8192      8192   4096   288  8   1280   bf16; prefill chunk
skew_t4096         4096   4096   288  8   1280   bf16; Zipf(1.1)-skewed expert selection
prefill_e32_t1024  1024   4096   32   8   1280   bf16; profiler-sized prefill-like case
prefill_e128_t4096 4096   4096   128  8   1280   bf16; same, with a wave of shared-expert units
decode_e32_t16     16     4096   32   8   1280   bf16; profiler-sized decode-like case
dense_ffn_t4096    4096   4096   1    1   11264  bf16; dense SwiGLU FFN, no shared expert
=================  =====  =====  ===  ==  =====  ======================================

Every workload has one shared expert with the routed experts' hidden size.  Distributions:
x ~ N(0, 1); every weight ~ N(0, 1/fan_in) (fan_in = d for W_r, W_gate, W_up; f for W_down);
router bias ~ U(-0.1, 0.1).  For ``skew_t4096`` the bias is b_e = -s * ln(rank_e) with
s = 1.1 and rank_e the 1-based position of expert e in a seeded random permutation, so that
exp(b_e) follows Zipf(1.1) over the permuted experts.  Tensors are drawn in the order
x, W_r, b, W_gate, W_up, W_down from one ``torch.Generator`` seeded with the workload's seed;
the routed experts' and the shared expert's matrices are one tensor each (shared = last),
drawn expert by expert.  bf16 tensors are the RNE rounding of the fp32 draws.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    n_shared: int = 1
    dtype: str = "bf16"  # "bf16" or "f32"
    seed: int = 0
    bias: str = "uniform"  # "uniform" or "zipf"
    routed_scale: float = 1.0

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", T=64, d=256, E=16, k=2, f=64, dtype="f32"),
    "decode_t16": Workload("decode_t16", T=16, d=4096, E=288, k=8, f=1280),
    "decode_t256": Workload("decode_t256", T=256, d=4096, E=288, k=8, f=1280),
    "prefill_t8192": Workload("prefill_t8192", T=8192, d=4096, E=288, k=8, f=1280),
    "skew_t4096": Workload("skew_t4096", T=4096, d=4096, E=288, k=8, f=1280, bias="zipf"),
    # small case with prefill's per-expert load (~256 tokens per expert) and full-size
    # expert matrices, ~1 GB of weights: for profiler captures that must stay small
    "prefill_e32_t1024": Workload("prefill_e32_t1024", T=1024, d=4096, E=32, k=8, f=1280),
    # the same per-expert load with enough tokens (80 shared-expert up units, more than the
    # 74 CTA pairs) that the CTA-pair up GEMM writes the sorted copy of x itself; ~4 GB of
    # weights
    "prefill_e128_t4096": Workload("prefill_e128_t4096", T=4096, d=4096, E=128, k=8, f=1280),
    # small case with decode's per-expert load (~4 tokens per expert, the same 16-token tiles
    # with rows gathered by TMA) and full-size expert matrices, ~1 GB of weights
    "decode_e32_t16": Workload("decode_e32_t16", T=16, d=4096, E=32, k=8, f=1280),
    # dense SwiGLU FFN of the first layers / MTP heads (hidden 11264): one expert, k = 1, no
    # shared expert, so every token's gate is exactly 1
    "dense_ffn_t4096": Workload("dense_ffn_t4096", T=4096, d=4096, E=1, k=1, f=11264,
                                n_shared=0),
}


@dataclasses.dataclass
class LayerInputs:
    w: Workload
    x: torch.Tensor          # [T, d]
    w_router: torch.Tensor   # [E, d]
    bias: torch.Tensor       # [E] fp32
    w_gate: torch.Tensor     # [E + n_shared, f, d]
    w_up: torch.Tensor       # [E + n_shared, f, d]
    w_down: torch.Tensor     # [E + n_shared, d, f]


def _normal(gen, shape, std, device, dtype):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _expert_stack(gen, n, rows, cols, std, device, dtype):
    out = torch.empty((n, rows, cols), device=device, dtype=dtype)
    for e in range(n):  # expert by expert keeps the fp32 temporary small
        out[e] = _normal(gen, (rows, cols), std, device, dtype)
    return out


def make_bias(w: Workload, gen, device) -> torch.Tensor:
    if w.bias == "uniform":
        return (torch.rand((w.E,), generator=gen, device=device, dtype=torch.float32) * 0.2 - 0.1)
    if w.bias == "zipf":
        order = torch.randperm(w.E, generator=gen, device=device)
        rank = torch.empty(w.E, device=device, dtype=torch.float32)
        rank[order] = torch.arange(1, w.E + 1, device=device, dtype=torch.float32)
        return -1.1 * torch.log(rank)
    raise ValueError(w.bias)


def make_inputs(w: Workload, device="cpu", T: int | None = None) -> LayerInputs:
    """Draw one workload's inputs on `device` (a CUDA device for the full-size workloads)."""
    T = w.T if T is None else T
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    G = w.E + w.n_shared
    x = _normal(gen, (T, w.d), 1.0, device, dt)
    w_router = _normal(gen, (w.E, w.d), 1.0 / math.sqrt(w.d), device, dt)
    bias = make_bias(w, gen, device)
    w_gate = _expert_stack(gen, G, w.f, w.d, 1.0 / math.sqrt(w.d), device, dt)
    w_up = _expert_stack(gen, G, w.f, w.d, 1.0 / math.sqrt(w.d), device, dt)
    w_down = _expert_stack(gen, G, w.d, w.f, 1.0 / math.sqrt(w.f), device, dt)
    return LayerInputs(w, x, w_router, bias, w_gate, w_up, w_down)


def make_x(w: Workload, T: int, device="cpu", seed: int | None = None) -> torch.Tensor:
    """Fresh activations only (used to vary the batch between steps)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    return _normal(gen, (T, w.d), 1.0, device, w.torch_dtype)


def make_logits(T: int, E: int, seed: int = 0, ties: bool = False, device="cpu") -> torch.Tensor:
    """Synthetic fp32 router logits ~ N(0, 1); with `ties`, values are drawn from a coarse
    grid (multiples of 1/8 in [-2, 2]) so that many scores are exactly equal."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    if ties:
        return (torch.randint(-16, 17, (T, E), generator=gen, device=device).float() / 8.0)
    return torch.randn((T, E), generator=gen, device=device, dtype=torch.float32)


def to_numpy_bits(t: torch.Tensor):
    """Host NumPy view for the oracle: bf16 -> uint16 bit patterns, fp32 -> float32."""
    import numpy as np

    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
