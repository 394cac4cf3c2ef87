"""Seeded synthetic inputs for the BCQ LUT-GEMM path.

This module is shared by the oracle side and the CUDA side of the tests and the
benchmark. It only draws random numbers: it holds none of the method's
arithmetic (no packing, no tables, no dequantisation). Every draw uses a CPU
``torch.Generator`` seeded by the caller, so both sides see identical bytes.

Shapes follow the workloads of the LUT-GEMM paper card (Park et al.,
"LUT-GEMM: Quantized Matrix Multiplication based on LUTs for Efficient
Inference in Large-Scale Generative Language Models", Key points: OPT-175B and
LLaMA layer shapes, 3-bit weights, g = 128). The pages ship no weights, so the
values are random stand-ins with the stated distributions.

Layout conventions used everywhere in this repository:

* signs   int8  [q][m][n]      each element -1 or +1 (plane i, output row j, input k)
* alpha   fp16  [q][n/g][m]    group-major scales (plane, group, row)
* codes   uint8 [m][n]         uniform integer codes in [0, 2^q)
* scale   fp16  [n/g][m]       uniform scale s per (group, row)
* zero    uint8 [n/g][m]       uniform integer zero-point z per (group, row)
* x       fp16  [batch][n]     activations
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = [
    "generator",
    "draw_signs",
    "draw_random_bytes",
    "draw_alpha",
    "draw_uniform",
    "draw_x",
    "draw_weights",
    "draw_block_planes",
    "draw_outliers",
    "Shape",
    "WORKLOADS",
]


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def draw_signs(gen: torch.Generator, q: int, m: int, n: int) -> torch.Tensor:
    """Uniform random {-1,+1} int8 tensor [q][m][n]."""
    bits = torch.randint(0, 2, (q, m, n), generator=gen, dtype=torch.int8)
    return bits * 2 - 1


def draw_random_bytes(gen: torch.Generator, nbytes: int) -> torch.Tensor:
    """``nbytes`` uniform random bytes (uint8).

    Uniform random bytes are uniform random bits whatever order a consumer
    reads them in, so a packed weight buffer of uniform random +-1 bits can be
    drawn directly without materialising the int8 sign tensor.
    """
    return torch.randint(0, 256, (int(nbytes),), generator=gen, dtype=torch.uint8)


def draw_alpha(gen: torch.Generator, q: int, m: int, n: int, g: int, sigma: float,
               sort_desc: bool = True) -> torch.Tensor:
    """|N(0, sigma)| scales as fp16 [q][n/g][m], optionally sorted descending over planes."""
    ng = n // g
    a = torch.randn((q, ng, m), generator=gen, dtype=torch.float32).mul_(sigma).abs_()
    if sort_desc and q > 1:
        a = torch.sort(a, dim=0, descending=True).values
    return a.to(torch.float16).contiguous()


def draw_uniform(gen: torch.Generator, m: int, n: int, g: int, q: int, s_sigma: float):
    """Uniform-quantiser inputs: codes [m][n], scale [n/g][m] fp16, zero [n/g][m]."""
    ng = n // g
    top = 1 << q
    codes = torch.randint(0, top, (m, n), generator=gen, dtype=torch.uint8)
    scale = torch.randn((ng, m), generator=gen, dtype=torch.float32).mul_(s_sigma).abs_()
    scale = scale.to(torch.float16).contiguous()
    zero = torch.randint(0, top, (ng, m), generator=gen, dtype=torch.uint8)
    return codes, scale, zero


def draw_weights(gen: torch.Generator, m: int, n: int, sigma: float) -> torch.Tensor:
    """Dense FP16 weights W ~ N(0, sigma) [m][n] (the input of BCQ fitting)."""
    w = torch.randn((m, n), generator=gen, dtype=torch.float32).mul_(sigma)
    return w.to(torch.float16).contiguous()


def draw_x(gen: torch.Generator, batch: int, n: int, outlier_frac: float = 0.0,
           outlier_scale: float = 20.0) -> torch.Tensor:
    """x ~ N(0,1) fp16 [batch][n]; optionally ceil(frac*n) shared columns scaled."""
    x = torch.randn((batch, n), generator=gen, dtype=torch.float32)
    if outlier_frac > 0.0:
        k = int(math.ceil(outlier_frac * n))
        idx = torch.randperm(n, generator=gen)[:k]
        x[:, idx] *= outlier_scale
    return x.to(torch.float16).contiguous()


def draw_block_planes(gen: torch.Generator, m: int, n: int, frac_hi: float, lo: int = 2,
                      hi: int = 4) -> torch.Tensor:
    """Plane count of every (1024-input slice, 32-row tile) block, uint8
    [ceil(n/1024)][ceil(m/32)]: `hi` with probability frac_hi, else `lo`."""
    ns, mt = -(-n // 1024), -(-m // 32)
    u = torch.rand((ns, mt), generator=gen)
    return torch.where(u < frac_hi, hi, lo).to(torch.uint8).contiguous()


def draw_outliers(gen: torch.Generator, m: int, n: int, density: float, sigma: float = 0.1):
    """Sparse fp16 outlier weights ~ N(0, sigma) at round(density*m*n)
    positions drawn without replacement, as row CSR: (row_ptr int32 [m+1],
    col int32 [nnz] increasing within a row, val fp16 [nnz])."""
    nnz = int(round(density * m * n))
    flat = torch.randperm(m * n, generator=gen)[:nnz].sort().values
    rows, cols = flat // n, flat % n
    val = (torch.randn(nnz, generator=gen) * sigma).to(torch.float16)
    row_ptr = torch.zeros(m + 1, dtype=torch.int64)
    row_ptr[1:] = torch.bincount(rows, minlength=m).cumsum(0)
    return row_ptr.to(torch.int32), cols.to(torch.int32), val


@dataclass(frozen=True)
class Shape:
    """One matmul of a workload: m outputs, n inputs."""
    name: str
    m: int
    n: int


@dataclass(frozen=True)
class Workload:
    key: str
    description: str
    shapes: tuple
    q: tuple
    g: int
    alpha_sigma: float
    batches: tuple
    seed: int
    uniform: bool = False
    s_sigma: float = 0.0
    outlier_frac: float = 0.0
    extra: dict = field(default_factory=dict)


# The five workloads, in the order the task lists them.  Seeds 0..4.
WORKLOADS = {
    "tiny": Workload(
        key="tiny", description="Tiny BCQ GEMV m=n=512, q=3, g=128, batch 1",
        shapes=(Shape("tiny", 512, 512),), q=(3,), g=128, alpha_sigma=0.02,
        batches=(1,), seed=0),
    "uniform4": Workload(
        key="uniform4", description="Uniform 4-bit rewritten as BCQ, m=n=5120, g=128, batch 1",
        shapes=(Shape("sq5120", 5120, 5120),), q=(4,), g=128, alpha_sigma=0.0,
        batches=(1,), seed=1, uniform=True, s_sigma=0.01),
    "opt175b_ffn": Workload(
        key="opt175b_ffn", description="OPT-175B FFN FC1 49152x12288 and FC2 12288x49152, q=3, g=128",
        shapes=(Shape("fc1", 49152, 12288), Shape("fc2", 12288, 49152)), q=(3,), g=128,
        alpha_sigma=0.02, batches=(1,), seed=2),
    "llama70b": Workload(
        key="llama70b", description="LLaMA-70B layers q=2, g=64, 0.1% outlier columns x20",
        shapes=(Shape("attn", 8192, 8192), Shape("up", 28672, 8192), Shape("down", 8192, 28672)),
        q=(2,), g=64, alpha_sigma=0.03, batches=(1, 2, 4, 8), seed=3, outlier_frac=0.001),
    "opt175b_layer": Workload(
        key="opt175b_layer", description="OPT-175B decoder-layer linears QKV/out/FC1/FC2, g=128",
        shapes=(Shape("qkv", 36864, 12288), Shape("out", 12288, 12288),
                Shape("fc1", 49152, 12288), Shape("fc2", 12288, 49152)),
        q=(2, 3, 4), g=128, alpha_sigma=0.02, batches=(1, 4, 16, 32), seed=4),
}
