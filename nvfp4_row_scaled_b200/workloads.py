"""Seeded synthetic inputs for the grouped NVFP4 cast.

This module generates inputs only: packed bf16 activations and expert
routings. It holds none of the method's arithmetic, and it is the one module
that both the CUDA path's tests/benchmark and the CPU oracle's tests use, so
both sides always see identical bytes.

The shapes follow the workloads the method is built for: packed MoE expert
activations ``(sum_M, K)`` split into expert groups whose sizes are multiples
of 128 rows (the grouped GEMM's 128-row alignment, torchtitan #14 "[NVFP4
4over6] grouped-experts four-over-six converter", Design notes; "uniform
expert sizes require 128-row alignment", TransformerEngine #3649 summary),
DeepSeek-V3-like expert counts and hidden sizes, empty experts, and routing
that lives on the device for CUDA-graph replay (TransformerEngine #3649,
Description).

All random numbers come from ``torch.Generator`` on the CPU with a fixed seed;
large tensors are drawn in fixed chunks of ``CHUNK_ROWS`` rows so the result
does not depend on available memory.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

CHUNK_ROWS = 4096
ALIGN = 128


@dataclasses.dataclass
class Workload:
    name: str
    K: int
    x: torch.Tensor                 # bf16 [capacity_rows, K], CPU unless moved
    m_splits: List[int]             # host routing; sum(m_splits) <= capacity_rows
    routings: List[List[int]]       # extra routings to replay (graph-safe config)
    description: str = ""

    @property
    def E(self) -> int:
        return len(self.m_splits)

    @property
    def sum_M(self) -> int:
        return int(sum(self.m_splits))

    @property
    def capacity_rows(self) -> int:
        return int(self.x.shape[0])

    @property
    def elements(self) -> int:
        return self.sum_M * self.K


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _chunked(rows: int, K: int, g: torch.Generator, fill) -> torch.Tensor:
    """Build a bf16 [rows, K] tensor chunk by chunk; fill(n, g) -> fp32 [n, K]."""
    out = torch.empty(rows, K, dtype=torch.bfloat16)
    for r0 in range(0, rows, CHUNK_ROWS):
        n = min(CHUNK_ROWS, rows - r0)
        out[r0:r0 + n] = fill(n, g).to(torch.bfloat16)
    return out


def zipf_weights(n: int, s: float, g: torch.Generator) -> torch.Tensor:
    """Zipf(s) popularity over n experts in a random rank order."""
    ranks = torch.randperm(n, generator=g).to(torch.float64) + 1.0
    return ranks.pow(-s)


def multinomial_counts(weights: torch.Tensor, draws: int, g: torch.Generator) -> List[int]:
    idx = torch.multinomial(weights.to(torch.float64), draws, replacement=True, generator=g)
    return torch.bincount(idx, minlength=weights.numel()).tolist()


def pad_up(m: int, a: int = ALIGN) -> int:
    return ((m + a - 1) // a) * a


# ----------------------------------------------------------------- configs

def config1() -> Workload:
    """Tiny grouped cast: 4 experts, K=512, m_splits=[128,256,0,384];
    x = N(0,1) * 2^U(-8,8) with one U per row; seed 0."""
    g = _gen(0)
    K, ms = 512, [128, 256, 0, 384]
    rows = sum(ms)
    z = torch.randn(rows, K, generator=g)
    u = torch.rand(rows, generator=g) * 16.0 - 8.0
    x = (z * torch.exp2(u)[:, None]).to(torch.bfloat16)
    return Workload("tiny_e4_k512", K, x, ms, [], "E=4 K=512 m=[128,256,0,384]")


def config2() -> Workload:
    """8 experts, K=2048, sum_M=16384 in 128-row splits from a multinomial;
    N(0,1) with 1% of rows x100 and 0.1% of rows exactly zero; seed 1."""
    g = _gen(1)
    K, E, rows = 2048, 8, 16384
    ms = [c * ALIGN for c in multinomial_counts(torch.ones(E), rows // ALIGN, g)]
    x = torch.randn(rows, K, generator=g)
    perm = torch.randperm(rows, generator=g)
    n_out, n_zero = round(0.01 * rows), round(0.001 * rows)
    x[perm[:n_out]] *= 100.0
    x[perm[n_out:n_out + n_zero]] = 0.0
    return Workload("e8_k2048_outliers", K, x.to(torch.bfloat16), ms, [],
                    "E=8 K=2048 sum_M=16384, 1% rows x100, 0.1% rows zero")


def deepseek_routing(g: torch.Generator, E: int = 256, tokens: int = 8192, topk: int = 8,
                     empty_frac: float = 0.10, zipf_s: float = 1.1):
    """Routed rows per expert for tokens*topk routed rows: a seeded ~10% of
    experts receive nothing, the rest draw from Zipf(s) popularity."""
    n_empty = round(empty_frac * E)
    perm = torch.randperm(E, generator=g)
    empty = set(perm[:n_empty].tolist())
    live = [e for e in range(E) if e not in empty]
    w = zipf_weights(len(live), zipf_s, g)
    c_live = multinomial_counts(w, tokens * topk, g)
    counts = [0] * E
    for e, c in zip(live, c_live):
        counts[e] = c
    return counts


def config3(tokens: int = 8192, align: int = ALIGN) -> Workload:
    """DeepSeek-V3-shaped MoE input: K=7168, 256 experts, 8192 tokens top-8
    (65536 routed rows), Zipf(1.1) popularity, ~10% empty experts, every group
    padded with zero rows up to a multiple of 128; routed rows are
    N(0,1) * 2^U(-4,4) per row; seed 2. ``tokens`` scales the workload down
    for small cases (same recipe); ``align`` = 16 pads groups to multiples of
    16 rows only (the unaligned-group variant)."""
    g = _gen(2)
    K, E = 7168, 256
    counts = deepseek_routing(g, E, tokens)
    ms = [pad_up(c, align) for c in counts]
    rows = sum(ms)
    routed = sum(counts)

    def fill(n, gen):
        z = torch.randn(n, K, generator=gen)
        u = torch.rand(n, generator=gen) * 8.0 - 4.0
        return z * torch.exp2(u)[:, None]

    dense = _chunked(routed, K, g, fill)
    x = torch.zeros(rows, K, dtype=torch.bfloat16)
    src, dst = 0, 0
    for c, m in zip(counts, ms):
        x[dst:dst + c] = dense[src:src + c]
        src += c
        dst += m
    name = f"deepseek_v3_e256_k7168_t{tokens}" + ("" if align == ALIGN else f"_pad{align}")
    return Workload(name, K, x, ms, [],
                    f"E=256 K=7168 {tokens} tokens top-8, Zipf(1.1), padded to {align}, sum_M={rows}")


def graphsafe_routing(seed: int, E: int, chunks: int, zipf: bool) -> List[int]:
    g = _gen(seed)
    w = zipf_weights(E, 1.1, g) if zipf else torch.ones(E, dtype=torch.float64)
    return [c * ALIGN for c in multinomial_counts(w, chunks, g)]


def config4(capacity: int = 131072) -> Workload:
    """Expert down-projection input for the graph-safe path: K=2048, 128
    experts, capacity rows; bf16 SiLU(a)*b with a, b ~ N(0,1); ten 128-aligned
    routings (seeds 100..109; 0-4 uniform, 5-9 Zipf(1.1))."""
    g = _gen(3)
    K, E = 2048, 128

    def fill(n, gen):
        a = torch.randn(n, K, generator=gen)
        b = torch.randn(n, K, generator=gen)
        return torch.nn.functional.silu(a) * b

    x = _chunked(capacity, K, g, fill)
    chunks = capacity // ALIGN
    routings = [graphsafe_routing(100 + i, E, chunks, zipf=(i >= 5)) for i in range(10)]
    return Workload(f"graphsafe_e128_k2048_cap{capacity}", K, x, routings[0], routings,
                    f"E=128 K=2048 capacity={capacity}, 10 routings")


def config5(M: int = 65536, K: int = 8192) -> Workload:
    """Single-group dense per-token cast: M x K bf16 N(0,1) * t_r with t_r a
    Student-t(3) draw per row (sign kept); seed 4."""
    g = _gen(4)

    def fill(n, gen):
        z = torch.randn(n, K, generator=gen)
        w = torch.randn(n, 4, generator=gen)
        t = w[:, 0] / torch.sqrt((w[:, 1:] ** 2).sum(dim=1) / 3.0)
        return z * t[:, None]

    x = _chunked(M, K, g, fill)
    return Workload(f"dense_m{M}_k{K}", K, x, [M], [], f"E=1 M={M} K={K}, Student-t(3) row scales")


CONFIGS = {1: config1, 2: config2, 3: config3, 4: config4, 5: config5}


def make(config_id: int, **kw) -> Workload:
    return CONFIGS[config_id](**kw)


# ------------------------------------------------------- small random cases

def random_case(seed: int, K: int, m_splits: List[int], capacity: Optional[int] = None,
                dist: str = "normal") -> Workload:
    """A small seeded case with the given splits (used by parity tests)."""
    g = _gen(seed)
    rows = sum(m_splits)
    cap = rows if capacity is None else capacity
    z = torch.randn(cap, K, generator=g)
    if dist == "wide":
        u = torch.rand(cap, generator=g) * 40.0 - 20.0
        z = z * torch.exp2(u)[:, None]
    elif dist == "heavy":
        w = torch.randn(cap, 4, generator=g)
        t = w[:, 0] / torch.sqrt((w[:, 1:] ** 2).sum(dim=1) / 3.0)
        z = z * t[:, None]
    x = z.to(torch.bfloat16)
    return Workload(f"case{seed}_k{K}", K, x, list(m_splits), [], "random case")


def bits(x: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (CPU)."""
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def row_offsets(m_splits: List[int]) -> List[int]:
    out = [0]
    for m in m_splits:
        out.append(out[-1] + int(m))
    return out


def tensor_offsets(m_splits: List[int], K: int) -> List[int]:
    """Element offsets (row offset * K) of each group, length E+1."""
    return [o * K for o in row_offsets(m_splits)]


def elements_of(m_splits: List[int], K: int) -> int:
    return int(sum(m_splits)) * K
