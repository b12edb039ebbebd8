"""Seeded synthetic workloads shared by the CUDA path's tests/bench and the CPU oracle.

This module only draws random numbers and names shapes. It holds none of the
attention arithmetic, so neither side of a parity comparison can borrow the
other's math through it.

Workloads (shapes, dtypes, seeds) stand in for the long-context runs that the
RingAttention pages describe (deep-architecture article, section 6 benchmark
table: 128k..10M tokens; newsletter page: 1M+ tokens). The pages give no data
distribution, so every tensor is i.i.d. N(0, 1), drawn in fp32 and rounded to
the workload dtype with round-to-nearest-even (torch ``.to``).

Generator recipe:
  * ``torch.Generator(device).manual_seed(seed)``; draws in the order q, k, v,
    each ``torch.randn(shape, dtype=float32)`` on that device, then ``.to(dtype)``.
  * The heavy-key variant (GQA workload) then, per (batch, kv-head), draws
    ``torch.randperm(S)`` from the same generator and multiplies the first
    floor(0.01*S) key rows by 4 in fp32 before the cast.
  * Small workloads are drawn on the CPU generator (bit-identical on every
    machine). The 131k- and 1M-token workloads are drawn on the CUDA generator of
    the device that runs them (drawing 3.2e9 normals on the CPU takes minutes);
    the oracle then reads a host copy of exactly those device tensors.
  * Sampled query rows: ``torch.Generator().manual_seed(seed + 1000)``,
    ``randperm(B*Hq*S)[:n]`` over flat (b, h, t) indices, plus t=0, t=S-1 and the
    first and last token of every shard for (b=0, h=0).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterable

import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_inputs", "make_dout", "make_decode_query", "sample_rows", "shard_boundary_rows"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str          # "fp32" | "bf16"
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    P: int
    causal: bool
    layout: str         # "contiguous" | "striped" | "zigzag"
    seed: int
    heavy_keys: bool = False
    gen_device: str = "cpu"   # "cpu" or "cuda": where the seeded draw happens
    description: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"fp32": torch.float32, "bf16": torch.bfloat16}[self.dtype]

    @property
    def Sq(self) -> int:
        return self.S // self.P

    def causal_flops(self) -> float:
        """4*B*Hq*S^2*D, halved when causal (QK^T and PV, 2 FLOPs per MAC)."""
        f = 4.0 * self.B * self.Hq * float(self.S) ** 2 * self.D
        return f * 0.5 if self.causal else f

    def exact_pair_count(self) -> int:
        """Number of (query, key) pairs that enter the softmax."""
        per_head = self.S * (self.S + 1) // 2 if self.causal else self.S * self.S
        return self.B * self.Hq * per_head

    def algorithmic_flops(self) -> float:
        """4*D FLOPs per allowed (query, key) pair (inclusive causal diagonal)."""
        return 4.0 * self.D * self.exact_pair_count()

    def qkvo_bytes(self) -> int:
        esz = 4 if self.dtype == "fp32" else 2
        q = self.B * self.Hq * self.S * self.D * esz
        kv = 2 * self.B * self.Hkv * self.S * self.D * esz
        lse = self.B * self.Hq * self.S * 4
        return 2 * q + kv + lse


WORKLOADS = {
    "c1_fp32_s1k": Workload("c1_fp32_s1k", "fp32", 1, 2, 2, 1024, 64, 4, False, "contiguous", 0,
                            description="fp32 S=1024 D=64 P=4 non-causal contiguous"),
    "c2_bf16_s16k_contig": Workload("c2_bf16_s16k_contig", "bf16", 1, 8, 8, 16384, 128, 8, True,
                                    "contiguous", 1,
                                    description="bf16 S=16384 P=8 causal contiguous (unbalanced ring)"),
    "c3_bf16_s16k_striped": Workload("c3_bf16_s16k_striped", "bf16", 1, 8, 8, 16384, 128, 8, True,
                                     "striped", 2, description="bf16 S=16384 P=8 causal striped"),
    "c4_bf16_gqa_s128k": Workload("c4_bf16_gqa_s128k", "bf16", 2, 32, 8, 131072, 128, 16, True,
                                  "striped", 3, heavy_keys=True, gen_device="cuda",
                                  description="bf16 GQA B=2 Hq=32 Hkv=8 S=131072 P=16 causal striped, "
                                              "1% heavy keys x4"),
    "c5_bf16_s1m_striped": Workload("c5_bf16_s1m_striped", "bf16", 1, 8, 8, 1048576, 128, 32, True,
                                    "striped", 4, gen_device="cuda",
                                    description="bf16 S=1048576 P=32 causal striped"),
    # the 1M workload's shape under the zigzag layout (chunks of 16384 tokens)
    "z5_bf16_s1m_zigzag": Workload("z5_bf16_s1m_zigzag", "bf16", 1, 8, 8, 1048576, 128, 32, True,
                                   "zigzag", 7, gen_device="cuda",
                                   description="bf16 S=1048576 P=32 causal zigzag"),
    # head dim 64 (the single-CTA tensor-core kernel), same token count and FLOPs as the 128k case
    "d64_bf16_s128k_striped": Workload("d64_bf16_s128k_striped", "bf16", 1, 16, 16, 131072, 64, 32, True,
                                       "striped", 8, gen_device="cuda",
                                       description="bf16 S=131072 Hq=16 D=64 P=32 causal striped"),
    # profiling stand-in: the 1M workload's shape at 1/8 the length (inputs 0.4 GB > L2,
    # ~45 ms per launch) so an ncu capture of every section ends in a minute or two
    "prof_bf16_s128k_striped": Workload("prof_bf16_s128k_striped", "bf16", 1, 8, 8, 131072, 128, 32, True,
                                        "striped", 5, gen_device="cuda",
                                        description="bf16 S=131072 P=32 causal striped (profiling case)"),
    # twice the length: with the 128k case it shows whether DRAM traffic grows with the work
    "prof_bf16_s256k_striped": Workload("prof_bf16_s256k_striped", "bf16", 1, 8, 8, 262144, 128, 32, True,
                                        "striped", 6, gen_device="cuda",
                                        description="bf16 S=262144 P=32 causal striped (profiling case)"),
    # the 128k profiling case in the contiguous layout (a shard's rows are adjacent in memory)
    "prof_bf16_s128k_contig": Workload("prof_bf16_s128k_contig", "bf16", 1, 8, 8, 131072, 128, 32, True,
                                       "contiguous", 10, gen_device="cuda",
                                       description="bf16 S=131072 P=32 causal contiguous (profiling case)"),
    "prof_bf16_s512k_striped": Workload("prof_bf16_s512k_striped", "bf16", 1, 8, 8, 524288, 128, 32, True,
                                        "striped", 9, gen_device="cuda",
                                        description="bf16 S=524288 P=32 causal striped (profiling case)"),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def custom(name: str, dtype: str, B: int, Hq: int, Hkv: int, S: int, D: int, P: int,
           causal: bool, layout: str, seed: int, heavy_keys: bool = False,
           gen_device: str = "cpu") -> Workload:
    """A workload outside the fixed table (parity sweeps, small cases)."""
    return Workload(name, dtype, B, Hq, Hkv, S, D, P, causal, layout, seed, heavy_keys, gen_device)


def make_inputs(w: Workload, device: str | torch.device | None = None):
    """Draw (q, k, v) for workload ``w`` following the module recipe.

    ``device`` is where the draw happens and the tensors live; by default the
    workload's own ``gen_device``. Returns contiguous tensors
    q [B,Hq,S,D], k/v [B,Hkv,S,D] in the workload dtype.
    """
    dev = torch.device(device if device is not None else w.gen_device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed)
    f32 = torch.float32
    q = torch.randn((w.B, w.Hq, w.S, w.D), generator=g, dtype=f32, device=dev)
    k = torch.randn((w.B, w.Hkv, w.S, w.D), generator=g, dtype=f32, device=dev)
    v = torch.randn((w.B, w.Hkv, w.S, w.D), generator=g, dtype=f32, device=dev)
    if w.heavy_keys:
        n_heavy = int(math.floor(0.01 * w.S))
        for b in range(w.B):
            for gh in range(w.Hkv):
                idx = torch.randperm(w.S, generator=g, device=dev)[:n_heavy]
                k[b, gh, idx, :] *= 4.0
    dt = w.torch_dtype
    return q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous()


def make_dout(w: Workload, device: str | torch.device | None = None) -> torch.Tensor:
    """The output gradient for backward tests: i.i.d. N(0, 1) drawn in fp32 with seed
    w.seed + 500 on ``device`` (default: the workload's gen_device), shaped like q and
    rounded to the workload dtype."""
    dev = torch.device(device if device is not None else w.gen_device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 500)
    d = torch.randn((w.B, w.Hq, w.S, w.D), generator=gen, device=dev, dtype=torch.float32)
    return d.to(w.torch_dtype).contiguous()


def make_decode_query(w: Workload, device: str | torch.device | None = None) -> torch.Tensor:
    """One new query row per head for a decode step against the workload's K/V cache:
    i.i.d. N(0, 1) drawn in fp32 with seed w.seed + 700, shape [B, Hq, D], rounded to
    the workload dtype."""
    dev = torch.device(device if device is not None else w.gen_device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + 700)
    q1 = torch.randn((w.B, w.Hq, w.D), generator=gen, device=dev, dtype=torch.float32)
    return q1.to(w.torch_dtype).contiguous()


def shard_boundary_rows(w: Workload) -> list[tuple[int, int, int]]:
    """(b=0, h=0, t) for t=0, t=S-1 and the first/last token of every shard."""
    ts = {0, w.S - 1}
    Sq = w.Sq
    for i in range(w.P):
        if w.layout == "contiguous":
            ts.add(i * Sq)
            ts.add(i * Sq + Sq - 1)
        elif w.layout == "zigzag":  # shard i holds chunks i and 2P-1-i of C = Sq/2 tokens
            C = Sq // 2
            for c in (i, 2 * w.P - 1 - i):
                ts.add(c * C)
                ts.add(c * C + C - 1)
        else:  # striped: shard i holds tokens a*P + i
            ts.add(i)
            ts.add((Sq - 1) * w.P + i)
    return [(0, 0, t) for t in sorted(ts)]


def sample_rows(w: Workload, n: int = 4096, extra: Iterable[tuple[int, int, int]] | None = None
                ) -> list[tuple[int, int, int]]:
    """Seeded distinct (b, h, t) query rows plus the boundary rows, sorted."""
    g = torch.Generator()
    g.manual_seed(w.seed + 1000)
    total = w.B * w.Hq * w.S
    n = min(n, total)
    flat = torch.randperm(total, generator=g)[:n].tolist()
    rows = set()
    for f in flat:
        b, rem = divmod(f, w.Hq * w.S)
        h, t = divmod(rem, w.S)
        rows.add((b, h, t))
    rows.update(shard_boundary_rows(w))
    if extra:
        rows.update(extra)
    return sorted(rows)
