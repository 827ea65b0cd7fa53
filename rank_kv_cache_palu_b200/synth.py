"""Seeded synthetic inputs for the latent-KV decode path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no projection, RoPE, softmax or quantisation).  Both the
CUDA path (through the tests and the bench) and the CPU oracle read the tensors
it returns, so both sides see the same bytes.

Every draw is keyed by ``(seed, tag, *unit)`` through numpy's SeedSequence and
the counter-based Philox generator, so one (sequence, group) unit can be
regenerated on its own without drawing the others.  That is what lets a test
check sampled units of a full-size workload against the oracle.

Distributions follow the workloads named for the method's decode step:
latents ~ N(0, 1) (the distribution of x·A for x ~ N(0, 1) of width d_model
and A ~ N(0, 1/d_model)), B ~ N(0, 1/r) (fan-in scaling), q ~ N(0, 1),
x ~ N(0, 1).  Values are rounded to the storage dtype by torch's own
conversion, so they are exactly representable in that dtype.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "TORCH_DTYPE",
    "Workload",
    "WORKLOADS",
    "normal",
    "normal_tensor",
    "page_permutation",
    "int_positions",
]

# Storage dtype names used across the library and the tests.
TORCH_DTYPE = {
    "f32": torch.float32,
    "f16": torch.float16,
    "bf16": torch.bfloat16,
}


def _key(seed: int, tag: str, unit: tuple[int, ...]) -> list[int]:
    return [int(seed), zlib.crc32(tag.encode()), *[int(u) for u in unit]]


def normal(seed: int, tag: str, shape, std: float = 1.0, unit: tuple[int, ...] = ()) -> np.ndarray:
    """N(0, std^2) float32 samples keyed by (seed, tag, unit)."""
    rng = np.random.Generator(np.random.Philox(np.random.SeedSequence(_key(seed, tag, unit))))
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def normal_tensor(seed: int, tag: str, shape, dtype: str, std: float = 1.0,
                  unit: tuple[int, ...] = ()) -> torch.Tensor:
    """CPU tensor of N(0, std^2) samples, converted to the storage dtype."""
    return torch.from_numpy(normal(seed, tag, shape, std, unit)).to(TORCH_DTYPE[dtype])


def page_permutation(seed: int, num_pages: int) -> np.ndarray:
    """A seeded shuffle of page indices, so that logical pages land out of order."""
    rng = np.random.Generator(np.random.Philox(np.random.SeedSequence(_key(seed, "pages", ()))))
    return rng.permutation(num_pages).astype(np.int32)


def int_positions(seed: int, tag: str, n: int, low: int, high: int) -> np.ndarray:
    """Seeded integer positions in [low, high)."""
    rng = np.random.Generator(np.random.Philox(np.random.SeedSequence(_key(seed, tag, ()))))
    return rng.integers(low, high, size=n, dtype=np.int64).astype(np.int32)


@dataclass(frozen=True)
class Workload:
    """One decode-step workload: the model shape, ranks, dtypes and batch/context."""

    name: str
    num_heads: int
    head_dim: int
    group_size: int
    rank_k: int
    rank_v: int
    batch: int
    context: int
    act_dtype: str          # q, x, A, B and the output
    latent_dtype: str       # cache storage: f32 | f16 | bf16 | int4
    rope_base: float = 10000.0
    page_size: int = 128
    d_model: int = 4096
    seed: int = 0
    # per-group ranks (a rank-search output); empty = rank_k / rank_v for every group
    ranks_k: tuple = ()
    ranks_v: tuple = ()
    notes: str = field(default="", compare=False)

    @property
    def groups(self) -> int:
        return self.num_heads // self.group_size

    @property
    def ranked(self) -> bool:
        return bool(self.ranks_k)

    @property
    def group_ranks(self) -> tuple[tuple, tuple]:
        """(key ranks, value ranks) of every group."""
        if self.ranks_k:
            return tuple(self.ranks_k), tuple(self.ranks_v)
        return (self.rank_k,) * self.groups, (self.rank_v,) * self.groups

    @property
    def width(self) -> int:
        return self.group_size * self.head_dim


def _w(name, **kw) -> Workload:
    return Workload(name=name, **kw)


# The workloads of the decode hot path.  "tiny" is the fp32 oracle case; the
# others are Llama-2-7B-shaped attention layers (32 heads of 128, 8 groups of 4
# heads, d_model 4096).
WORKLOADS = {
    w.name: w
    for w in [
        _w("tiny_f32", num_heads=8, head_dim=64, group_size=4, rank_k=64, rank_v=64,
           batch=1, context=256, act_dtype="f32", latent_dtype="f32", d_model=256, seed=0),
        _w("7b_f16_r256_b1_t4k", num_heads=32, head_dim=128, group_size=4, rank_k=256,
           rank_v=256, batch=1, context=4096, act_dtype="f16", latent_dtype="f16", seed=2),
        # the bf16 context sweep: context 4k / 16k / 64k x batch 1 / 8 / 16, key rank 256,
        # value rank 128
        *[_w(f"7b_bf16_r256v128_b{b}_t{t // 1024}k", num_heads=32, head_dim=128, group_size=4,
             rank_k=256, rank_v=128, batch=b, context=t, act_dtype="bf16", latent_dtype="bf16", seed=3)
          for t in (4096, 16384, 65536) for b in (1, 8, 16)],
        _w("7b_int4_r256_b8_t32k", num_heads=32, head_dim=128, group_size=4, rank_k=256,
           rank_v=256, batch=8, context=32768, act_dtype="f16", latent_dtype="int4", seed=4),
        _w("7b_bf16_r256_b32_t16k", num_heads=32, head_dim=128, group_size=4, rank_k=256,
           rank_v=256, batch=32, context=16384, act_dtype="bf16", latent_dtype="bf16", seed=5),
        # the same layer with one short sequence: a small case whose prefill (bench --prefill)
        # is the batch-32 workload's GEMM, for captures that must stay small on the device
        _w("7b_bf16_r256_b1_t4k", num_heads=32, head_dim=128, group_size=4, rank_k=256,
           rank_v=256, batch=1, context=4096, act_dtype="bf16", latent_dtype="bf16", seed=5),
        # attention without RoPE: the key up-projection folds into the query
        # (the fused, latent-space path)
        _w("7b_bf16_r256v128_b16_t16k_norope", num_heads=32, head_dim=128, group_size=4,
           rank_k=256, rank_v=128, batch=16, context=16384, act_dtype="bf16",
           latent_dtype="bf16", rope_base=0.0, seed=6),
        # a rank-search output: the 8 groups keep different key / value ranks
        # (mean key rank 208, value ranks 128 and 256), all on the tcgen05 path;
        # rank_k / rank_v name the largest
        _w("7b_bf16_ranked_b16_t16k", num_heads=32, head_dim=128, group_size=4, rank_k=256,
           rank_v=256, batch=16, context=16384, act_dtype="bf16", latent_dtype="bf16", seed=7,
           ranks_k=(128, 192, 256, 256, 128, 192, 256, 256),
           ranks_v=(128, 128, 128, 256, 128, 128, 128, 256)),
        _w("7b_bf16_ranked_b16_t16k_norope", num_heads=32, head_dim=128, group_size=4, rank_k=320,
           rank_v=256, batch=16, context=16384, act_dtype="bf16", latent_dtype="bf16", rope_base=0.0,
           seed=8, ranks_k=(128, 192, 256, 320, 128, 192, 256, 192),
           ranks_v=(128, 128, 128, 256, 128, 128, 128, 256)),
    ]
}
