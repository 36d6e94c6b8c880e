"""Seeded synthetic inputs for the paged-decode workloads.

This module only draws random numbers and names shapes: it holds none of the
attention, gather, slot or copy arithmetic, so the CUDA path and the CPU oracle
can both consume what it produces.

Workload shapes (sizes are those of the workloads the library is measured on):

* ``tiny``      1 layer, 4 seqs, context lens {5,16,17,40}, 4 q / 4 kv heads, head_dim 64,
                block_size 16, fp16, physical blocks drawn from a shuffled pool of 64.
* ``llama8b``   1 layer, 64 seqs, 32 q / 8 kv heads, head_dim 128, block_size 16, fp16,
                context lens uniform in [128, 2048], pool 1.2x the blocks needed.
* ``llama70b``  80 layers, 32 seqs, 64 q / 8 kv heads, head_dim 128, block_size 16, bf16,
                context lens uniform in [1000, 8000], pool 1.2x, one block table for all
                layers (327,680 KV bytes per token over the 80 layers).
* ``prefix``    16 prompts x 8 samples, 2048-token shared prefix per prompt plus 0..512
                private tokens per sample, 32 q / 8 kv heads, head_dim 128, block_size 16,
                fp16; a fork phase whose appends hit shared partial blocks.
* ``heavytail`` 256 seqs, context lens lognormal (median 512, sigma 1.2) clipped to
                [16, 32768], 32 q / 8 kv heads, head_dim 128, fp16, block_size swept over
                {1, 8, 16, 32}, fragmented placement, one 256-token append per step.

Values are N(0, 1) from ``torch.randn`` with a seeded ``torch.Generator`` on the
device that holds the tensor, rounded to fp16/bf16.  Integer draws (context lens,
pool order) use numpy's PCG64 with the workload seed, so they are identical on any
machine.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str            # "f16" or "bf16"
    layers: int
    seed: int
    pool_factor: float = 1.2
    pool_blocks: int = 0  # fixed pool size (0: pool_factor x blocks needed)


TINY = Workload("tiny", 4, 4, 4, 64, 16, "f16", 1, 0, pool_blocks=64)
LLAMA8B = Workload("llama8b", 64, 32, 8, 128, 16, "f16", 1, 1)
LLAMA70B = Workload("llama70b", 32, 64, 8, 128, 16, "bf16", 80, 2)
PREFIX = Workload("prefix", 128, 32, 8, 128, 16, "f16", 1, 3)
HEAVYTAIL = Workload("heavytail", 256, 32, 8, 128, 16, "f16", 1, 4)

WORKLOADS = {w.name: w for w in (TINY, LLAMA8B, LLAMA70B, PREFIX, HEAVYTAIL)}

PREFIX_PROMPTS = 16
PREFIX_SAMPLES = 8
PREFIX_LEN = 2048
PREFIX_PRIVATE_MAX = 512


def rng(seed: int, stream: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


def context_lens(w: Workload) -> np.ndarray:
    """Per-sequence context lengths (the newest token included), int32."""
    g = rng(w.seed, 1)
    if w.name == "tiny":
        return np.array([5, 16, 17, 40], dtype=np.int32)
    if w.name == "llama8b":
        return g.integers(128, 2048, size=w.num_seqs, endpoint=True).astype(np.int32)
    if w.name == "llama70b":
        return g.integers(1000, 8000, size=w.num_seqs, endpoint=True).astype(np.int32)
    if w.name == "heavytail":
        x = np.exp(g.normal(math.log(512.0), 1.2, size=w.num_seqs))
        return np.clip(np.rint(x), 16, 32768).astype(np.int32)
    if w.name == "prefix":
        priv = g.integers(0, PREFIX_PRIVATE_MAX, size=w.num_seqs, endpoint=True)
        return (PREFIX_LEN + priv).astype(np.int32)
    raise KeyError(w.name)


def prefix_fork_tails(w: Workload = PREFIX) -> np.ndarray:
    """Fork phase of the shared-prefix workload: per prompt, the number of tokens
    (1..15) by which its shared region runs into a partially filled block."""
    return rng(w.seed, 2).integers(1, 15, size=PREFIX_PROMPTS, endpoint=True).astype(np.int32)


def pool_order(num_blocks: int, seed: int) -> np.ndarray:
    """A seeded random permutation of the physical block ids 0..num_blocks-1: the
    order in which a fresh pool hands blocks out (fragmented placement)."""
    return rng(seed, 3).permutation(num_blocks).astype(np.int32)


def randn(shape, dtype: str, seed: int, device="cpu", stream: int = 0):
    """N(0,1) values rounded to fp16/bf16, as a torch tensor on `device`."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16 if dtype == "bf16" else torch.float16)


def randn_e4m3(shape, scale: float, seed: int, device="cpu", stream: int = 0):
    """Random 8-bit E4M3 cache codes whose values (scale * code) follow N(0, 1): N(0, 1)
    draws divided by `scale` and rounded to the nearest E4M3 code with torch's own
    float8_e4m3fn type, as uint8.  (Input data only: the library quantises with its own
    kernel.)"""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32) / scale
    x = x.clamp(-448.0, 448.0)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def torch_dtype(dtype: str):
    import torch

    return torch.bfloat16 if dtype == "bf16" else torch.float16
