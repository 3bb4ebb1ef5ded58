"""Seeded synthetic inputs for the routed-expert MoE prefill layer.

This module only draws random numbers and lays them out in the byte formats
the layer consumes.  It holds none of the layer's arithmetic (no decoding, no
routing, no matrix products) so that both the CUDA path and the float64
oracle can be fed from it without sharing any of the method.

Workloads (the shapes of the Red Lite dev72 page, section 4 "GPU profiling
with Xcode", second profile: 2,048 tokens, 512 experts, 20,480 pairs, and the
stand-in block formats Q1/Q2 that replace the IQ1_M / IQ2_XS grids the pages
do not give):

=====  ===================  =====  =====  ====  ====  ==  ======  =====
index  name                 T      H      I     E     k   format  skew
=====  ===================  =====  =====  ====  ====  ==  ======  =====
0      tiny                 64     256    128   16    2   Q2      no
1      verify2              2      2048   512   512   10  Q2      no
2      chunk512             512    2048   512   512   10  Q2      no
3      chunk2048_q2         2048   2048   512   512   10  Q2      no
4      chunk2048_q1_skew    2048   2048   512   512   10  Q1      yes
=====  ===================  =====  =====  ====  ====  ==  ======  =====

Value distributions:

* x: float32 N(0,1) rounded to bf16 (round to nearest even), returned as the
  uint16 bit patterns, row-major [T, H].
* router logits: float32 N(0,1), row-major [T, E].  With ``skew`` a
  per-expert bias 1.5*ln(1/rank) is added in float64 (rank 1..E from a seeded
  random permutation) and the sum rounded to float32 (Zipf-like expert load).
* blocks (256 values along K each):
  - Q2, 69 bytes: bytes 0-1 fp16 d (little endian), bytes 2-4 eight 3-bit
    sub-scales as one 24-bit little-endian integer, bytes 5-68 sixty-four bytes
    of 2-bit codes;
  - Q1, 38 bytes: bytes 0-1 fp16 d, bytes 2-4 sub-scales, byte 5 eight shift
    flags, bytes 6-37 thirty-two bytes of 1-bit codes.
  d = fp16(float32(0.01*(0.5+U[0,1)))); every other bit is uniform.
* expert blob: gate [I rows] then up [I rows] then down [H rows]; a row of a
  matrix with K columns is ceil(K/256) consecutive blocks.  All experts sit in
  one buffer at a stride rounded up to 256 bytes.
"""
from __future__ import annotations

import dataclasses

import numpy as np

FMT_Q1 = 1
FMT_Q2 = 2
BLOCK_VALUES = 256
BLOCK_BYTES = {FMT_Q1: 38, FMT_Q2: 69}
FMT_NAMES = {FMT_Q1: "Q1", FMT_Q2: "Q2"}
EXPERT_ALIGN = 256
BASE_SEED = 20261202


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    fmt: int
    skew: bool = False

    @property
    def pairs(self) -> int:
        return self.T * self.k


WORKLOADS = [
    Workload("tiny", 64, 256, 128, 16, 2, FMT_Q2),
    Workload("verify2", 2, 2048, 512, 512, 10, FMT_Q2),
    Workload("chunk512", 512, 2048, 512, 512, 10, FMT_Q2),
    Workload("chunk2048_q2", 2048, 2048, 512, 512, 10, FMT_Q2),
    Workload("chunk2048_q1_skew", 2048, 2048, 512, 512, 10, FMT_Q1, True),
]
HEADLINE = 3


def blocks_per_row(K: int) -> int:
    return (K + BLOCK_VALUES - 1) // BLOCK_VALUES


def expert_bytes(fmt: int, H: int, I: int) -> int:
    """Bytes of one expert blob: gate and up (I rows of K=H) then down (H rows of K=I)."""
    nblk = 2 * I * blocks_per_row(H) + H * blocks_per_row(I)
    return nblk * BLOCK_BYTES[fmt]


def expert_stride(fmt: int, H: int, I: int) -> int:
    b = expert_bytes(fmt, H, I)
    return (b + EXPERT_ALIGN - 1) // EXPERT_ALIGN * EXPERT_ALIGN


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) and return the uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def random_blocks(rng: np.random.Generator, fmt: int, nblk: int) -> np.ndarray:
    """nblk random blocks of format fmt, shape [nblk, BLOCK_BYTES[fmt]] uint8."""
    bb = BLOCK_BYTES[fmt]
    out = rng.integers(0, 256, size=(nblk, bb), dtype=np.uint8)
    u = rng.random(nblk)
    d = np.float32(0.01) * (np.float32(0.5) + u.astype(np.float32))
    out[:, 0:2] = d.astype(np.float16).view(np.uint8).reshape(nblk, 2)
    return out


def random_logits(rng: np.random.Generator, T: int, E: int, skew: bool) -> np.ndarray:
    n = rng.standard_normal((T, E), dtype=np.float32)
    if not skew:
        return n
    perm = rng.permutation(E)
    rank = np.empty(E, dtype=np.float64)
    rank[perm] = np.arange(1, E + 1, dtype=np.float64)
    bias = 1.5 * np.log(1.0 / rank)
    return (n.astype(np.float64) + bias[None, :]).astype(np.float32)


@dataclasses.dataclass
class Inputs:
    wl: Workload
    x_bits: np.ndarray       # uint16 [T, H] bf16 patterns
    logits: np.ndarray       # float32 [T, E]
    blobs: np.ndarray        # uint8 [E, stride]; expert e = blobs[e, :expert_bytes]
    seed: int

    @property
    def stride(self) -> int:
        return self.blobs.shape[1]


def make_inputs(wl: Workload, seed: int | None = None) -> Inputs:
    """Draw the inputs of one workload.  Default seed: BASE_SEED + its index."""
    if seed is None:
        seed = BASE_SEED + WORKLOADS.index(wl) if wl in WORKLOADS else BASE_SEED
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((wl.T, wl.H), dtype=np.float32)
    x_bits = f32_to_bf16_bits(x)
    logits = random_logits(rng, wl.T, wl.E, wl.skew)
    nbytes = expert_bytes(wl.fmt, wl.H, wl.I)
    stride = expert_stride(wl.fmt, wl.H, wl.I)
    nblk = nbytes // BLOCK_BYTES[wl.fmt]
    blobs = np.zeros((wl.E, stride), dtype=np.uint8)
    blk = random_blocks(rng, wl.fmt, wl.E * nblk)
    blobs[:, :nbytes] = blk.reshape(wl.E, nbytes)
    return Inputs(wl, x_bits, logits, blobs, seed)


def router_weights(E: int, H: int, seed: int) -> np.ndarray:
    """Router weights W_r [E, H] as bf16 bit patterns: float32 N(0, 1/H)
    rounded to bf16, so that with x ~ N(0,1) the logits are about N(0, 1)
    like the other workloads' logits."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((E, H), dtype=np.float32) / np.float32(np.sqrt(H))
    return f32_to_bf16_bits(w)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a bit shift, no rounding)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)
