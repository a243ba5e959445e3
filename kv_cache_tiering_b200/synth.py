"""Seeded synthetic inputs for tiered decode attention.

This module serves both the CUDA path and the float64 oracle, and holds none of the
method's arithmetic: it draws random numbers, rounds them to BF16 storage, and arranges
tokens into the memory layouts the library reads (contiguous, token-major, paged).
Every tensor comes from its own counter-keyed stream, so any sample (one sequence, one
layer) can be regenerated alone.

Workloads (shapes, value distributions and structure of the five decode workloads this
library is measured on):
  tiny     batch 1, 1 query head / 1 KV head, d 64, 256 tokens, N(0,1), seed 0,
           softmax scale 1/8, 4 splits of 64 tokens
  exact    batch 8, 32 / 8 heads, d 128, 8192 tokens per sequence, N(0,1), contiguous
           head-major layout, 512-token splits
  hybrid   batch 4, 32 / 8 heads, d 128, 32768 tokens: newest 2048 exact, older 30720
           compact; K, V ~ N(0,1)
  staged   batch 1, 16 layers, 32 / 8 heads, d 128, 131072 tokens per layer in pinned
           host memory, token-major, 4096-token chunks, one new token per step
  staged-hybrid  the staged shape with the newest 2048 tokens per layer BF16 on the device
           and the older 129024 compact in pinned host memory, staged in 4096-token chunks
  ragged   batch 64, lengths uniform in [1024, 65536], 16-token pages with a seeded
           random page permutation, newest 1024 exact, K ~ Student-t(3), V, q ~ N(0,1)
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field

import numpy as np

PAGE_TOKENS = 16


def stream(seed: int, *key) -> np.random.Generator:
    """An independent PCG64 stream for (seed, key...).  String keys are hashed with CRC32."""
    spawn = tuple(int(zlib.crc32(k.encode())) if isinstance(k, str) else int(k) for k in key)
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=spawn)))


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bfloat16 storage (round-to-nearest-even), as uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    rounded = ((u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)).astype(np.uint16)
    return np.where(nan, np.uint16(0x7FC0), rounded).astype(np.uint16)


def normal_bf16(gen: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(gen.standard_normal(shape, dtype=np.float32))


def student_t_bf16(gen: np.random.Generator, shape, nu: float = 3.0) -> np.ndarray:
    return f32_to_bf16_bits(gen.standard_t(nu, size=shape).astype(np.float32))


# ----------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    split_tokens: int
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=1, Hkv=1, d=64, split_tokens=64, extra={"T": 256}),
    "exact": Workload("exact", B=8, Hq=32, Hkv=8, d=128, split_tokens=512, extra={"T": 8192}),
    "hybrid": Workload("hybrid", B=4, Hq=32, Hkv=8, d=128, split_tokens=512,
                       extra={"T": 32768, "window": 2048}),
    "staged": Workload("staged", B=1, Hq=32, Hkv=8, d=128, split_tokens=512,
                       extra={"T": 131072, "layers": 16, "chunk": 4096, "buffers": 2}),
    "staged-hybrid": Workload("staged-hybrid", B=1, Hq=32, Hkv=8, d=128, split_tokens=512,
                              extra={"T": 131072, "layers": 16, "chunk": 4096, "buffers": 2, "window": 2048}),
    "ragged": Workload("ragged", B=64, Hq=32, Hkv=8, d=128, split_tokens=512,
                       extra={"min_len": 1024, "max_len": 65536, "window": 1024, "nu": 3.0}),
}


def queries(wl: Workload, layer: int = 0, step: int = 0, B: int | None = None) -> np.ndarray:
    """q bf16 bits [B, Hq, d] ~ N(0,1)."""
    B = wl.B if B is None else B
    return normal_bf16(stream(wl.seed, wl.name, "q", layer, step), (B, wl.Hq, wl.d))


def history_head_major(wl: Workload, b: int, T: int, layer: int = 0, key_dist: str = "normal"):
    """K, V bf16 bits [Hkv, T, d] of sequence b (one layer)."""
    gk = stream(wl.seed, wl.name, "k", layer, b)
    gv = stream(wl.seed, wl.name, "v", layer, b)
    shape = (wl.Hkv, T, wl.d)
    k = student_t_bf16(gk, shape, wl.extra.get("nu", 3.0)) if key_dist == "student_t" else normal_bf16(gk, shape)
    return k, normal_bf16(gv, shape)


def history_token_major(wl: Workload, layer: int, T: int, b: int = 0):
    """K, V bf16 bits [T, Hkv, d] of one layer: the host staging layout, where a run of
    consecutive tokens is one contiguous span."""
    gk = stream(wl.seed, wl.name, "k", layer, b)
    gv = stream(wl.seed, wl.name, "v", layer, b)
    shape = (T, wl.Hkv, wl.d)
    return normal_bf16(gk, shape), normal_bf16(gv, shape)


def new_token(wl: Workload, layer: int, step: int, b: int = 0):
    """K, V bf16 bits [Hkv, d] of the token appended at decode step ``step``."""
    g = stream(wl.seed, wl.name, "knew", layer, step, b)
    h = stream(wl.seed, wl.name, "vnew", layer, step, b)
    return normal_bf16(g, (wl.Hkv, wl.d)), normal_bf16(h, (wl.Hkv, wl.d))


def ragged_lengths(wl: Workload, B: int | None = None) -> np.ndarray:
    """Sequence lengths uniform on the integers [min_len, max_len] (inclusive)."""
    B = wl.B if B is None else B
    g = stream(wl.seed, wl.name, "lens")
    return g.integers(wl.extra["min_len"], wl.extra["max_len"], size=B, endpoint=True).astype(np.int32)


def page_permutation(wl: Workload, pool: str, n_pages: int) -> np.ndarray:
    """A seeded random permutation of the physical page ids of one pool."""
    return stream(wl.seed, wl.name, "perm", pool).permutation(n_pages).astype(np.int32)


def page_tables(lens_pages, perm: np.ndarray) -> np.ndarray:
    """Page table int32 [B, max_pages]: sequence b's logical pages take the next
    len_pages[b] entries of the permutation, in order; unused entries are -1."""
    lens_pages = np.asarray(lens_pages, dtype=np.int64)
    B = lens_pages.size
    width = max(1, int(lens_pages.max(initial=0)))
    table = np.full((B, width), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        n = int(lens_pages[b])
        table[b, :n] = perm[off:off + n]
        off += n
    return table


def scatter_pages(tokens_hd: np.ndarray, table_row: np.ndarray, pool: np.ndarray) -> None:
    """Copy one sequence's tokens [Hkv, T, d] into a page pool [P, Hkv, 16, d] through
    its page-table row (logical page j -> physical page table_row[j])."""
    hkv, T, d = tokens_hd.shape
    n_pages = -(-T // PAGE_TOKENS)
    for j in range(n_pages):
        a, e = j * PAGE_TOKENS, min((j + 1) * PAGE_TOKENS, T)
        pool[table_row[j], :, : e - a, :] = tokens_hd[:, a:e, :]


def rotation_sign_bits(seed: int, d: int, key: str = "signs") -> int:
    """d random bits (bit i: coordinate i's sign flip) for a randomised rotation."""
    bits = stream(seed, "rotation", key).integers(0, 2, size=d)
    return int(sum(int(b) << i for i, b in enumerate(bits)))


# ----------------------------------------------------------------------------------
# device-side generators for full-size workloads (same distributions, BF16 rounding RNE)
# ----------------------------------------------------------------------------------


def torch_generator(seed: int, *key, device="cuda"):
    """A seeded torch generator on `device` for (seed, key...)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(stream(seed, "torch", *key).integers(0, 2**62)))
    return g


def torch_normal_bf16(g, shape, device="cuda"):
    """N(0,1) rounded to BF16; returns an int16 tensor holding the BF16 bits."""
    import torch
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16).view(torch.int16)


def torch_student_t3_bf16(g, shape, device="cuda"):
    """Student-t with 3 degrees of freedom, z / sqrt((z1^2 + z2^2 + z3^2) / 3), rounded to BF16."""
    import torch
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(3):
        chi2.add_(torch.randn(shape, generator=g, device=device, dtype=torch.float32).square_())
    return (z / torch.sqrt(chi2 / 3.0)).to(torch.bfloat16).view(torch.int16)


def torch_sequence_kv(wl: Workload, b: int, L: int, key_dist: str = "student_t", key: str = "kv", device="cuda"):
    """K, V of sequence b, [Hkv, L, d] int16 tensors of BF16 bits, drawn on `device` from the
    sequence's own seeded generator (keys Student-t(3) or N(0,1), values N(0,1)).  The same
    call always returns the same bits, so a test can redraw any sequence of a full-size batch."""
    g = torch_generator(wl.seed, wl.name, key, b, device=device)
    shape = (wl.Hkv, L, wl.d)
    k = torch_student_t3_bf16(g, shape, device) if key_dist == "student_t" else torch_normal_bf16(g, shape, device)
    return k, torch_normal_bf16(g, shape, device)
