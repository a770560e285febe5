"""Seeded synthetic BF16 weight blocks, shared by the tests, the benchmark,
the smoke check and the oracle's pins.

This module only draws random numbers and rounds them to BF16; it holds none
of the codec's arithmetic.  The shapes follow the models the DFloat11 pages
measure (Llama-3.1-8B transformer blocks, a FLUX.1-style DiT block); trained
checkpoints are not available, so normal / Student-t draws stand in for them.
Every generator is deterministic in its seed.
"""
from __future__ import annotations

import os

import numpy as np

# --------------------------------------------------------------- rounding


def to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns, round to nearest even (finite inputs).

    The rounding the page "DFloat11: lossless BFloat16 compression" uses to
    make its synthetic tensor (section "How it works: the core algorithm").
    """
    u = np.ascontiguousarray(x, dtype=np.float32).reshape(-1).view(np.uint32)
    out = np.empty(u.size, np.uint16)
    step = 1 << 20
    r = np.empty(min(step, u.size), np.uint32)
    for lo in range(0, u.size, step):
        a = u[lo: lo + step]
        t = r[: a.size]
        np.right_shift(a, 16, out=t)
        np.bitwise_and(t, 1, out=t)
        np.add(t, 0x7FFF, out=t)
        np.add(t, a, out=t)
        np.right_shift(t, 16, out=t)
        out[lo: lo + a.size] = t
    return out.reshape(np.shape(x))


def _normal_bf16(rng: np.random.Generator, shape, sigma: float) -> np.ndarray:
    n = int(np.prod(shape))
    x = rng.standard_normal(n, dtype=np.float32)
    x *= np.float32(sigma)
    return to_bf16(x).reshape(shape)


# ------------------------------------------------------------------ blocks

LLAMA8B_BLOCK_SHAPES = [
    ("q_proj", (4096, 4096)),
    ("k_proj", (1024, 4096)),
    ("v_proj", (1024, 4096)),
    ("o_proj", (4096, 4096)),
    ("gate_proj", (14336, 4096)),
    ("up_proj", (14336, 4096)),
    ("down_proj", (4096, 14336)),
]

FLUX_BLOCK_SHAPES = (
    [("qkv", (9216, 3072)), ("proj", (3072, 3072)), ("mlp_in", (12288, 3072)),
     ("mlp_out", (3072, 12288)), ("adaln", (18432, 3072))]
    + [(f"small_{i:02d}", (3072, 256)) for i in range(64)]
)


def single_matrix(seed: int = 0, shape=(1024, 1024), sigma: float = 0.02):
    """One matrix of N(0, sigma) weights: the page's worked-example recipe
    (numpy default_rng(seed).normal(0, sigma) in float64, cast to float32)."""
    rng = np.random.default_rng(seed)
    x = rng.normal(0.0, sigma, int(np.prod(shape))).astype(np.float32)
    return [("w", to_bf16(x).reshape(shape))]


def llama_block(seed: int = 1000, scale_div: int = 1):
    """A Llama-3.1-8B-shaped transformer block: 7 matrices, per-matrix sigma
    drawn uniformly from [0.01, 0.04] (all 7 drawn first), then float32
    normals.  scale_div > 1 shrinks every row count (small test variant)."""
    rng = np.random.default_rng(seed)
    sig = rng.uniform(0.01, 0.04, len(LLAMA8B_BLOCK_SHAPES))
    out = []
    for (name, (r, c)), s in zip(LLAMA8B_BLOCK_SHAPES, sig):
        out.append((name, _normal_bf16(rng, (max(1, r // scale_div), c), float(s))))
    return out


def llama_model_seeds(n_blocks: int = 32, first_seed: int = 1000):
    """Seeds of the blocks of the 8B-scale stream (block i uses first_seed+i)."""
    return [first_seed + i for i in range(n_blocks)]


def _llama_block_flat(args):
    seed, scale_div = args
    return seed, np.concatenate([m.reshape(-1) for _, m in llama_block(seed, scale_div=scale_div)])


def llama_model_blocks(seeds, scale_div: int = 1, processes: int | None = None):
    """Yields (seed, flat uint16 BF16 bits of llama_block(seed)) in seed
    order, the blocks drawn by a pool of worker processes (numpy draws one
    block on one core; a 32-block stream would take minutes serially).  The
    pool uses the spawn start method, so it is safe in a process that has
    already initialised CUDA.  Same numbers as llama_block(seed)."""
    import multiprocessing as mp
    seeds = list(seeds)
    if processes is None:
        processes = max(1, min(8, (os.cpu_count() or 2) - 1, len(seeds)))
    if processes <= 1 or len(seeds) <= 1:
        for sd in seeds:
            yield _llama_block_flat((sd, scale_div))
        return
    with mp.get_context("spawn").Pool(processes) as pool:
        yield from pool.imap(_llama_block_flat, [(sd, scale_div) for sd in seeds])


def flux_block(seed: int = 5000, scale_div: int = 1):
    """FLUX.1-style DiT block, hidden 3072, N(0, 0.02): 5 large matrices and
    64 small 3072x256 ones, in that order."""
    rng = np.random.default_rng(seed)
    out = []
    for name, (r, c) in FLUX_BLOCK_SHAPES:
        out.append((name, _normal_bf16(rng, (max(1, r // scale_div), c), 0.02)))
    return out


SPECIAL_BF16 = [0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x7F81]


def heavy_tail(seed: int = 4001, shape=(4096, 4096)):
    """Student-t (nu=3) * 0.02; 0.1% of entries get a uniformly random exponent
    field (sign and mantissa kept); then 64 copies each of +-0, +-Inf and three
    NaN patterns, and 1024 random subnormals, at random positions."""
    rng = np.random.default_rng(seed)
    n = int(np.prod(shape))
    x = (rng.standard_t(3, n) * 0.02).astype(np.float32)
    w = to_bf16(x)
    k = max(1, n // 1000)
    idx = rng.choice(n, size=k, replace=False)
    new_exp = rng.integers(0, 256, k).astype(np.uint16)
    w[idx] = (w[idx] & np.uint16(0x807F)) | (new_exp << np.uint16(7))
    specials = np.repeat(np.array(SPECIAL_BF16, np.uint16), 64)
    sub_sign = rng.integers(0, 2, 1024).astype(np.uint16) << np.uint16(15)
    sub_mant = rng.integers(1, 128, 1024).astype(np.uint16)
    specials = np.concatenate([specials, sub_sign | sub_mant])
    pos = rng.choice(n, size=specials.size, replace=False)
    w[pos] = specials
    return [("heavy_tail", w.reshape(shape))]


def single_exponent(seed: int = 4002, shape=(4096, 4096), exponent: int = 0x79):
    """N(0, 0.02) with every exponent field forced to one value."""
    rng = np.random.default_rng(seed)
    n = int(np.prod(shape))
    w = to_bf16(rng.standard_normal(n, dtype=np.float32) * np.float32(0.02))
    w = (w & np.uint16(0x807F)) | np.uint16(exponent << 7)
    return [("single_exponent", w.reshape(shape))]


def uniform_bits(seed: int = 4003, shape=(4096, 4096)):
    """Uniformly random 16-bit patterns (every exponent, NaNs and Infs included)."""
    rng = np.random.default_rng(seed)
    w = rng.integers(0, 65536, int(np.prod(shape)), dtype=np.uint16)
    return [("uniform_bits", w.reshape(shape))]


def llama_block_device(seed: int, device="cuda", scale_div: int = 1):
    """The Llama-3.1-8B-shaped block drawn on the GPU with torch's CUDA
    generator (seeded), for streams of many blocks where host generation is
    too slow: sigma_i = uniform(0.01, 0.04) for the 7 matrices first, then
    float32 normals; BF16 by torch's round-to-nearest-even cast.  Returns one
    contiguous int16 tensor of BF16 bit patterns (matrices in order).  Not the
    same numbers as llama_block(seed): a different generator."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    sig = torch.rand(len(LLAMA8B_BLOCK_SHAPES), generator=g, device=device, dtype=torch.float64)
    sig = (0.01 + 0.03 * sig).tolist()
    parts = []
    for (name, (r, c)), s in zip(LLAMA8B_BLOCK_SHAPES, sig):
        x = torch.randn(max(1, r // scale_div) * c, generator=g, device=device, dtype=torch.float32)
        x.mul_(s)
        parts.append(x.to(torch.bfloat16).view(torch.int16))
    return torch.cat(parts)


def many_tables(seed: int = 4004, n: int = 1 << 21, rare_fraction: float = 1 / 64,
                rare_exponents=range(256)):
    """One exponent (0x79) almost everywhere and the other exponents of
    rare_exponents (default: all 255 others) uniformly rare, random sign and
    mantissa: the dominant exponent gets a 1-bit code and the rare ones
    long codes spread over many second-level tables (with all 255: ~128
    tables, a block whose decode tables fill a large part of shared
    memory)."""
    rng = np.random.default_rng(seed)
    e = np.full(n, 0x79, dtype=np.uint16)
    k = int(n * rare_fraction)
    pos = rng.choice(n, size=k, replace=False)
    others = np.array([x for x in rare_exponents if x != 0x79], dtype=np.uint16)
    e[pos] = others[rng.integers(0, others.size, k)]
    sm = rng.integers(0, 256, n, dtype=np.uint16)
    w = ((sm >> 7) << 15) | (e << 7) | (sm & 0x7F)
    return [("many_tables", w.astype(np.uint16).reshape(1024, -1))]


def activations(seed: int, n_tokens: int, cols: int, sigma: float = 1.0):
    """Activation rows for the fused matrix-vector products: n_tokens x cols
    float32 N(0, sigma) rounded to BF16 (uint16 bit patterns)."""
    rng = np.random.default_rng(seed)
    return _normal_bf16(rng, (n_tokens, cols), sigma)


def small_cols_block(seed: int = 6000):
    """Matrices with rows shorter than 256 elements (and one of 8), so one
    step of 256 elements crosses several rows: 512x64, 64x8, 8x1024, 100x16."""
    rng = np.random.default_rng(seed)
    return [(f"m{i}", _normal_bf16(rng, shape, 0.02))
            for i, shape in enumerate([(512, 64), (64, 8), (8, 1024), (100, 16)])]


# The five workloads by name; each returns a list of (name, uint16 array).
WORKLOADS = {
    "single_1024x1024": lambda: single_matrix(0),
    "llama8b_block": lambda: llama_block(1000),
    "adversarial_heavy_tail": lambda: heavy_tail(4001),
    "adversarial_single_exponent": lambda: single_exponent(4002),
    "adversarial_uniform_bits": lambda: uniform_bits(4003),
    "flux_dit_block": lambda: flux_block(5000),
}


def numel(mats) -> int:
    return int(sum(m.size for _, m in mats))
