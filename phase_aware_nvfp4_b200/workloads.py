"""Seeded synthetic inputs shaped like the paper's long-context prefill workloads.

This module holds no quantization arithmetic; it only draws random tensors.
It is the one piece shared by the CUDA path's tests/benchmark and the CPU
oracle, so both see bit-identical inputs.

Shapes follow the Qwen3-8B layer the paper evaluates ("Mix-Quant: Quantized
Prefilling, Precise Decoding for Agentic LLMs", section 4.1 "Models"; the
131K-token context of the "Evaluation Setup" paragraph sets the long-context
length): hidden 4096, KV projection 1024, MLP intermediate 12288.  The
benchmarks the paper evaluates on are not available, so these seeded tensors
stand in for their activations: Student-t(3) values with 1% of the channels
scaled by 20 (heavy tails plus outlier channels, the activation statistics
that make 4-bit quantization hard), weights N(0, 0.02^2).

Every tensor is produced as BF16 bit patterns (numpy uint16), row-major, by
rounding float32 draws to nearest-even.  Generation is chunked by rows; each
chunk has its own ``SeedSequence((seed, tag, chunk))`` stream so a tensor is a
pure function of (seed, shape).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK_ROWS = 2048
_MAX_THREADS = 8


def _by_chunks(rows: int, fill):
    """Run fill(c, r0, r1) for every CHUNK_ROWS chunk.  Each chunk has its own
    generator, so the result does not depend on the order or the threads the
    chunks run on; numpy drops the GIL inside the bulk draws and arithmetic."""
    spans = [(c, r0, min(rows, r0 + CHUNK_ROWS)) for c, r0 in enumerate(range(0, rows, CHUNK_ROWS))]
    threads = min(len(spans), _MAX_THREADS, os.cpu_count() or 1)
    if threads <= 1:
        for sp in spans:
            fill(*sp)
        return
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda sp: fill(*sp), spans))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _gen(seed: int, tag: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(tag), int(chunk)])))


def normal_bf16(rows: int, cols: int, std: float, seed: int) -> np.ndarray:
    """N(0, std^2) as BF16, [rows, cols]."""
    out = np.empty((rows, cols), dtype=np.uint16)

    def fill(c, r0, r1):
        z = _gen(seed, 1, c).standard_normal((r1 - r0, cols), dtype=np.float32)
        out[r0:r1] = f32_to_bf16_bits(z * np.float32(std))
    _by_chunks(rows, fill)
    return out


def outlier_channels(cols: int, frac: float, seed: int) -> np.ndarray:
    """The round(frac * cols) channel indices that carry the x20 outliers."""
    n = int(round(frac * cols))
    perm = _gen(seed, 2, 0).permutation(cols)
    return np.sort(perm[:n])


def heavy_tailed_bf16(rows: int, cols: int, seed: int, outlier_frac: float = 0.01,
                      outlier_scale: float = 20.0) -> np.ndarray:
    """Student-t(3) activations with outlier channels, as BF16 [rows, cols].

    t = z0 / sqrt((z1^2 + z2^2 + z3^2) / 3) with z_i ~ N(0, 1) (the textbook
    construction of Student-t with 3 degrees of freedom); the columns chosen
    by ``outlier_channels`` are multiplied by ``outlier_scale`` before the
    BF16 cast.
    """
    ch = outlier_channels(cols, outlier_frac, seed)
    colscale = np.ones(cols, dtype=np.float32)
    colscale[ch] = np.float32(outlier_scale)
    out = np.empty((rows, cols), dtype=np.uint16)

    def fill(c, r0, r1):
        z = _gen(seed, 3, c).standard_normal((4, r1 - r0, cols), dtype=np.float32)
        chi2 = z[1] * z[1] + z[2] * z[2] + z[3] * z[3]
        t = z[0] / np.sqrt(chi2 / np.float32(3.0))
        out[r0:r1] = f32_to_bf16_bits(t * colscale)
    _by_chunks(rows, fill)
    return out


def ragged_heavy_tailed_bf16(lengths, cols: int, seed: int):
    """Concatenated sequences, each with its own seeded outlier channel set.

    Returns (x [sum(lengths), cols] BF16, offsets [len+1]).
    """
    lengths = [int(n) for n in lengths]
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    out = np.empty((int(offsets[-1]), cols), dtype=np.uint16)
    for i, n in enumerate(lengths):
        out[offsets[i]:offsets[i + 1]] = heavy_tailed_bf16(n, cols, seed * 100 + i)
    return out, offsets


# --------------------------------------------------------------------------
# Named workloads
# --------------------------------------------------------------------------

QWEN3_8B_HIDDEN = 4096
QWEN3_8B_KV = 1024
QWEN3_8B_INTER = 12288
WEIGHT_STD = 0.02

# Ragged multi-turn prefill: {2k, 4k, 8k, 8k, 16k, 16k, 32k, 42k} tokens.
# The listed "45k" last turn would make the total 134144; the total is kept at
# the 131072-token long context and the last sequence gets 43008 tokens.
RAGGED_LENGTHS = (2048, 4096, 8192, 8192, 16384, 16384, 32768, 43008)


@dataclass(frozen=True)
class Projection:
    """One linear layer Y[M, N] = X[M, K] W[N, K]^T of a prefill pass."""
    name: str
    M: int
    K: int
    N: int
    x_seed: int
    w_seed: int
    x_kind: str = "heavy"      # "heavy" | "normal"
    x_group: str = ""          # projections with the same group share X

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


@dataclass(frozen=True)
class Workload:
    name: str
    projections: tuple = field(default_factory=tuple)

    @property
    def flops(self) -> int:
        return sum(p.flops for p in self.projections)


def tiny() -> Workload:
    """X 128x256 ~ N(0,1), W 256x256 ~ N(0, 0.02^2), seed 0 (X stream 0, W stream 1)."""
    return Workload("tiny_nvfp4_linear_128x256x256",
                    (Projection("tiny", 128, 256, 256, x_seed=0, w_seed=1, x_kind="normal", x_group="x"),))


def qwen3_8b_projections(M: int = 8192) -> Workload:
    """Qwen3-8B-shaped projections at M prefill tokens.

    q-proj (K=4096, N=4096) and k-proj (K=4096, N=1024) read the same
    attention input; up-proj (K=4096, N=12288) reads the MLP input; down-proj
    (K=12288, N=4096) reads the MLP intermediate.  Seeds follow
    1000*config + 10*shape + {0: X, 1: W}.
    """
    base = 2000
    return Workload(f"qwen3_8b_projections_M{M}", (
        Projection("q_proj", M, 4096, 4096, base + 0, base + 1, x_group="attn_in"),
        Projection("k_proj", M, 4096, 1024, base + 0, base + 11, x_group="attn_in"),
        Projection("up_proj", M, 4096, 12288, base + 20, base + 21, x_group="mlp_in"),
        Projection("down_proj", M, 12288, 4096, base + 30, base + 31, x_group="mlp_mid"),
    ))


def make_x(p: Projection) -> np.ndarray:
    if p.x_kind == "normal":
        return normal_bf16(p.M, p.K, 1.0, p.x_seed)
    return heavy_tailed_bf16(p.M, p.K, p.x_seed)


def make_w(p: Projection) -> np.ndarray:
    return normal_bf16(p.N, p.K, WEIGHT_STD, p.w_seed)


def mlp_weights(seed: int, hidden: int = QWEN3_8B_HIDDEN, inter: int = QWEN3_8B_INTER):
    """(W_gate_up [2*inter, hidden] with gate rows first, W_down [hidden, inter])."""
    w_gu = normal_bf16(2 * inter, hidden, WEIGHT_STD, seed + 1)
    w_dn = normal_bf16(hidden, inter, WEIGHT_STD, seed + 2)
    return w_gu, w_dn


def rope_cos_sin(max_pos: int, head_dim: int = 128, theta: float = 1.0e6) -> np.ndarray:
    """Rotary-embedding table input [max_pos, head_dim] float32: row p holds
    cos(p * f_i) for i < head_dim/2 followed by sin(p * f_i), f_i =
    theta^(-2i/head_dim) (theta = 1e6 as in the Qwen3 models).  Evaluated in
    float64 and rounded once; an input of the K/V projection, like the weights."""
    half = head_dim // 2
    f = theta ** (-2.0 * np.arange(half, dtype=np.float64) / head_dim)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * f[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)
