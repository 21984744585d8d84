"""Shared helpers of the GPU parity tests: host/device transfer of BF16 bit
patterns, the scale-layout mapping, and the GEMM tolerance check against the
oracle."""
import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq

# GEMM tolerance.  The primary gate is the relative Frobenius error of 2e-3.
# Per element, both sides round nearly the same real number to BF16, so
#   |y_gpu - y_ref| <= 1 ulp_bf16(|y|) + GAMMA * S + 2^-22 |y|,
# where S = |alpha_x alpha_w| sum_k |xhat' what'| bounds the FP32
# accumulation error of the tensor cores (GAMMA) and the two FP32 roundings of
# the tensor-scale multiply add 2^-22 relative.
REL_FROB_MAX = 2e-3
GAMMA = 2.0 ** -16


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), f"this library targets sm_100a, found sm_{major}{minor}"
    import os
    if not os.path.exists(mq.LIB_PATH):
        from phase_aware_nvfp4_b200 import build
        build.build()
    mq.load()


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """BF16 bit patterns (uint16) -> torch.bfloat16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def scales_from_layout(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Read row-major [rows, cols/16] scales out of the MMA scale layout (host-side mapping)."""
    atoms = ((cols + 255) // 256) * 4
    r = np.arange(rows)[:, None]
    kb = np.arange(cols // 16)[None, :]
    off = ((r // 128) * atoms + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (kb % 4)
    return buf[off]


def nvfp4_host(t: "mq.NVFP4Tensor"):
    """(codes, row-major scales, alpha) of a device NVFP4 tensor."""
    codes = t.codes.cpu().numpy()
    scales = scales_from_layout(t.scales.cpu().numpy(), t.rows, t.cols)
    alpha = float(t.alpha.cpu().numpy()[0])
    return codes, scales, alpha


def gemm_check(y_gpu_bits: np.ndarray, y64: np.ndarray, sabs: np.ndarray, gamma: float = GAMMA,
               rel_max: float = REL_FROB_MAX):
    """Assert the GPU BF16 output is within tolerance of the oracle; returns (rel_frob, max_abs, bound_max)."""
    y_gpu = oracle.bf16_to_f64(y_gpu_bits)
    y_ref = oracle.bf16_to_f64(oracle.round_bf16(y64))
    rel = oracle.rel_frobenius(y_gpu, y_ref)
    ulp = np.maximum(oracle.bf16_ulp(y_ref), oracle.bf16_ulp(y_gpu))
    bound = ulp + gamma * sabs + 2.0 ** -22 * np.abs(y64)
    err = np.abs(y_gpu - y_ref)
    bad = err > bound
    assert rel <= rel_max, f"rel-Frobenius {rel:.3e} > {rel_max}"
    assert not bad.any(), (f"{int(bad.sum())} elements over the bound; worst excess "
                           f"{float((err - bound).max()):.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}")
    return rel, float(err.max()), float(bound.max())


def sample_rows(M: int, n: int = 64, seed: int = 0, extra=()) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist())
    rows |= {0, M - 1, *[int(e) for e in extra if 0 <= e < M]}
    return np.array(sorted(rows), dtype=np.int64)


def block_rows(M: int, seed: int = 0, block: int = 128, extra=()) -> np.ndarray:
    """One seeded random row in every `block`-row block of an M-row output, plus the first
    and last rows: a tile-scheduler or raster slip that hits only some tiles shows up in
    at least one sampled row."""
    rng = np.random.default_rng(seed)
    rows = {0, M - 1, *[int(e) for e in extra if 0 <= e < M]}
    for b0 in range(0, M, block):
        rows.add(int(rng.integers(b0, min(b0 + block, M))))
    return np.array(sorted(rows), dtype=np.int64)


def silu_mul_check(h_gpu_bits: np.ndarray, g64: np.ndarray, u64: np.ndarray, sg: np.ndarray, su: np.ndarray,
                   rel_max: float = REL_FROB_MAX):
    """Assert the fused epilogue's h = bf16(silu(g) u) is within tolerance of the oracle's.

    g64, u64: the oracle's FP64 gate/up GEMM outputs (tensor scales applied); sg, su: their
    sum_k |products| bounds (nvfp4_linear_rows' second result).  The GPU's g and u differ
    from fl32(g64), fl32(u64) by at most dg = GAMMA*sg + 2^-22|g64| (tensor-core FP32
    accumulation, two FP32 roundings of the tensor-scale multiply), likewise du.  With
    |silu'| <= 1.1 and both sides rounding their own FP32 silu (expf vs libm exp, a few
    binary32 ulps) and product before one BF16 rounding each:
        |h_gpu - h_ref| <= ulp_bf16(max|h|) + 1.1 |u| dg + (|silu(g)| + 1.1 dg) du + 2^-19 |h_ref|.
    Gates: rel-Frobenius <= rel_max and that bound on every element.
    Returns (rel_frob, max_abs, bound_max)."""
    hg = oracle.bf16_to_f64(h_gpu_bits)
    g = np.asarray(g64, dtype=np.float64)
    u = np.asarray(u64, dtype=np.float64)
    h_ref = oracle.bf16_to_f64(oracle.silu_mul(g, u))
    rel = oracle.rel_frobenius(hg, h_ref)
    dg = GAMMA * np.asarray(sg) + 2.0 ** -22 * np.abs(g)
    du = GAMMA * np.asarray(su) + 2.0 ** -22 * np.abs(u)
    silu = np.abs(g / (1.0 + np.exp(-np.clip(g, -700.0, 700.0))))
    bound = (np.maximum(oracle.bf16_ulp(h_ref), oracle.bf16_ulp(hg)) + 1.1 * np.abs(u) * dg
             + (silu + 1.1 * dg) * du + 2.0 ** -19 * np.abs(h_ref))
    err = np.abs(hg - h_ref)
    bad = err > bound
    assert rel <= rel_max, f"h rel-Frobenius {rel:.3e} > {rel_max}"
    assert not bad.any(), (f"{int(bad.sum())} h elements over the bound; worst excess "
                           f"{float((err - bound).max()):.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}")
    return rel, float(err.max()), float(bound.max())
