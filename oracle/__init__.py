"""CPU oracle of the NVFP4 prefill linear layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow and (by construction) obviously correct reference of what the
CUDA path computes, written from "Mix-Quant: Quantized Prefilling, Precise
Decoding for Agentic LLMs", section 3.3, Eq. 2 (element quantization /
dequantization) and Eq. 3 (amax block scale), plus the format text around
them (E2M1 values, g = 16 element blocks with FP8-E4M3 scales, a tensor-level
scale, RTN with clipping, blocks contiguous along the GEMM K dimension) and
the phase split of the same section (W4A4 prefill, BF16 decode).

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference legs of ``bench.py`` may import this package.  The product library
(``phase_aware_nvfp4_b200``) never imports it and the two share no code.

Layering:
  * ``mq_oracle.c`` (compiled to ``liboracle.so``) holds the per-element
    arithmetic: E2M1 / E4M3 encode (exhaustive nearest search) and decode,
    the tensor scale, block quantization, dequantization, BF16 rounding and
    the SiLU-mul of the MLP; the opt-in per-block scale search (the paper's
    "scale optimization", read as trying the Eq. 3 scale code and its two
    E4M3 neighbours); and RMSNorm with its BF16 output (the producer of the
    quantized activation).
  * The matmuls are numpy float64 ``@`` on the dequantized operands (a library
    primitive used as one step), followed by the tensor scales and BF16
    rounding in C.
  * ``kv_rope_rows`` applies rotate-half rotary embedding to the K projection
    output in float64 and rounds K and V to BF16 (the KV cache in the decode
    precision, "Prefill-Decode Disaggregation Deployment").

Every function here has at least one pin in ``tests/test_oracle_pins.py``
against facts fixed by the format definitions or the mathematics (closed
forms, exhaustive enumeration, brute force, invariants, hand-worked blocks).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Formats: constants fixed by the E2M1 / E4M3 definitions.
E2M1_MAX = 6.0          # q_max in Eq. 3: largest finite FP4 (E2M1) magnitude
E4M3_MAX = 448.0        # largest finite E4M3 value
BLOCK = 16              # g, the block size of the NVFP4 partition


def build(force: bool = False) -> str:
    """Compile ``mq_oracle.c`` into ``liboracle.so`` with gcc (no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            u8p = ctypes.POINTER(ctypes.c_uint8)
            u16p = ctypes.POINTER(ctypes.c_uint16)
            f32p = ctypes.POINTER(ctypes.c_float)
            f64p = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lib.orc_e2m1_value.argtypes = [ctypes.c_uint]
            lib.orc_e2m1_value.restype = ctypes.c_double
            lib.orc_e4m3_value.argtypes = [ctypes.c_uint]
            lib.orc_e4m3_value.restype = ctypes.c_double
            lib.orc_e4m3_round.argtypes = [ctypes.c_float]
            lib.orc_e4m3_round.restype = ctypes.c_uint
            lib.orc_e2m1_round.argtypes = [ctypes.c_float]
            lib.orc_e2m1_round.restype = ctypes.c_uint
            lib.orc_double_to_bf16.argtypes = [ctypes.c_double]
            lib.orc_double_to_bf16.restype = ctypes.c_uint16
            lib.orc_tensor_alpha.argtypes = [u16p, i64, f32p, f32p]
            lib.orc_tensor_alpha.restype = ctypes.c_int
            lib.orc_quantize_rows.argtypes = [u16p, i64, i64, ctypes.c_float, u8p, u8p]
            lib.orc_quantize_rows.restype = None
            lib.orc_quantize_rows_search.argtypes = [u16p, i64, i64, ctypes.c_float, u8p, u8p]
            lib.orc_quantize_rows_search.restype = None
            lib.orc_rmsnorm_rows.argtypes = [u16p, i64, i64, u16p, ctypes.c_float, u16p,
                                             ctypes.POINTER(ctypes.c_float)]
            lib.orc_rmsnorm_rows.restype = None
            lib.orc_dequantize_rows.argtypes = [u8p, u8p, i64, i64, ctypes.c_float, f64p]
            lib.orc_dequantize_rows.restype = None
            lib.orc_round_bf16.argtypes = [f64p, i64, u16p]
            lib.orc_round_bf16.restype = None
            lib.orc_silu_mul.argtypes = [f64p, f64p, i64, u16p]
            lib.orc_silu_mul.restype = None
            lib.orc_num_threads.argtypes = []
            lib.orc_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# --------------------------------------------------------------------------
# Formats
# --------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code (sign bit 3)."""
    return float(_L().orc_e2m1_value(int(code)))


def e4m3_value(code: int) -> float:
    """Value of an 8-bit E4M3 (FN) code; NaN for S.1111.111."""
    return float(_L().orc_e4m3_value(int(code)))


def e4m3_round(s: float) -> int:
    """Pi_E4M3 of Eq. 3 for s >= 0: nearest finite E4M3, ties to even, satfinite."""
    return int(_L().orc_e4m3_round(ctypes.c_float(s)))


def e2m1_round(m: float) -> int:
    """Pi_FP4 of Eq. 2 on a magnitude m >= 0: index of the nearest E2M1 magnitude."""
    return int(_L().orc_e2m1_round(ctypes.c_float(m)))


def bf16_to_f64(h: np.ndarray) -> np.ndarray:
    """Exact widening of BF16 bit patterns (uint16) to float64."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to BF16 bit patterns (RNE, no double rounding)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _L().orc_round_bf16(_ptr(v, ctypes.c_double), v.size, _ptr(out, ctypes.c_uint16))
    return out


# --------------------------------------------------------------------------
# Eq. 2 / Eq. 3
# --------------------------------------------------------------------------

def tensor_alpha(x_bf16: np.ndarray):
    """(amax, alpha, nonfinite) of a BF16 tensor; alpha = amax / (6 * 448)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    amax = ctypes.c_float(0.0)
    alpha = ctypes.c_float(0.0)
    bad = _L().orc_tensor_alpha(_ptr(x, ctypes.c_uint16), x.size, ctypes.byref(amax), ctypes.byref(alpha))
    return float(amax.value), float(np.float32(alpha.value)), bool(bad)


def quantize(x_bf16: np.ndarray, alpha: float, search: bool = False):
    """NVFP4-quantize BF16 rows [rows, K] with tensor scale ``alpha``.

    Returns (codes [rows, K/2] uint8, scales [rows, K/16] uint8 E4M3 codes),
    the plain row-major layout: element k of a row sits in byte k/2, even k
    in the low nibble; scale b covers elements 16b..16b+15.

    ``search``: per block, the Eq. 3 scale code and its two E4M3 neighbours
    are tried and the one with the smallest binary32 squared error is kept
    (the opt-in "scale optimization" reading; ties keep the Eq. 3 scale).
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    assert x.ndim == 2 and x.shape[1] % BLOCK == 0
    rows, K = x.shape
    codes = np.empty((rows, K // 2), dtype=np.uint8)
    scales = np.empty((rows, K // BLOCK), dtype=np.uint8)
    fn = _L().orc_quantize_rows_search if search else _L().orc_quantize_rows
    fn(_ptr(x, ctypes.c_uint16), rows, K, ctypes.c_float(alpha), _ptr(codes, ctypes.c_uint8),
       _ptr(scales, ctypes.c_uint8))
    return codes, scales


def rmsnorm(x_bf16: np.ndarray, gamma_bf16: np.ndarray, eps: float):
    """RMSNorm rows of BF16 x with BF16 weight gamma -> (h BF16 bits [rows, K], rstd float32 [rows]).

    ms = fl32(sum x^2 (binary64) / K), rstd = fl32(1 / sqrt(ms + eps)) (binary64, one rounding),
    h = bf16(fl32(fl32(x * rstd) * gamma)): the BF16 tensor an unfused norm would hand to the
    quantizer of the next linear layer.
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    g = np.ascontiguousarray(gamma_bf16, dtype=np.uint16).ravel()
    rows, K = x.shape
    assert g.shape == (K,)
    h = np.empty_like(x)
    r = np.empty(rows, dtype=np.float32)
    _L().orc_rmsnorm_rows(_ptr(x, ctypes.c_uint16), rows, K, _ptr(g, ctypes.c_uint16), ctypes.c_float(eps),
                          _ptr(h, ctypes.c_uint16), r.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return h, r


def dequantize(codes: np.ndarray, scales: np.ndarray, alpha: float) -> np.ndarray:
    """xhat = alpha * sigma_b * q_i in float64 (Eq. 2, right-hand side)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    assert scales.shape == (rows, K // BLOCK)
    out = np.empty((rows, K), dtype=np.float64)
    _L().orc_dequantize_rows(_ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint8), rows, K,
                             ctypes.c_float(alpha), _ptr(out, ctypes.c_double))
    return out


# --------------------------------------------------------------------------
# Matmuls
# --------------------------------------------------------------------------

def nvfp4_linear_rows(xq, wq, rows=None):
    """Block-scaled FP4 GEMM on the selected activation rows.

    xq, wq: (codes, scales, alpha) of X [M, K] and W [N, K] in the plain layout.
    Returns (y, sabs): y[i, n] = alpha_x * alpha_w * sum_k xhat'[r_i, k] * what'[n, k]
    in float64 (xhat', what' = sigma * q without tensor scales) and
    sabs = |alpha_x * alpha_w| * sum_k |xhat' * what'| for error bounds.
    """
    xc, xs, ax = xq
    wc, ws, aw = wq
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        xc, xs = xc[rows], xs[rows]
    xd = dequantize(xc, xs, 1.0)
    wd = dequantize(wc, ws, 1.0)
    a = float(np.float32(ax)) * float(np.float32(aw))
    y = a * (xd @ wd.T)
    sabs = abs(a) * (np.abs(xd) @ np.abs(wd).T)
    return y, sabs


def kv_rope_rows(yk: np.ndarray, yv: np.ndarray, positions: np.ndarray, cos_sin: np.ndarray, head_dim: int = 128):
    """RoPE on the K projection output and the KV-cache values in BF16 (the decode precision).

    yk, yv: float64 [M, H*head_dim] projection outputs (before BF16 rounding).  For every head
    and i < head_dim/2, with c = cos_sin[pos, i], s = cos_sin[pos, head_dim/2 + i]:
    k'_i = k_i c - k_{i+d/2} s and k'_{i+d/2} = k_{i+d/2} c + k_i s (rotate-half form), in float64.
    Returns (K', V) as BF16 bit patterns [M, H*head_dim].
    """
    yk = np.asarray(yk, dtype=np.float64)
    M, n = yk.shape
    H, d2 = n // head_dim, head_dim // 2
    cs = np.asarray(cos_sin, dtype=np.float64)[np.asarray(positions, dtype=np.int64)]   # [M, head_dim]
    c, s = cs[:, None, :d2], cs[:, None, d2:]
    k = yk.reshape(M, H, head_dim)
    a, b = k[:, :, :d2], k[:, :, d2:]
    kr = np.concatenate([a * c - b * s, b * c + a * s], axis=2).reshape(M, n)
    return round_bf16(kr), round_bf16(np.asarray(yv, dtype=np.float64))


def bf16_linear_rows(x_bf16: np.ndarray, w_bf16: np.ndarray, rows=None) -> np.ndarray:
    """y = x @ w^T in float64 on BF16 inputs (the precise decode path)."""
    x = x_bf16 if rows is None else x_bf16[np.asarray(rows, dtype=np.int64)]
    return bf16_to_f64(x) @ bf16_to_f64(w_bf16).T


def silu_mul(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """h = bf16(fl32(silu(fl32 gate)) * fl32 up) as BF16 bit patterns."""
    g = np.ascontiguousarray(gate, dtype=np.float64)
    u = np.ascontiguousarray(up, dtype=np.float64)
    assert g.shape == u.shape
    h = np.empty(g.shape, dtype=np.uint16)
    _L().orc_silu_mul(_ptr(g, ctypes.c_double), _ptr(u, ctypes.c_double), g.size, _ptr(h, ctypes.c_uint16))
    return h


def num_threads() -> int:
    """Threads the C oracle uses (OpenMP)."""
    return int(_L().orc_num_threads())


# --------------------------------------------------------------------------
# Error metrics
# --------------------------------------------------------------------------

def rel_frobenius(y: np.ndarray, y_ref: np.ndarray) -> float:
    """Relative Frobenius error ||y - y_ref||_F / ||y_ref||_F over all elements, in float64.

    The denominator is the reference's norm.  A zero reference has no relative
    scale: the result is 0 when y is zero as well and +inf otherwise, so a gate
    on it fails for any deviation instead of turning into an absolute one.
    """
    y = np.asarray(y, dtype=np.float64).ravel()
    y_ref = np.asarray(y_ref, dtype=np.float64).ravel()
    assert y.shape == y_ref.shape, f"shapes differ: {y.shape} vs {y_ref.shape}"
    num = float(np.linalg.norm(y - y_ref))
    den = float(np.linalg.norm(y_ref))
    if den > 0:
        return num / den
    return 0.0 if num == 0 else float("inf")


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of BF16 numbers at |v| (2^(e-7) for normal v, 2^-133 below)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.exp2(e - 7.0), 2.0 ** -133)
