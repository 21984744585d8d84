"""Fused RMSNorm -> NVFP4 (mq_rmsnorm_quantize) vs the oracle: the normalized BF16 h, its
tensor scale, codes and block scales must be bit-exact (the reading fixes every rounding:
sum of squares in binary64, one rounding of ms and of rstd, binary32 products, BF16 h)."""
import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import nvfp4_host, require_gpu, to_dev, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check(x, g, eps):
    M, K = x.shape
    h_dbg = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    t = mq.rmsnorm_quantize(to_dev(x), to_dev(g), eps, h_debug=h_dbg)
    torch.cuda.synchronize()
    h_ref, _ = oracle.rmsnorm(x, g, eps)
    h_gpu = to_host_bits(h_dbg)
    assert np.array_equal(h_gpu, h_ref), f"{int((h_gpu != h_ref).sum())} of {h_ref.size} h values differ"
    codes, scales, alpha = nvfp4_host(t)
    _, a_ref, _ = oracle.tensor_alpha(h_ref)
    assert np.float32(alpha) == np.float32(a_ref)
    rc, rs = oracle.quantize(h_ref, a_ref)
    assert np.array_equal(scales, rs), f"{int((scales != rs).sum())} scale mismatches"
    assert np.array_equal(codes, rc), f"{int((codes != rc).sum())} code byte mismatches"
    return t, h_dbg


@pytest.mark.parametrize("M,K,eps", [(128, 256, 1e-6), (200, 1088, 1e-5), (1, 64, 0.0), (1000, 4096, 1e-6)])
def test_rmsnorm_quantize_bit_exact(M, K, eps):
    x = wl.heavy_tailed_bf16(M, K, 61 + M)
    g = wl.normal_bf16(1, K, 1.0, 62)[0]
    _check(x, g, eps)


def test_rmsnorm_quantize_full_size_and_matches_unfused_path():
    x = wl.heavy_tailed_bf16(8192, 4096, 63)
    g = wl.normal_bf16(1, 4096, 1.0, 64)[0]
    t, h_dbg = _check(x, g, 1e-6)
    # the unfused path (quantize the materialized BF16 h) gives the same NVFP4 tensor
    u = mq.quantize_activation(h_dbg)
    torch.cuda.synchronize()
    a, b = nvfp4_host(t), nvfp4_host(u)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]


def test_rmsnorm_quantize_closed_form_and_nonfinite():
    g = wl.normal_bf16(1, 256, 1.0, 65)[0]
    x = wl.f32_to_bf16_bits(np.full((128, 256), 2.0, np.float32))     # rstd = 0.5: h = gamma in every row
    h_dbg = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
    mq.rmsnorm_quantize(to_dev(x), to_dev(g), 0.0, h_debug=h_dbg)
    torch.cuda.synchronize()
    assert np.array_equal(to_host_bits(h_dbg), np.tile(g, (128, 1)))
    ws = mq.workspace(128, 256)
    xb = wl.heavy_tailed_bf16(128, 256, 66)
    xb[3, 5] = 0x7FC0
    mq.rmsnorm_quantize(to_dev(xb), to_dev(g), 1e-6, ws=ws)
    assert mq.async_status(ws) == 5
    assert mq.async_status(ws) == 0


def test_rmsnorm_quantize_extreme_magnitudes_bit_exact():
    """Squares that binary32 cannot hold: rows with one element of 2^64 (x^2 = 2^128, past FP32's
    range) and rows scaled to ~2^-72 (x^2 ~ 2^-144, FP32 subnormal).  The definition squares and
    adds in binary64, where both are exact, so h and its NVFP4 tensor stay bit-exact."""
    M, K = 64, 512
    base = wl.bf16_bits_to_f32(wl.heavy_tailed_bf16(M, K, 67))
    big = wl.f32_to_bf16_bits(base[:32])
    for r in range(32):
        big[r, (37 * r) % K] = 0x5F80          # 2^64
    tiny = wl.f32_to_bf16_bits(base[32:] * np.float32(2.0 ** -72))
    x = np.concatenate([big, tiny])
    assert np.all((x[32:] & 0x7F80) != 0x7F80)
    g = wl.normal_bf16(1, K, 1.0, 68)[0]
    _check(x, g, 0.0)
