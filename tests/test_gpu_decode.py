"""GPU BF16 decode GEMV / skinny GEMM (the precise phase) vs the oracle."""
import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import require_gpu, to_dev, to_host_bits

pytestmark = pytest.mark.gpu

# FP32 accumulation of exact BF16 products: |y_gpu - bf16(y)| <= 1 ulp_bf16 + 2^-16 sum|x w|.
GAMMA = 2.0 ** -16


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def decode_check(y_bits, x, w):
    y64 = oracle.bf16_linear_rows(x, w)
    sabs = np.abs(oracle.bf16_to_f64(x)) @ np.abs(oracle.bf16_to_f64(w)).T
    y_ref = oracle.bf16_to_f64(oracle.round_bf16(y64))
    y_gpu = oracle.bf16_to_f64(y_bits)
    ulp = np.maximum(oracle.bf16_ulp(y_ref), oracle.bf16_ulp(y_gpu))
    err = np.abs(y_gpu - y_ref)
    assert oracle.rel_frobenius(y_gpu, y_ref) < 1e-3
    assert np.all(err <= ulp + GAMMA * sabs), float((err - ulp - GAMMA * sabs).max())


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (8, 1024, 4096), (32, 512, 1024), (64, 768, 2048),
                                   (17, 272, 320), (200, 256, 512), (256, 128, 128), (1, 4096, 12288)])
def test_decode_linear_vs_oracle(M, N, K):
    x = wl.heavy_tailed_bf16(M, K, M + K)
    w = wl.normal_bf16(N, K, 0.02, N + K)
    y = mq.decode_linear(to_dev(x), to_dev(w))
    torch.cuda.synchronize()
    decode_check(to_host_bits(y), x, w)


def test_decode_exact_small_integers():
    rng = np.random.default_rng(0)
    xi = rng.integers(-4, 5, size=(8, 1024)).astype(np.float32)
    wi = rng.integers(-4, 5, size=(512, 1024)).astype(np.float32)
    y = mq.decode_linear(to_dev(wl.f32_to_bf16_bits(xi)), to_dev(wl.f32_to_bf16_bits(wi)))
    torch.cuda.synchronize()
    assert np.array_equal(to_host_bits(y), oracle.round_bf16((xi.astype(np.float64) @ wi.T.astype(np.float64))))
