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
                                   (17, 272, 320), (200, 256, 512), (256, 128, 128), (1, 4096, 12288),
                                   (1, 16, 64), (1, 400, 1088), (2, 400, 1088), (1, 16, 131072)])
def test_decode_linear_vs_oracle(M, N, K):
    """M = 1 runs the CUDA-core kernel (unless the token, 2K bytes, exceeds shared memory, as at
    K = 131072), larger M the tensor-core kernel."""
    x = wl.heavy_tailed_bf16(M, K, M + K)
    w = wl.normal_bf16(N, K, 0.02, N + K)
    y = mq.decode_linear(to_dev(x), to_dev(w))
    torch.cuda.synchronize()
    decode_check(to_host_bits(y), x, w)


@pytest.mark.parametrize("M", [1, 8])
def test_decode_exact_small_integers(M):
    rng = np.random.default_rng(M)
    xi = rng.integers(-4, 5, size=(M, 1024)).astype(np.float32)
    wi = rng.integers(-4, 5, size=(512, 1024)).astype(np.float32)
    y = mq.decode_linear(to_dev(wl.f32_to_bf16_bits(xi)), to_dev(wl.f32_to_bf16_bits(wi)))
    torch.cuda.synchronize()
    assert np.array_equal(to_host_bits(y), oracle.round_bf16((xi.astype(np.float64) @ wi.T.astype(np.float64))))


# ---------------------------------------------------------------- uniform-NVFP4 decode

def _nvfp4_decode_check(x, w, y_gpu_bits, alpha_x=None):
    """Oracle: quantize X (dynamic alpha over its M rows unless given) and W, FP64 block-scaled matmul."""
    from gpu_helpers import gemm_check
    ax = oracle.tensor_alpha(x)[1] if alpha_x is None else alpha_x
    aw = oracle.tensor_alpha(w)[1]
    y64, sabs = oracle.nvfp4_linear_rows((*oracle.quantize(x, ax), ax), (*oracle.quantize(w, aw), aw))
    return gemm_check(y_gpu_bits, y64, sabs)


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (7, 400, 1088), (32, 512, 1024), (64, 768, 2048),
                                   (100, 272, 320), (128, 128, 4096), (1, 4096, 12288), (1, 12288, 4096),
                                   (8, 12288, 4096), (16, 12288, 4096), (16, 4096, 12288), (64, 12288, 4096),
                                   (128, 4096, 12288), (2, 400, 1024), (3, 1024, 2048), (4, 12288, 4096),
                                   (2, 4096, 12288), (1, 272, 8192), (1, 16, 131072)])
def test_decode_nvfp4_vs_oracle(M, N, K):
    """Ragged tokens (MMA N padded to 32), ragged weight rows (N % 128 != 0) and a partial last
    256-element stage (K % 256 != 0) are all covered, as are the launch shapes the call picks:
    the single kernel that quantizes the tokens itself (K split over clusters of 1 to 8 CTAs
    exchanging their slice maxima, or over independent CTAs adding partials through the
    workspace) and, above 32K token elements per CTA or where the token slice does not fit in
    shared memory, the quantization kernel followed by the decode GEMM."""
    x = wl.heavy_tailed_bf16(M, K, 3 * M + K)
    w = wl.normal_bf16(N, K, 0.02, 5 * N + K)
    Wq = mq.quantize_weight(to_dev(w))
    y = mq.decode_linear_nvfp4(to_dev(x), Wq)
    torch.cuda.synchronize()
    rel, mx, bmax = _nvfp4_decode_check(x, w, to_host_bits(y))
    print(f"nvfp4 decode M={M} N={N} K={K}: rel-Frobenius {rel:.2e}")


@pytest.mark.parametrize("M,K", [(16, 512), (3, 2048), (1, 4096), (1, 192)])
def test_decode_nvfp4_static_alpha_and_grid_inputs_exact(M, K):
    """Grid-valued inputs whose blocks all hold a 6: X with a static alpha of 1 and W with a 2688
    anchor alone in its block (alpha_w = 1) get block scales of exactly 1 (448 for the anchor), so
    Y = bf16(X W^T) exactly (the FP32 sums stay below 2^24 quarter units), on the quantization
    kernel + decode GEMM (16 tokens) and on the single kernel (1 and 3 tokens; K = 192 ends in a
    partial 256-element stage)."""
    rng = np.random.default_rng(3)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    xi = (rng.choice(grid, size=(M, K)) * rng.choice([-1, 1], size=(M, K))).astype(np.float32)
    wi = (rng.choice(grid, size=(256, K)) * rng.choice([-1, 1], size=(256, K))).astype(np.float32)
    xi[:, ::16] = 6.0
    wi[:, ::16] = 6.0
    wi[0, :16] = 0.0
    wi[0, 0] = 2688.0      # alone in its block (sigma 448 would round its neighbours to 0)
    Wq = mq.quantize_weight(to_dev(wl.f32_to_bf16_bits(wi)))
    assert float(Wq.alpha.cpu()[0]) == 1.0
    y = mq.decode_linear_nvfp4(to_dev(wl.f32_to_bf16_bits(xi)), Wq, alpha_static=torch.ones(1, device="cuda"))
    torch.cuda.synchronize()
    exact = xi.astype(np.float64) @ wi.T.astype(np.float64)
    assert np.array_equal(to_host_bits(y), oracle.round_bf16(exact))


@pytest.mark.parametrize("M,N,K", [(4, 12288, 4096), (1, 4096, 12288)])
def test_decode_nvfp4_repeatable_and_static_alpha(M, N, K):
    """The single-kernel decode gives the same bits on a repeated call (split-K partials added in
    rank order), and with a static alpha_x equal to the tokens' own amax / 2688 it gives the same
    bits as with the dynamic one (every CTA derives the same alpha_x)."""
    x = wl.heavy_tailed_bf16(M, K, 5 * M + N)
    w = wl.normal_bf16(N, K, 0.02, 13 * N + K)
    Wq = mq.quantize_weight(to_dev(w))
    X = to_dev(x)
    y1 = to_host_bits(mq.decode_linear_nvfp4(X, Wq))
    y2 = to_host_bits(mq.decode_linear_nvfp4(X, Wq))
    assert np.array_equal(y1, y2)
    ax = oracle.tensor_alpha(x)[1]
    y3 = to_host_bits(mq.decode_linear_nvfp4(X, Wq, alpha_static=torch.full((1,), ax, dtype=torch.float32,
                                                                             device="cuda")))
    assert np.array_equal(y1, y3)
    _nvfp4_decode_check(x, w, y1, alpha_x=ax)


def test_decode_nvfp4_matches_prefill_on_same_weight():
    """Uniform-NVFP4 decode and the NVFP4 prefill linear on the same tokens and the same
    12288 x 4096 weight agree, and match the oracle on 2048 weight rows."""
    from gpu_helpers import gemm_check
    x = wl.heavy_tailed_bf16(64, 4096, 77)
    w = wl.normal_bf16(12288, 4096, 0.02, 4001)
    Wq = mq.quantize_weight(to_dev(w))
    X = to_dev(x)
    yd = mq.decode_linear_nvfp4(X, Wq)
    yp = mq.prefill_linear(X, Wq)
    torch.cuda.synchronize()
    a, b = oracle.bf16_to_f64(to_host_bits(yd)), oracle.bf16_to_f64(to_host_bits(yp))
    assert oracle.rel_frobenius(a, b) < 1e-3
    ax = oracle.tensor_alpha(x)[1]
    aw = oracle.tensor_alpha(w)[1]
    wc, wsc = oracle.quantize(w[:2048], aw)
    y64, sabs = oracle.nvfp4_linear_rows((*oracle.quantize(x, ax), ax), (wc, wsc, aw))
    gemm_check(to_host_bits(yd)[:, :2048], y64, sabs)


def test_decode_nvfp4_reports_nonfinite_tokens():
    """A NaN among the tokens is excluded from the tensor amax and reported as MQ_ERR_NONFINITE;
    the other tokens are still quantized with the finite maximum."""
    x = wl.heavy_tailed_bf16(4, 2048, 91)
    x[2, 777] = 0x7FC0                       # BF16 NaN
    w = wl.normal_bf16(512, 2048, 0.02, 92)
    Wq = mq.quantize_weight(to_dev(w))
    ws = mq.workspace(4, 2048)
    y = mq.decode_linear_nvfp4(to_dev(x), Wq, ws=ws)
    assert mq.async_status(ws) == 5          # MQ_ERR_NONFINITE
    finite = np.array([0, 1, 3])
    xf = x.copy()
    xf[2, 777] = 0
    ax = oracle.tensor_alpha(x)[1]           # NaN excluded, as on the device
    assert ax == oracle.tensor_alpha(xf)[1]
    _nvfp4_decode_check(x[finite], w, to_host_bits(y)[finite], alpha_x=ax)


def test_decode_nvfp4_single_token_nonfinite_and_zero():
    """One token: a NaN is reported as MQ_ERR_NONFINITE; an all-zero token gives alpha_x = 1, zero
    codes and an exactly zero output."""
    w = wl.normal_bf16(256, 1024, 0.02, 93)
    Wq = mq.quantize_weight(to_dev(w))
    x = wl.heavy_tailed_bf16(1, 1024, 94)
    x[0, 5] = 0x7FC0
    ws = mq.workspace(1, 1024)
    mq.decode_linear_nvfp4(to_dev(x), Wq, ws=ws)
    assert mq.async_status(ws) == 5          # MQ_ERR_NONFINITE
    z = np.zeros((1, 1024), np.uint16)
    y = mq.decode_linear_nvfp4(to_dev(z), Wq, ws=ws)
    assert mq.async_status(ws) == 0
    assert not np.any(to_host_bits(y) & 0x7FFF)


@pytest.mark.parametrize("M,N,K", [(8, 1024, 4096), (8, 12288, 4096), (64, 4096, 2048)])
def test_decode_cluster_split_with_a_small_workspace(M, N, K):
    """With only the control block (BF16) or mq_workspace_bytes(M, K) (NVFP4) as workspace, the K
    split runs over thread-block clusters (partials added through distributed shared memory);
    the default decode workspace splits K over independent CTAs instead.  Both are within the
    oracle's tolerance, and each path repeated on its workspace gives the same bits (the
    split-K sums run in a fixed order; the per-tile counters reset themselves)."""
    from gpu_helpers import gemm_check
    x = wl.heavy_tailed_bf16(M, K, 7 * M + N)
    w = wl.normal_bf16(N, K, 0.02, 11 * N + K)
    X, Wd = to_dev(x), to_dev(w)
    Wq = mq.quantize_weight(Wd)
    small, small_q = mq.workspace(), mq.workspace(M, K)
    big = mq.decode_workspace(M, N, K)
    outs = []
    for ws in (small, big):
        y1 = to_host_bits(mq.decode_linear(X, Wd, ws=ws))
        y2 = to_host_bits(mq.decode_linear(X, Wd, ws=ws))
        assert np.array_equal(y1, y2)
        decode_check(y1, x, w)
        outs.append(y1)
    for ws in (small_q, big):
        y1 = to_host_bits(mq.decode_linear_nvfp4(X, Wq, ws=ws))
        y2 = to_host_bits(mq.decode_linear_nvfp4(X, Wq, ws=ws))
        assert np.array_equal(y1, y2)
        _nvfp4_decode_check(x, w, y1)
    for ws in (small, small_q, big):
        assert mq.async_status(ws) == 0
