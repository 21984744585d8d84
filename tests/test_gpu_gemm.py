"""GPU block-scaled NVFP4 GEMM (the prefill linear layer) vs the oracle."""
import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import gemm_check, nvfp4_host, require_gpu, silu_mul_check, to_dev, to_host_bits

pytestmark = pytest.mark.gpu

E2M1_POS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def oracle_linear(x, w, rows=None, alpha_x=None):
    ax = oracle.tensor_alpha(x)[1] if alpha_x is None else alpha_x
    aw = oracle.tensor_alpha(w)[1]
    xs = x if rows is None else x[rows]
    xq = (*oracle.quantize(xs, ax), ax)
    wq = (*oracle.quantize(w, aw), aw)
    return oracle.nvfp4_linear_rows(xq, wq)


def _grid(rows, K, rng, anchor_block):
    """E2M1-grid values, a +-6 in every block (sigma = 1), and one block [2688, 0, ...]
    (amax = 6*448, so alpha = 1).  X and W put the anchor in different blocks so no
    product exceeds 2688*6 and every FP32 partial sum stays exact."""
    v = rng.choice(np.array(E2M1_POS + [-p for p in E2M1_POS[1:]]), size=(rows, K)).reshape(rows, K // 16, 16)
    v[:, :, 0] = rng.choice([6.0, -6.0], size=(rows, K // 16))
    v = v.reshape(rows, K)
    b = anchor_block
    v[0, 16 * b:16 * b + 16] = 0.0
    v[0, 16 * b] = 2688.0
    return v


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 1024), (200, 336, 320), (1, 16, 64),
                                   (3300, 3072, 256), (3000, 3328, 256)])
def test_closed_form_grid_inputs_bit_exact(M, N, K):
    """alpha = sigma = 1 and grid-valued inputs make every product exact: Y = bf16(X W^T) exactly."""
    rng = np.random.default_rng(M + N + K)
    xv, wv = _grid(M, K, rng, 0), _grid(N, K, rng, 1)
    x, w = wl.f32_to_bf16_bits(xv.astype(np.float32)), wl.f32_to_bf16_bits(wv.astype(np.float32))
    W = mq.quantize_weight(to_dev(w))
    y = mq.prefill_linear(to_dev(x), W)
    torch.cuda.synchronize()
    exact = xv @ wv.T          # all values are multiples of 1/4 below 2^40: exact in float64
    assert np.array_equal(to_host_bits(y), oracle.round_bf16(exact))


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (300, 1024, 1024), (200, 336, 320), (129, 272, 4096),
                                   (1, 16, 64), (640, 768, 2048),
                                   # shapes that take 256 x 384 pair tiles (fewer waves than 256 x 256):
                                   # N % 384 == 0, and == 256 (the last tile 256 wide); ragged M
                                   (3300, 3072, 1024), (3000, 3328, 512)])
def test_prefill_linear_vs_oracle(M, N, K):
    x = wl.heavy_tailed_bf16(M, K, M * 7 + K)
    w = wl.normal_bf16(N, K, 0.02, N * 3 + K)
    W = mq.quantize_weight(to_dev(w))
    y = mq.prefill_linear(to_dev(x), W)
    torch.cuda.synchronize()
    y64, sabs = oracle_linear(x, w)
    gemm_check(to_host_bits(y), y64, sabs)


def test_tiny_workload_full_parity():
    p = wl.tiny().projections[0]
    x, w = wl.make_x(p), wl.make_w(p)
    W = mq.quantize_weight(to_dev(w))
    y = mq.prefill_linear(to_dev(x), W)
    torch.cuda.synchronize()
    y64, sabs = oracle_linear(x, w)
    gemm_check(to_host_bits(y), y64, sabs)


def test_prequantized_activation_and_static_alpha():
    M, N, K = 256, 512, 768
    x = wl.heavy_tailed_bf16(M, K, 4)
    w = wl.normal_bf16(N, K, 0.02, 5)
    W = mq.quantize_weight(to_dev(w))
    Xq = mq.quantize_activation(to_dev(x))
    y1 = mq.prefill_linear(W=W, Xq=Xq)
    alpha = torch.tensor([0.05], device="cuda")
    y2 = mq.prefill_linear(to_dev(x), W, alpha_static=alpha)
    torch.cuda.synchronize()
    y64, sabs = oracle_linear(x, w)
    gemm_check(to_host_bits(y1), y64, sabs)
    y64s, sabss = oracle_linear(x, w, alpha_x=float(np.float32(0.05)))
    gemm_check(to_host_bits(y2), y64s, sabss)


def test_workspace_reuse_across_shapes():
    ws = mq.workspace(512, 2048)
    for (M, N, K) in [(512, 256, 2048), (64, 512, 1024), (512, 1024, 2048)]:
        x = wl.heavy_tailed_bf16(M, K, M + N)
        w = wl.normal_bf16(N, K, 0.02, K)
        W = mq.quantize_weight(to_dev(w))
        y = mq.prefill_linear(to_dev(x), W, ws=ws)
        torch.cuda.synchronize()
        y64, sabs = oracle_linear(x, w)
        gemm_check(to_host_bits(y), y64, sabs)
    assert mq.async_status(ws) == 0


def _interleave_perm(I):
    perm = np.empty(2 * I, np.int64)
    for r in range(2 * I):
        c, t = divmod(r, 32)
        perm[r] = 16 * c + t if t < 16 else I + 16 * c + (t - 16)
    return perm


@pytest.mark.parametrize("M,I,K", [(128, 128, 256), (300, 256, 512), (256, 384, 1024)])
def test_fused_silu_mul_requant_epilogue(M, I, K):
    """gate/up GEMM with the SiLU-mul + NVFP4 requantize epilogue, then the down GEMM.

    h itself is compared with tolerance (the GEMM accumulation order and expf
    differ from the oracle's FP64 path); the NVFP4 codes and scales of h must
    equal the oracle's quantization of the GPU's own h bit for bit."""
    x = wl.heavy_tailed_bf16(M, K, 31 + M)
    wgu = wl.normal_bf16(2 * I, K, 0.02, 32 + I)
    wdn = wl.normal_bf16(K, I, 0.02, 33 + I)
    alpha_h = np.float32(0.002)
    Wgu = mq.quantize_weight(to_dev(wgu), gate_up_interleave=True)
    h_dbg = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    H = mq.prefill_linear(to_dev(x), Wgu, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4,
                          alpha_h=torch.tensor([alpha_h], device="cuda"), h_debug=h_dbg)
    H.alpha.fill_(float(alpha_h))
    Wdn = mq.quantize_weight(to_dev(wdn))
    y = mq.prefill_linear(W=Wdn, Xq=H)
    torch.cuda.synchronize()

    # (1) h vs the oracle's SiLU-mul of its own gate/up GEMM
    y64, sabs = oracle_linear(x, wgu)
    h_gpu = to_host_bits(h_dbg)
    silu_mul_check(h_gpu, y64[:, :I], y64[:, I:], sabs[:, :I], sabs[:, I:])
    # (2) codes and scales of h: bit-exact against the oracle quantizing the GPU's h with alpha_h
    codes, scales, _ = nvfp4_host(H)
    rc, rs = oracle.quantize(h_gpu, float(alpha_h))
    assert np.array_equal(scales, rs), f"{int((scales != rs).sum())} h scale mismatches"
    assert np.array_equal(codes, rc), f"{int((codes != rc).sum())} h code mismatches"
    # (3) down projection on the NVFP4 h
    aw = oracle.tensor_alpha(wdn)[1]
    yd64, sabsd = oracle.nvfp4_linear_rows((rc, rs, float(alpha_h)), (*oracle.quantize(wdn, aw), aw))
    gemm_check(to_host_bits(y), yd64, sabsd)


@pytest.mark.parametrize("M,I,K", [(128, 128, 256), (300, 256, 512), (256, 384, 1024), (1000, 192, 320)])
def test_unfused_silu_mul_bf16_epilogue_and_dynamic_alpha_h(M, I, K):
    """The unfused MLP path: gate/up GEMM with a BF16 h output (MQ_EPI_SILU_MUL_BF16), then the
    down projection quantizing h with its own dynamic tensor scale.  h equals the fused
    epilogue's h bit for bit (same arithmetic) and is within the h bound of the oracle; the down
    projection is within the GEMM tolerance of the oracle quantizing the GPU's h with
    alpha_h = amax|h| / 2688."""
    x = wl.heavy_tailed_bf16(M, K, 41 + M)
    wgu = wl.normal_bf16(2 * I, K, 0.02, 42 + I)
    wdn = wl.normal_bf16(K, I, 0.02, 43 + I)
    X = to_dev(x)
    Wgu = mq.quantize_weight(to_dev(wgu), gate_up_interleave=True)
    h_fused = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    mq.prefill_linear(X, Wgu, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=torch.ones(1, device="cuda"),
                      h_debug=h_fused)
    h = mq.prefill_linear(X, Wgu, epilogue=mq.MQ_EPI_SILU_MUL_BF16)
    assert tuple(h.shape) == (M, I)
    Wdn = mq.quantize_weight(to_dev(wdn))
    y = mq.prefill_linear(h, Wdn)                 # dynamic alpha_h: amax + quantize of h
    torch.cuda.synchronize()
    hg = to_host_bits(h)
    assert np.array_equal(hg, to_host_bits(h_fused))
    y64, sabs = oracle_linear(x, wgu)
    silu_mul_check(hg, y64[:, :I], y64[:, I:], sabs[:, :I], sabs[:, I:])
    ah = oracle.tensor_alpha(hg)[1]
    aw = oracle.tensor_alpha(wdn)[1]
    yd64, sabsd = oracle.nvfp4_linear_rows((*oracle.quantize(hg, ah), ah), (*oracle.quantize(wdn, aw), aw))
    gemm_check(to_host_bits(y), yd64, sabsd)


def test_interleaved_weight_plain_epilogue_is_permuted_columns():
    M, I, K = 128, 128, 256
    x = wl.heavy_tailed_bf16(M, K, 5)
    wgu = wl.normal_bf16(2 * I, K, 0.02, 6)
    Wi = mq.quantize_weight(to_dev(wgu), gate_up_interleave=True)
    y = mq.prefill_linear(to_dev(x), Wi)
    torch.cuda.synchronize()
    y64, sabs = oracle_linear(x, wgu)
    perm = _interleave_perm(I)
    gemm_check(to_host_bits(y), y64[:, perm], sabs[:, perm])
