"""mq_prefill_linear_noalloc: the prefill linear layer without a workspace.

This entry point exists for callers that cannot hand the library any device
memory of their own for scratch -- an inference-engine plugin that is not
allowed to allocate when it is enqueued (the engine owns the memory), or a
latency-critical serving loop that must never call cudaMalloc because it can
synchronize the device.  Its scratch lives in a static device array of the
library instead.

The test drives it through the C ABI on three calls in a row on the one
static array (dynamic scale with the single-launch amax, a static scale, and
a dynamic scale on an activation with more quantizer tiles than SMs, which
takes the two-launch amax and fills 54 MB of the 64 MB array).  Each output
is checked against the regular entry point's output on the same inputs,
within the GEMM tolerance of the other parity tests and, since both run the
same kernels on the same data, bit for bit; and against the oracle on one row
of every 128-row block.  An activation too large for the array is refused.

The file name sorts last so a stop-at-first-failure run reaches it only after
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import REL_FROB_MAX, block_rows, gemm_check, require_gpu, to_dev, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _call_noalloc(x, W, alpha_static, y):
    """Call the C entry point directly (ctypes), with the current torch stream."""
    lib = mq.load()
    wc = W.c()
    st = lib.mq_prefill_linear_noalloc(ctypes.c_void_p(x.data_ptr()), x.shape[0], ctypes.byref(wc),
                                       None if alpha_static is None else ctypes.c_void_p(alpha_static.data_ptr()),
                                       ctypes.c_void_p(y.data_ptr()),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _close(y_bits, y_ref_bits):
    a, b = oracle.bf16_to_f64(y_bits), oracle.bf16_to_f64(y_ref_bits)
    assert oracle.rel_frobenius(a, b) <= REL_FROB_MAX
    assert np.all(np.abs(a - b) <= oracle.bf16_ulp(b))


def test_noalloc_matches_workspace_entry_point_and_oracle_on_three_calls():
    cases = [(384, 512, 1024, None), (1000, 272, 4096, 0.04), (8192, 512, 12288, None)]
    for M, N, K, alpha in cases:                 # calls in a row on the same static scratch
        x = wl.heavy_tailed_bf16(M, K, M + K)
        w = wl.normal_bf16(N, K, 0.02, N + 3)
        X = to_dev(x)
        W = mq.quantize_weight(to_dev(w))
        a = None if alpha is None else torch.tensor([alpha], device="cuda")
        y_ref = mq.prefill_linear(X, W, alpha_static=a)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(X, W, a, y) == 0
        torch.cuda.synchronize()
        yb, yrb = to_host_bits(y), to_host_bits(y_ref)
        _close(yb, yrb)
        assert np.array_equal(yb, yrb), f"{int((yb != yrb).sum())} outputs differ from mq_prefill_linear"
        # the oracle on one row of every 128-row block (plus the first and last rows)
        rows = block_rows(M, seed=M)
        ax = np.float32(alpha) if alpha is not None else oracle.tensor_alpha(x)[1]
        aw = oracle.tensor_alpha(w)[1]
        y64, sabs = oracle.nvfp4_linear_rows((*oracle.quantize(x[rows], float(ax)), float(ax)),
                                             (*oracle.quantize(w, aw), aw))
        gemm_check(yb[rows], y64, sabs)


def test_noalloc_rejects_activation_beyond_the_static_scratch():
    K = 16384
    M = mq.NOALLOC_SCRATCH_BYTES // (K // 2) + 1      # the codes alone exceed the array
    W = mq.nvfp4_empty(16, K)
    x = torch.empty((1, 8), dtype=torch.bfloat16, device="cuda")   # never read: rejected before launch
    y = torch.empty((1, 8), dtype=torch.bfloat16, device="cuda")
    lib = mq.load()
    wc = W.c()
    st = lib.mq_prefill_linear_noalloc(ctypes.c_void_p(x.data_ptr()), M, ctypes.byref(wc), None,
                                       ctypes.c_void_p(y.data_ptr()), None)
    assert st == 4      # MQ_ERR_WORKSPACE
