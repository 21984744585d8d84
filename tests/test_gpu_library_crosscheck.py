"""The prefill GEMM against a library block-scaled NVFP4 matmul on the same operands.

The oracle is the authority on what the prefill linear computes; this test adds an
independent check of the storage format: torch's NVFP4 matmul (a cuBLASLt kernel)
reads our codes (even k in the low nibble), our E4M3 block scales in the MMA scale
layout (its "32_4_4" swizzle) and our FP32 tensor scales, and must produce the same
BF16 output up to the order of the FP32 accumulation."""
import numpy as np
import pytest
import torch

from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    import torch.nn.functional as F
    if not hasattr(torch, "float4_e2m1fn_x2") or not hasattr(F, "scaled_mm"):
        pytest.skip("this torch build has no NVFP4 scaled_mm")


def library_linear(Xq, W):
    import torch.nn.functional as F
    ST, SW = F.ScalingType, F.SwizzleType
    return F.scaled_mm(Xq.codes.view(torch.float4_e2m1fn_x2), W.codes.view(torch.float4_e2m1fn_x2).t(),
                       [Xq.scales.view(torch.float8_e4m3fn), Xq.alpha], [ST.BlockWise1x16, ST.TensorWise],
                       [W.scales.view(torch.float8_e4m3fn), W.alpha], [ST.BlockWise1x16, ST.TensorWise],
                       swizzle_a=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE], swizzle_b=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE],
                       output_dtype=torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(256, 512, 1024), (300, 640, 512), (8192, 1024, 4096)])
def test_prefill_linear_matches_library_nvfp4_matmul(M, N, K):
    x = to_dev(wl.heavy_tailed_bf16(M, K, 9100 + M))
    w = to_dev(wl.normal_bf16(N, K, 0.02, 9200 + N))
    ws = mq.workspace(M, K)
    W = mq.quantize_weight(w, ws=ws)
    Xq = mq.quantize_activation(x, ws=ws)
    y = mq.prefill_linear(W=W, Xq=Xq, ws=ws)
    yl = library_linear(Xq, W)
    torch.cuda.synchronize()
    assert mq.async_status(ws) == 0
    yo, yr = y.double(), yl.double()
    rel = float(torch.linalg.norm(yo - yr) / torch.linalg.norm(yr))
    assert rel <= 1e-3, rel
    # Same products, different FP32 summation order: most outputs round to the same BF16.
    same = float((y.view(torch.int16) == yl.view(torch.int16)).double().mean())
    assert same >= 0.5, same
    assert np.isfinite(rel)
