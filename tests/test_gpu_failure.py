"""Failure detection on the GPU without a fault: a bounded pipeline wait that
runs out must surface as MQ_ERR_TIMEOUT through the workspace status, and the
context must stay usable afterwards."""
import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import nvfp4_host, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = mq.workspace()
    assert mq.async_status(ws) == 0
    waited = mq.selftest_timeout(ws, 2_000_000)         # 2 ms; nothing ever arrives
    assert 2_000_000 <= waited < 1_000_000_000, waited
    assert mq.async_status(ws) == 6                     # MQ_ERR_TIMEOUT
    assert mq.async_status(ws) == 0                     # read clears it
    # the same workspace and context still produce exact results
    x = wl.heavy_tailed_bf16(256, 512, 21)
    t = mq.quantize_activation(to_dev(x), ws=ws)
    torch.cuda.synchronize()
    codes, scales, alpha = nvfp4_host(t)
    _, a_ref, _ = oracle.tensor_alpha(x)
    rc, rs = oracle.quantize(x, a_ref)
    assert np.float32(alpha) == np.float32(a_ref)
    assert np.array_equal(codes, rc) and np.array_equal(scales, rs)
    assert mq.async_status(ws) == 0


def test_timeout_status_is_per_workspace():
    ws_a, ws_b = mq.workspace(), mq.workspace()
    mq.selftest_timeout(ws_a, 1_000_000)
    assert mq.async_status(ws_b) == 0
    assert mq.async_status(ws_a) == 6
