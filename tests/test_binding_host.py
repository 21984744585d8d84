"""The Python binding's argument marshalling, on CPU.

Host tensors stand in for device buffers: the library validates every argument
on the host before it touches the device, so a call whose arguments the
binding marshals correctly gets as far as the device check and fails there
(MQ_ERR_CUDA or MQ_ERR_DEVICE without a GPU), while a call the binding
marshals wrongly, or whose arguments are wrong, fails validation first
(MQ_ERR_SHAPE, MQ_ERR_INVALID_ARG, MQ_ERR_WORKSPACE).  Nothing here runs a kernel."""
from types import SimpleNamespace

import pytest
import torch

from phase_aware_nvfp4_b200 import mixquant as mq

NO_DEVICE = (7, 8)          # MQ_ERR_CUDA, MQ_ERR_DEVICE
STREAM = SimpleNamespace(cuda_stream=0)


@pytest.fixture(scope="module", autouse=True)
def _host_only():
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the device check would pass and kernels would run on host pointers")
    import os
    if not os.path.exists(mq.LIB_PATH):
        from phase_aware_nvfp4_b200 import build
        build.build()


def status_of(fn, *a, **k):
    with pytest.raises(mq.MQError) as e:
        fn(*a, stream=STREAM, **k)
    return e.value.status


def nvfp4_host(rows, cols):
    cb, sb = mq.nvfp4_sizes(rows, cols) if cols % 64 == 0 else (rows * cols // 2, 4096)
    return mq.NVFP4Tensor(torch.zeros((rows, cols // 2), dtype=torch.uint8), torch.zeros(sb, dtype=torch.uint8),
                          torch.zeros(1, dtype=torch.float32), rows, cols)


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def ws_for(M=0, K=0):
    return torch.zeros(mq.workspace_bytes(M, K), dtype=torch.uint8)


def test_prefill_linear_marshals_shapes_and_workspace():
    W = nvfp4_host(256, 256)
    X, Y = bf16(128, 256), bf16(128, 256)
    assert status_of(mq.prefill_linear, X, W, Y=Y, ws=ws_for(128, 256)) in NO_DEVICE
    # the workspace must hold the NVFP4 copy of X: the binding passes its true size
    assert status_of(mq.prefill_linear, X, W, Y=Y, ws=ws_for()) == 4
    # an NVFP4 X (no quantization in the workspace) needs only the control block
    assert status_of(mq.prefill_linear, W=W, Xq=nvfp4_host(128, 256), Y=Y, ws=ws_for()) in NO_DEVICE
    assert status_of(mq.prefill_linear, X, nvfp4_host(256, 200), Y=Y, ws=ws_for(128, 256)) == 2
    # fused epilogue: H must be [M, N/2]
    H = nvfp4_host(128, 128)
    a = torch.ones(1)
    assert status_of(mq.prefill_linear, X, W, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=a, H=H,
                     ws=ws_for(128, 256)) in NO_DEVICE
    assert status_of(mq.prefill_linear, X, W, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=a, H=nvfp4_host(128, 256),
                     ws=ws_for(128, 256)) == 2
    with pytest.raises(ValueError):
        mq.prefill_linear(X, W, Xq=nvfp4_host(128, 256), Y=Y, ws=ws_for(128, 256))


def test_kv_rope_marshals_table_and_cache_sizes():
    H, M, K = 2, 64, 256
    W = nvfp4_host(2 * H * 128, K)
    args = dict(n_kv_heads=H, positions=torch.zeros(M, dtype=torch.int32), slots=torch.zeros(M, dtype=torch.int64),
                ws=ws_for(M, K))
    cs, kc, vc = torch.zeros((512, 128)), bf16(M, H, 128), bf16(M, H, 128)
    assert status_of(mq.prefill_kv_rope, bf16(M, K), W, cos_sin=cs, k_cache=kc, v_cache=vc, **args) in NO_DEVICE
    args["n_kv_heads"] = 3
    assert status_of(mq.prefill_kv_rope, bf16(M, K), W, cos_sin=cs, k_cache=kc, v_cache=vc, **args) == 2


def test_kv_rope_passes_table_rows_and_cache_rows(monkeypatch):
    """max_pos is the cos/sin table's row count and num_slots the cache's (seen through a
    stand-in for the library that records what it is given)."""
    seen = {}

    class Lib:
        def mq_prefill_kv_rope(self, *a):
            seen["args"] = a
            return 0
    H, M, K = 1, 16, 256
    W, ws, wsb = nvfp4_host(256, K), ws_for(M, K), mq.workspace_bytes(M, K)
    monkeypatch.setattr(mq, "load", lambda: Lib())
    mq.prefill_kv_rope(bf16(M, K), W, n_kv_heads=H, positions=torch.zeros(M, dtype=torch.int32),
                       cos_sin=torch.zeros((777, 128)), slots=torch.zeros(M, dtype=torch.int64),
                       k_cache=bf16(99, H, 128), v_cache=bf16(99, H, 128), ws=ws, stream=STREAM)
    a = seen["args"]
    assert a[2] == M and a[4] == H and a[7] == 777 and a[11] == 99
    assert a[13].value == wsb


def test_decode_and_quantize_entries_marshal_their_limits():
    W = bf16(256, 256)
    assert status_of(mq.decode_linear, bf16(8, 256), W, Y=bf16(8, 256), ws=ws_for()) in NO_DEVICE
    assert status_of(mq.decode_linear, bf16(300, 256), W, Y=bf16(300, 256), ws=ws_for()) == 2
    Wq = nvfp4_host(256, 256)
    assert status_of(mq.decode_linear_nvfp4, bf16(128, 256), Wq, Y=bf16(128, 256), ws=ws_for(128, 256)) in NO_DEVICE
    assert status_of(mq.decode_linear_nvfp4, bf16(129, 256), Wq, Y=bf16(129, 256), ws=ws_for(129, 256)) == 2
    assert status_of(mq.quantize, bf16(200, 256), scale_search=True, out=nvfp4_host(200, 256),
                     ws=ws_for()) in NO_DEVICE
    assert status_of(mq.quantize, bf16(200, 256), gate_up_interleave=True, out=nvfp4_host(200, 256),
                     ws=ws_for()) == 2
    assert status_of(mq.quantize_weight, bf16(256, 256), out=nvfp4_host(256, 256), ws=ws_for()) in NO_DEVICE
    assert status_of(mq.quantize_activation, bf16(64, 256), out=nvfp4_host(64, 128), ws=ws_for()) == 2
    g = bf16(256)
    assert status_of(mq.rmsnorm_quantize, bf16(64, 256), g, 1e-6, out=nvfp4_host(64, 256),
                     ws=ws_for(64, 256)) in NO_DEVICE
    assert status_of(mq.rmsnorm_quantize, bf16(64, 256), g, -1.0, out=nvfp4_host(64, 256), ws=ws_for(64, 256)) == 1
