"""Guard bands around every output buffer (a stand-in for a memory checker,
which is not available on the GPU pool): each entry point runs on ragged
shapes with its outputs and its workspace placed in the middle of larger
buffers whose head and tail are filled with a sentinel byte; after the call
the sentinels must be intact, so no kernel wrote before or past the end of
any buffer it was given.  The shapes cover the single-launch and two-launch
quantizers, both GEMM kernels (at most 128 rows, CTA pairs), the fused MLP
and KV epilogues, both decode paths and the RMSNorm producer, with M, N and
K off the tile sizes.
"""
import numpy as np
import pytest
import torch

from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import require_gpu, to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (a multiple of 256 keeps every view 256-byte aligned)
SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


class Guarded:
    """`shape` of `dtype` in the middle of a byte buffer with sentinel-filled guards."""
    registry = []

    def __init__(self, shape, dtype, fill=SENTINEL, name=""):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n, self.name = n, name
        self.buf = torch.full((GUARD + (n + 255) // 256 * 256 + GUARD,), SENTINEL, dtype=torch.uint8,
                              device="cuda")
        inner = self.buf[GUARD:GUARD + n]
        if fill != SENTINEL:
            inner.fill_(fill)
        self.t = inner.view(dtype).view(shape)
        Guarded.registry.append(self)

    def intact(self):
        b = self.buf.cpu().numpy()
        head, tail = b[:GUARD], b[GUARD + self.n:]
        return bool((head == SENTINEL).all() and (tail == SENTINEL).all())


def nvfp4_guarded(rows, cols, name):
    _, sb = mq.nvfp4_sizes(rows, cols)
    return mq.NVFP4Tensor(Guarded((rows, cols // 2), torch.uint8, name=name + ".codes").t,
                          Guarded((sb,), torch.uint8, fill=0, name=name + ".scales").t,
                          Guarded((1,), torch.float32, fill=0, name=name + ".alpha").t, rows, cols)


def ws_guarded(M=0, K=0):
    return Guarded((mq.workspace_bytes(M, K),), torch.uint8, fill=0, name="workspace").t


@pytest.fixture(autouse=True)
def _check_guards():
    Guarded.registry = []
    yield
    torch.cuda.synchronize()
    broken = [g.name for g in Guarded.registry if not g.intact()]
    assert not broken, f"guard bands overwritten: {broken}"


def _x(M, K, seed):
    return to_dev(wl.heavy_tailed_bf16(M, K, seed))


@pytest.mark.parametrize("M,K", [(200, 320), (1, 64), (3000, 2112)])
def test_quantize_activation(M, K):
    ws = ws_guarded()
    out = nvfp4_guarded(M, K, "X")
    mq.quantize_activation(_x(M, K, M + K), out=out, ws=ws)
    assert mq.async_status(ws) == 0


def test_quantize_weight_interleaved_and_scale_search():
    ws = ws_guarded()
    w = to_dev(wl.normal_bf16(384, 320, 0.02, 9))
    mq.quantize_weight(w, gate_up_interleave=True, out=nvfp4_guarded(384, 320, "Wgu"), ws=ws)
    mq.quantize(w[:200], scale_search=True, out=nvfp4_guarded(200, 320, "Wsearch"), ws=ws)
    assert mq.async_status(ws) == 0


@pytest.mark.parametrize("M,N,K", [(200, 336, 320), (100, 272, 4096), (1, 16, 64)])
def test_prefill_linear_bf16(M, N, K):
    ws = ws_guarded(M, K)
    W = mq.quantize_weight(to_dev(wl.normal_bf16(N, K, 0.02, N)), out=nvfp4_guarded(N, K, "W"))
    Y = Guarded((M, N), torch.bfloat16, name="Y").t
    mq.prefill_linear(_x(M, K, M), W, Y=Y, ws=ws)
    assert mq.async_status(ws) == 0


@pytest.mark.parametrize("M,I,K", [(300, 192, 512), (100, 128, 256)])
def test_prefill_linear_fused_mlp(M, I, K):
    ws = ws_guarded(M, K)
    Wgu = mq.quantize_weight(to_dev(wl.normal_bf16(2 * I, K, 0.02, I)), gate_up_interleave=True)
    H = nvfp4_guarded(M, I, "H")
    h_dbg = Guarded((M, I), torch.bfloat16, name="h_debug").t
    ah = torch.tensor([0.002], device="cuda")
    mq.prefill_linear(_x(M, K, M), Wgu, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=ah, H=H, h_debug=h_dbg, ws=ws)
    assert mq.async_status(ws) == 0


@pytest.mark.parametrize("M,N,K", [(7, 400, 320), (200, 272, 4096)])
def test_decode_linear_bf16(M, N, K):
    ws = ws_guarded()
    Y = Guarded((M, N), torch.bfloat16, name="Y").t
    mq.decode_linear(_x(M, K, M), to_dev(wl.normal_bf16(N, K, 0.02, N)), Y=Y, ws=ws)
    assert mq.async_status(ws) == 0


@pytest.mark.parametrize("M,N,K", [(7, 400, 320), (100, 272, 4096), (3, 400, 2048), (1, 272, 8192)])
def test_decode_linear_nvfp4(M, N, K):
    ws = ws_guarded(M, K)
    W = mq.quantize_weight(to_dev(wl.normal_bf16(N, K, 0.02, N)))
    Y = Guarded((M, N), torch.bfloat16, name="Y").t
    mq.decode_linear_nvfp4(_x(M, K, M), W, Y=Y, ws=ws)
    assert mq.async_status(ws) == 0


@pytest.mark.parametrize("M,K", [(200, 320), (1, 64)])
def test_rmsnorm_quantize(M, K):
    ws = ws_guarded(M, K)
    gamma = to_dev(wl.normal_bf16(1, K, 1.0, 3)[0])
    h_dbg = Guarded((M, K), torch.bfloat16, name="h_debug").t
    mq.rmsnorm_quantize(_x(M, K, M), gamma, 1e-6, out=nvfp4_guarded(M, K, "h"), h_debug=h_dbg, ws=ws)
    assert mq.async_status(ws) == 0


@pytest.mark.parametrize("M,H,K", [(200, 2, 320), (100, 1, 256)])
def test_prefill_kv_rope(M, H, K):
    ws = ws_guarded(M, K)
    W = mq.quantize_weight(to_dev(wl.normal_bf16(2 * H * 128, K, 0.02, H)))
    cs = torch.from_numpy(wl.rope_cos_sin(512)).cuda()
    pos = torch.randint(0, 512, (M,), dtype=torch.int32, device="cuda")
    slots = torch.randperm(M + 5, device="cuda")[:M].contiguous()
    kc = Guarded((M + 5, H, 128), torch.bfloat16, fill=0, name="k_cache").t
    vc = Guarded((M + 5, H, 128), torch.bfloat16, fill=0, name="v_cache").t
    mq.prefill_kv_rope(_x(M, K, M), W, n_kv_heads=H, positions=pos, cos_sin=cs, slots=slots, k_cache=kc,
                       v_cache=vc, ws=ws)
    assert mq.async_status(ws) == 0


def test_unswizzle_scales():
    t = mq.quantize_activation(_x(200, 320, 1))
    out = Guarded((200, 20), torch.uint8, name="rowmajor").t
    mq.unswizzle_scales(t, out=out)
