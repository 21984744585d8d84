"""Thin ctypes binding of libmixquant (include/mixquant.h).

Argument marshalling only: every step of the path runs in the CUDA library.
PyTorch provides the device buffers (``torch.empty`` on the current CUDA
device) and the stream (``torch.cuda.current_stream()``).  The binding never
computes anything itself and has no fallback: if ``libmixquant.so`` is
missing or a call returns an error, it raises.

Names mirror the C ABI: ``quantize_weight``, ``quantize_activation``,
``quantize`` (general entry: gate/up interleave, opt-in scale search),
``prefill_linear`` (BF16 or fused SiLU-mul + NVFP4 epilogue),
``prefill_linear_noalloc``, ``prefill_kv_rope``, ``rmsnorm_quantize``,
``decode_linear`` (BF16), ``decode_linear_nvfp4``, ``unswizzle_scales``,
``async_status``, ``selftest_e2m1``, ``selftest_timeout``, ``nvfp4_sizes``,
``workspace_bytes``, ``decode_workspace_bytes``.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmixquant.so")

MQ_OK = 0
MQ_EPI_BF16 = 0
MQ_EPI_SILU_MUL_NVFP4 = 1
MQ_EPI_SILU_MUL_BF16 = 2
WS_CONTROL_BYTES = 16384

STATUS_NAMES = {0: "MQ_OK", 1: "MQ_ERR_INVALID_ARG", 2: "MQ_ERR_SHAPE", 3: "MQ_ERR_ALIGNMENT",
                4: "MQ_ERR_WORKSPACE", 5: "MQ_ERR_NONFINITE", 6: "MQ_ERR_TIMEOUT", 7: "MQ_ERR_CUDA",
                8: "MQ_ERR_DEVICE", 9: "MQ_ERR_INDEX"}

# Every symbol the header declares (checked by the ABI tests).
EXPORTS = ("mq_status_string", "mq_version", "mq_nvfp4_sizes", "mq_workspace_bytes", "mq_quantize_weight",
           "mq_quantize_activation", "mq_prefill_linear", "mq_decode_linear", "mq_unswizzle_scales",
           "mq_async_status", "mq_prefill_linear_noalloc", "mq_selftest_e2m1", "mq_selftest_timeout",
           "mq_decode_linear_nvfp4", "mq_quantize", "mq_rmsnorm_quantize", "mq_prefill_kv_rope",
           "mq_decode_workspace_bytes")
NOALLOC_SCRATCH_BYTES = 64 << 20


class MQError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = int(status)
        super().__init__(f"{call} failed: {STATUS_NAMES.get(self.status, self.status)}")


class _NVFP4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


_lock = threading.Lock()
_lib = None


def load(path: str = LIB_PATH):
    """Load libmixquant.so (raises FileNotFoundError if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise FileNotFoundError(
                    f"{path} is missing: build it with `python -m phase_aware_nvfp4_b200.build`")
            lib = ctypes.CDLL(path)
            vp, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
            nvp = ctypes.POINTER(_NVFP4)
            lib.mq_status_string.argtypes = [i32]
            lib.mq_status_string.restype = ctypes.c_char_p
            lib.mq_version.argtypes = []
            lib.mq_version.restype = ctypes.c_char_p
            lib.mq_nvfp4_sizes.argtypes = [i64, i64, ctypes.POINTER(sz), ctypes.POINTER(sz)]
            lib.mq_nvfp4_sizes.restype = i32
            lib.mq_workspace_bytes.argtypes = [i64, i64]
            lib.mq_workspace_bytes.restype = sz
            lib.mq_decode_workspace_bytes.argtypes = [i64, i64, i64]
            lib.mq_decode_workspace_bytes.restype = sz
            lib.mq_quantize_weight.argtypes = [vp, i64, i64, i32, nvp, vp, sz, vp]
            lib.mq_quantize_weight.restype = i32
            lib.mq_quantize_activation.argtypes = [vp, i64, i64, vp, nvp, vp, sz, vp]
            lib.mq_quantize_activation.restype = i32
            lib.mq_prefill_linear.argtypes = [vp, nvp, i64, nvp, i32, vp, vp, vp, nvp, vp, vp, sz, vp]
            lib.mq_prefill_linear.restype = i32
            lib.mq_decode_linear.argtypes = [vp, i64, vp, i64, i64, vp, vp, sz, vp]
            lib.mq_decode_linear.restype = i32
            lib.mq_unswizzle_scales.argtypes = [nvp, vp, vp]
            lib.mq_unswizzle_scales.restype = i32
            lib.mq_async_status.argtypes = [vp, vp]
            lib.mq_async_status.restype = i32
            lib.mq_selftest_e2m1.argtypes = [vp, vp]
            lib.mq_selftest_e2m1.restype = i32
            lib.mq_selftest_timeout.argtypes = [vp, sz, ctypes.c_uint64, vp, vp]
            lib.mq_selftest_timeout.restype = i32
            lib.mq_decode_linear_nvfp4.argtypes = [vp, i64, nvp, vp, vp, vp, sz, vp]
            lib.mq_decode_linear_nvfp4.restype = i32
            lib.mq_quantize.argtypes = [vp, i64, i64, vp, ctypes.c_uint, nvp, vp, sz, vp]
            lib.mq_quantize.restype = i32
            lib.mq_rmsnorm_quantize.argtypes = [vp, i64, i64, vp, ctypes.c_float, nvp, vp, vp, sz, vp]
            lib.mq_rmsnorm_quantize.restype = i32
            lib.mq_prefill_kv_rope.argtypes = [vp, nvp, i64, nvp, i64, vp, vp, i64, vp, vp, vp, i64, vp, sz, vp]
            lib.mq_prefill_kv_rope.restype = i32
            lib.mq_prefill_linear_noalloc.argtypes = [vp, i64, nvp, vp, vp, vp]
            lib.mq_prefill_linear_noalloc.restype = i32
            _lib = lib
    return _lib


def _check(status: int, call: str):
    if status != MQ_OK:
        raise MQError(status, call)


def _torch():
    import torch
    return torch


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# ----------------------------------------------------------------- tensors

@dataclass
class NVFP4Tensor:
    """Device buffers of an NVFP4 [rows, cols] tensor (layout in include/mixquant.h)."""
    codes: object    # torch.uint8 [rows, cols/2]
    scales: object   # torch.uint8 [scales_bytes] in the MMA scale layout
    alpha: object    # torch.float32 [1]
    rows: int
    cols: int

    def c(self) -> _NVFP4:
        return _NVFP4(self.codes.data_ptr(), self.scales.data_ptr(), self.alpha.data_ptr(), self.rows, self.cols)


def nvfp4_sizes(rows: int, cols: int):
    cb, sb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(load().mq_nvfp4_sizes(rows, cols, ctypes.byref(cb), ctypes.byref(sb)), "mq_nvfp4_sizes")
    return cb.value, sb.value


def workspace_bytes(M: int = 0, K: int = 0) -> int:
    return int(load().mq_workspace_bytes(M, K))


def nvfp4_empty(rows: int, cols: int, device=None) -> NVFP4Tensor:
    torch = _torch()
    device = device or torch.device("cuda", torch.cuda.current_device())
    cb, sb = nvfp4_sizes(rows, cols)
    return NVFP4Tensor(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                       torch.zeros(sb, dtype=torch.uint8, device=device),
                       torch.zeros(1, dtype=torch.float32, device=device), rows, cols)


def decode_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load().mq_decode_workspace_bytes(M, N, K))


def decode_workspace(M: int, N: int, K: int, device=None):
    """A zero-filled workspace for the decode calls on M tokens and an [N, K] weight."""
    torch = _torch()
    device = device or torch.device("cuda", torch.cuda.current_device())
    return torch.zeros(decode_workspace_bytes(M, N, K), dtype=torch.uint8, device=device)


def workspace(M: int = 0, K: int = 0, device=None):
    """A zero-filled workspace for an M x K activation (16-byte aligned)."""
    torch = _torch()
    device = device or torch.device("cuda", torch.cuda.current_device())
    return torch.zeros(workspace_bytes(M, K), dtype=torch.uint8, device=device)


def _ws_args(ws):
    return _ptr(ws), ctypes.c_size_t(ws.numel())


# ----------------------------------------------------------------- calls

def quantize_weight(W, gate_up_interleave: bool = False, out: NVFP4Tensor | None = None, ws=None,
                    stream=None) -> NVFP4Tensor:
    """mq_quantize_weight: BF16 [N, K] -> NVFP4 (offline, dynamic alpha_w)."""
    N, K = W.shape
    out = out or nvfp4_empty(N, K, W.device)
    ws = ws if ws is not None else workspace(device=W.device)
    cs = out.c()
    _check(load().mq_quantize_weight(_ptr(W), N, K, int(bool(gate_up_interleave)), ctypes.byref(cs),
                                     *_ws_args(ws), _stream(stream)), "mq_quantize_weight")
    return out


MQ_QUANT_GATE_UP_INTERLEAVE = 1
MQ_QUANT_SCALE_SEARCH = 2


def quantize(X, alpha_static=None, gate_up_interleave: bool = False, scale_search: bool = False,
             out: NVFP4Tensor | None = None, ws=None, stream=None) -> NVFP4Tensor:
    """mq_quantize: BF16 [rows, K] -> NVFP4, optionally with the per-block scale search."""
    rows, K = X.shape
    out = out or nvfp4_empty(rows, K, X.device)
    ws = ws if ws is not None else workspace(device=X.device)
    flags = (MQ_QUANT_GATE_UP_INTERLEAVE if gate_up_interleave else 0) | (MQ_QUANT_SCALE_SEARCH if scale_search else 0)
    oc = out.c()
    _check(load().mq_quantize(_ptr(X), rows, K, _ptr(alpha_static), flags, ctypes.byref(oc), *_ws_args(ws),
                              _stream(stream)), "mq_quantize")
    return out


def prefill_kv_rope(X=None, W: NVFP4Tensor = None, *, Xq: NVFP4Tensor | None = None, n_kv_heads: int,
                    positions, cos_sin, slots, k_cache, v_cache, ws=None, stream=None):
    """mq_prefill_kv_rope: K/V projection with RoPE on K, BF16 K/V written to cache slots."""
    if (X is None) == (Xq is None):
        raise ValueError("give exactly one of X (BF16) and Xq (NVFP4)")
    M = X.shape[0] if X is not None else Xq.rows
    dev = W.codes.device
    if ws is None:
        ws = workspace(M, W.cols, dev) if X is not None else workspace(device=dev)
    xq_c = Xq.c() if Xq is not None else None
    w_c = W.c()
    _check(load().mq_prefill_kv_rope(_ptr(X), ctypes.byref(xq_c) if xq_c is not None else None, M,
                                     ctypes.byref(w_c), n_kv_heads, _ptr(positions), _ptr(cos_sin),
                                     cos_sin.shape[0], _ptr(slots), _ptr(k_cache), _ptr(v_cache), k_cache.shape[0],
                                     *_ws_args(ws), _stream(stream)), "mq_prefill_kv_rope")


def rmsnorm_quantize(X, gamma, eps: float = 1e-6, out: NVFP4Tensor | None = None, h_debug=None, ws=None,
                     stream=None) -> NVFP4Tensor:
    """mq_rmsnorm_quantize: NVFP4 copy of RMSNorm(X) * gamma without writing the BF16 norm output."""
    M, K = X.shape
    out = out or nvfp4_empty(M, K, X.device)
    ws = ws if ws is not None else workspace(M, K, X.device)
    oc = out.c()
    _check(load().mq_rmsnorm_quantize(_ptr(X), M, K, _ptr(gamma), ctypes.c_float(eps), ctypes.byref(oc),
                                      _ptr(h_debug), *_ws_args(ws), _stream(stream)), "mq_rmsnorm_quantize")
    return out


def quantize_activation(X, alpha_static=None, out: NVFP4Tensor | None = None, ws=None,
                        stream=None) -> NVFP4Tensor:
    """mq_quantize_activation: BF16 [M, K] -> NVFP4 (dynamic alpha unless alpha_static)."""
    M, K = X.shape
    out = out or nvfp4_empty(M, K, X.device)
    ws = ws if ws is not None else workspace(device=X.device)
    cs = out.c()
    _check(load().mq_quantize_activation(_ptr(X), M, K, _ptr(alpha_static), ctypes.byref(cs), *_ws_args(ws),
                                         _stream(stream)), "mq_quantize_activation")
    return out


def prefill_linear(X=None, W: NVFP4Tensor = None, *, Xq: NVFP4Tensor | None = None, epilogue: int = MQ_EPI_BF16,
                   alpha_static=None, alpha_h=None, Y=None, H: NVFP4Tensor | None = None, h_debug=None, ws=None,
                   stream=None):
    """mq_prefill_linear.  Returns Y (BF16 [M, N]; BF16 h [M, N/2] with MQ_EPI_SILU_MUL_BF16)
    or H (NVFP4 [M, N/2])."""
    torch = _torch()
    if (X is None) == (Xq is None):
        raise ValueError("give exactly one of X (BF16) and Xq (NVFP4)")
    M = X.shape[0] if X is not None else Xq.rows
    K = W.cols
    N = W.rows
    dev = W.codes.device
    if ws is None:
        ws = workspace(M, K, dev) if X is not None else workspace(device=dev)
    xq_c = Xq.c() if Xq is not None else None
    w_c = W.c()
    h_c = None
    if epilogue == MQ_EPI_BF16:
        Y = Y if Y is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    elif epilogue == MQ_EPI_SILU_MUL_BF16:
        Y = Y if Y is not None else torch.empty((M, N // 2), dtype=torch.bfloat16, device=dev)
    else:
        H = H or nvfp4_empty(M, N // 2, dev)
        h_c = H.c()
    _check(load().mq_prefill_linear(_ptr(X), ctypes.byref(xq_c) if xq_c is not None else None, M,
                                    ctypes.byref(w_c), int(epilogue), _ptr(alpha_static), _ptr(alpha_h),
                                    _ptr(Y) if epilogue != MQ_EPI_SILU_MUL_NVFP4 else None,
                                    ctypes.byref(h_c) if h_c is not None else None, _ptr(h_debug), *_ws_args(ws),
                                    _stream(stream)), "mq_prefill_linear")
    return H if epilogue == MQ_EPI_SILU_MUL_NVFP4 else Y


def prefill_linear_noalloc(X, W: NVFP4Tensor, alpha_static=None, Y=None, stream=None):
    """mq_prefill_linear_noalloc: prefill linear without a workspace (static device scratch)."""
    torch = _torch()
    M = X.shape[0]
    Y = Y if Y is not None else torch.empty((M, W.rows), dtype=torch.bfloat16, device=X.device)
    w_c = W.c()
    _check(load().mq_prefill_linear_noalloc(_ptr(X), M, ctypes.byref(w_c), _ptr(alpha_static), _ptr(Y),
                                            _stream(stream)), "mq_prefill_linear_noalloc")
    return Y


def decode_linear(X, W, Y=None, ws=None, stream=None):
    """mq_decode_linear: BF16 Y[M, N] = X[M, K] W[N, K]^T (M <= 256)."""
    torch = _torch()
    M, K = X.shape
    N = W.shape[0]
    Y = Y if Y is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    ws = ws if ws is not None else decode_workspace(M, N, K, X.device)
    _check(load().mq_decode_linear(_ptr(X), M, _ptr(W), N, K, _ptr(Y), *_ws_args(ws), _stream(stream)),
           "mq_decode_linear")
    return Y


def decode_linear_nvfp4(X, W: NVFP4Tensor, alpha_static=None, Y=None, ws=None, stream=None):
    """mq_decode_linear_nvfp4: Y[M, N] = X[M, K] W^T with X quantized on the fly and W NVFP4 (M <= 128)."""
    torch = _torch()
    M = X.shape[0]
    Y = Y if Y is not None else torch.empty((M, W.rows), dtype=torch.bfloat16, device=X.device)
    ws = ws if ws is not None else decode_workspace(M, W.rows, W.cols, X.device)
    w_c = W.c()
    _check(load().mq_decode_linear_nvfp4(_ptr(X), M, ctypes.byref(w_c), _ptr(alpha_static), _ptr(Y), *_ws_args(ws),
                                         _stream(stream)), "mq_decode_linear_nvfp4")
    return Y


def unswizzle_scales(t: NVFP4Tensor, out=None, stream=None):
    """mq_unswizzle_scales: MMA scale layout -> row-major uint8 [rows, cols/16]."""
    torch = _torch()
    out = out if out is not None else torch.empty((t.rows, t.cols // 16), dtype=torch.uint8,
                                                  device=t.scales.device)
    cs = t.c()
    _check(load().mq_unswizzle_scales(ctypes.byref(cs), _ptr(out), _stream(stream)), "mq_unswizzle_scales")
    return out


def selftest_e2m1(stream=None):
    """mq_selftest_e2m1: (mismatches on positive inputs, on negative inputs); both should be 0."""
    torch = _torch()
    counts = torch.zeros(2, dtype=torch.int64, device=torch.device("cuda", torch.cuda.current_device()))
    _check(load().mq_selftest_e2m1(_ptr(counts), _stream(stream)), "mq_selftest_e2m1")
    c = counts.cpu().tolist()
    return int(c[0]), int(c[1])


def selftest_timeout(ws, timeout_ns: int, stream=None) -> int:
    """mq_selftest_timeout: a bounded wait that runs out; returns the nanoseconds waited.
    Read the posted MQ_ERR_TIMEOUT with async_status(ws)."""
    torch = _torch()
    waited = torch.zeros(1, dtype=torch.int64, device=ws.device)
    _check(load().mq_selftest_timeout(*_ws_args(ws), ctypes.c_uint64(int(timeout_ns)), _ptr(waited), _stream(stream)),
           "mq_selftest_timeout")
    return int(waited.cpu()[0])


def async_status(ws, stream=None) -> int:
    """mq_async_status: synchronize the stream, return and clear the device error bits."""
    return int(load().mq_async_status(_ptr(ws), _stream(stream)))
