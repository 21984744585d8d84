"""The C ABI library on a machine without a GPU: it loads, exports every
declared symbol, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from phase_aware_nvfp4_b200 import mixquant as mqb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mixquant.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(mqb.LIB_PATH):
        from phase_aware_nvfp4_b200 import build
        build.build()
    return mqb.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MQ_API\s+[\w\s\*]+?\b(mq_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(mqb.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_only_mq_symbols_are_exported(lib):
    out = os.popen(f"nm -D --defined-only {mqb.LIB_PATH}").read()
    names = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared_symbols()) <= names
    assert all(n.startswith("mq_") for n in names), sorted(n for n in names if not n.startswith("mq_"))


def test_status_strings_and_version(lib):
    for code, name in mqb.STATUS_NAMES.items():
        assert lib.mq_status_string(code).decode() == name
    assert lib.mq_version().decode() == "0.1.0"


def test_sizes(lib):
    cb, sb = mqb.nvfp4_sizes(8192, 4096)
    assert cb == 8192 * 2048
    assert sb == 64 * 16 * 2048            # 64 row blocks x 16 chunks of 4 atoms
    cb, sb = mqb.nvfp4_sizes(200, 320)
    assert cb == 200 * 160
    assert sb == 2 * 8 * 512               # 320 cols -> 2 chunks of 256 -> 8 atoms per row block
    assert mqb.workspace_bytes(0, 0) == mqb.WS_CONTROL_BYTES
    assert mqb.workspace_bytes(8192, 4096) >= mqb.WS_CONTROL_BYTES + cb
    with pytest.raises(mqb.MQError):
        mqb.nvfp4_sizes(8, 100)
    # decode workspace: the NVFP4 token copy, then 8 splits x 96 tiles x M x 128 FP32 partials
    # (the per-tile counters live in the control block)
    wq = mqb.workspace_bytes(4, 4096)
    assert mqb.decode_workspace_bytes(4, 12288, 4096) == -(-wq // 256) * 256 + 8 * 96 * 4 * 128 * 4
    assert mqb.decode_workspace_bytes(0, 12288, 4096) == mqb.WS_CONTROL_BYTES


class _NV(ctypes.Structure):
    _fields_ = mqb._NVFP4._fields_


def _nv(rows, cols, base=0x10000000):
    return mqb._NVFP4(base, base + 0x1000000, base + 0x2000000, rows, cols)


def test_argument_errors_are_synchronous(lib):
    """Validation happens on the host before any launch; no GPU is needed to see it."""
    P = 0x7F0000000000
    ws, wsb = ctypes.c_void_p(P), ctypes.c_size_t(1 << 30)
    w = _nv(256, 256)
    # null / bad enum
    assert lib.mq_prefill_linear(None, None, 128, ctypes.byref(w), 0, None, None, P, None, None, ws, wsb, None) == 1
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 7, None, None, P, None, None, ws, wsb, None) == 1
    # shapes: K % 64, N % 16, M range
    bad_k = _nv(256, 200)
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(bad_k), 0, None, None, P, None, None, ws, wsb, None) == 2
    bad_n = _nv(250, 256)
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(bad_n), 0, None, None, P, None, None, ws, wsb, None) == 2
    assert lib.mq_prefill_linear(P, None, 0, ctypes.byref(w), 0, None, None, P, None, None, ws, wsb, None) == 2
    # alignment
    assert lib.mq_prefill_linear(P + 2, None, 128, ctypes.byref(w), 0, None, None, P, None, None, ws, wsb,
                                 None) == 3
    # workspace too small for in-workspace activation quantization
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 0, None, None, P, None, None, ws,
                                 ctypes.c_size_t(100), None) == 4
    # fused epilogue needs N % 128 and an H_out of [M, N/2]
    h = _nv(128, 128)
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 1, None, P, None, None, None, ws, wsb, None) == 1
    h_bad = _nv(128, 64)
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 1, None, P, None, ctypes.byref(h_bad), None, ws,
                                 wsb, None) == 2
    # unfused MLP epilogue (BF16 h into Y): needs Y and N % 128; epilogue 3 does not exist
    w336 = _nv(336, 256)
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w336), 2, None, None, P, None, None, ws, wsb, None) == 2
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 2, None, None, None, None, None, ws, wsb, None) == 1
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 2, None, None, P + 8, None, None, ws, wsb, None) == 3
    assert lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 3, None, None, P, None, None, ws, wsb, None) == 1
    # decode: M in [1, 256]
    assert lib.mq_decode_linear(P, 300, P, 256, 256, P, ws, wsb, None) == 2
    assert lib.mq_decode_linear(P, 4, P, 256, 100, P, ws, wsb, None) == 2
    assert lib.mq_decode_linear(None, 4, P, 256, 256, P, ws, wsb, None) == 1
    # weight quantization: interleave needs N % 128
    out = _nv(200, 256)
    assert lib.mq_quantize_weight(P, 200, 256, 1, ctypes.byref(out), ws, wsb, None) == 2
    assert lib.mq_quantize_weight(P, 200, 256, 0, None, ws, wsb, None) == 1
    assert lib.mq_async_status(None, None) == 1
    # general quantization entry: unknown flag bits, interleave needs rows % 128
    q = _nv(200, 256)
    assert lib.mq_quantize(P, 200, 256, None, ctypes.c_uint(4), ctypes.byref(q), ws, wsb, None) == 1
    assert lib.mq_quantize(P, 200, 256, None, ctypes.c_uint(1), ctypes.byref(q), ws, wsb, None) == 2
    assert lib.mq_quantize(P + 2, 200, 256, None, ctypes.c_uint(2), ctypes.byref(q), ws, wsb, None) == 3
    # fused RMSNorm + quantization: gamma required, eps finite >= 0, K % 64
    rq = _nv(128, 256)
    assert lib.mq_rmsnorm_quantize(P, 128, 256, None, ctypes.c_float(1e-6), ctypes.byref(rq), None, ws, wsb,
                                   None) == 1
    assert lib.mq_rmsnorm_quantize(P, 128, 256, P, ctypes.c_float(-1.0), ctypes.byref(rq), None, ws, wsb, None) == 1
    assert lib.mq_rmsnorm_quantize(P, 128, 200, P, ctypes.c_float(1e-6), ctypes.byref(rq), None, ws, wsb, None) == 2
    assert lib.mq_rmsnorm_quantize(P, 128, 256, P + 8, ctypes.c_float(1e-6), ctypes.byref(rq), None, ws, wsb,
                                   None) == 3
    # K/V projection with RoPE: W rows = 2 * heads * 128, index arrays and caches required/aligned
    wkv = _nv(512, 256)
    args = lambda X, heads, pos, cs, sl, kc: (X, None, 128, ctypes.byref(wkv), heads, pos, cs, 1024, sl, kc, P,
                                               4096, ws, wsb, None)
    assert lib.mq_prefill_kv_rope(*args(P, 3, P, P, P, P)) == 2             # 2 * 3 * 128 != 512
    assert lib.mq_prefill_kv_rope(*args(P, 2, None, P, P, P)) == 1
    assert lib.mq_prefill_kv_rope(*args(P, 2, P + 2, P, P, P)) == 3          # positions 4-byte aligned
    assert lib.mq_prefill_kv_rope(*args(P, 2, P, P, P + 4, P)) == 3          # slots 8-byte aligned
    assert lib.mq_prefill_kv_rope(*args(P, 2, P, P + 4, P, P)) == 3          # cos/sin 16-byte aligned
    assert lib.mq_prefill_kv_rope(*args(None, 2, P, P, P, P)) == 1           # neither X nor X_q
    # sizes beyond 2^30 in any dimension are refused by every entry point
    big, bigk = (1 << 30) + 128, (1 << 30) + 64
    ob = _nv(big, 256)
    assert lib.mq_quantize_weight(P, big, 256, 0, ctypes.byref(ob), ws, wsb, None) == 2
    assert lib.mq_quantize_weight(P, 256, bigk, 0, ctypes.byref(_nv(256, bigk)), ws, wsb, None) == 2
    assert lib.mq_quantize_activation(P, big, 256, None, ctypes.byref(ob), ws, wsb, None) == 2
    assert lib.mq_quantize(P, big, 256, None, ctypes.c_uint(0), ctypes.byref(ob), ws, wsb, None) == 2
    assert lib.mq_prefill_linear(P, None, big, ctypes.byref(w), 0, None, None, P, None, None, ws, wsb, None) == 2
    assert lib.mq_decode_linear(P, 4, P, big, 256, P, ws, wsb, None) == 2
    assert lib.mq_rmsnorm_quantize(P, big, 256, P, ctypes.c_float(1e-6), ctypes.byref(ob), None, ws, wsb, None) == 2
    # timeout self-test: timeout in (0, 2 s], a workspace, an aligned result slot
    assert lib.mq_selftest_timeout(ws, wsb, ctypes.c_uint64(0), None, None) == 1
    assert lib.mq_selftest_timeout(ws, wsb, ctypes.c_uint64(3 * 10 ** 9), None, None) == 1
    assert lib.mq_selftest_timeout(None, wsb, ctypes.c_uint64(10 ** 6), None, None) == 4
    assert lib.mq_selftest_timeout(ws, wsb, ctypes.c_uint64(10 ** 6), ctypes.c_void_p(P + 4), None) == 3
    del h


def test_noalloc_refuses_exactly_what_the_workspace_entry_point_refuses(lib):
    """mq_prefill_linear_noalloc and mq_prefill_linear (BF16 X, BF16 epilogue) give the same
    status for the same bad argument, before anything touches a device."""
    P = 0x7F0000000000
    ws, wsb = ctypes.c_void_p(P), ctypes.c_size_t(1 << 30)

    def both(X, M, w, Y):
        a = lib.mq_prefill_linear(X, None, M, ctypes.byref(w), 0, None, None, Y, None, None, ws, wsb, None)
        b = lib.mq_prefill_linear_noalloc(X, M, ctypes.byref(w), None, Y, None)
        return a, b

    ok = _nv(256, 256)
    cases = {
        "alpha misaligned": (P, 128, mqb._NVFP4(P, P + 0x100000, P + 0x200002, 256, 256), P, 3),
        "codes misaligned": (P, 128, mqb._NVFP4(P + 8, P + 0x100000, P + 0x200000, 256, 256), P, 3),
        "null scales": (P, 128, mqb._NVFP4(P, 0, P + 0x200000, 256, 256), P, 1),
        "K % 64": (P, 128, _nv(256, 200), P, 2),
        "N % 16": (P, 128, _nv(250, 256), P, 2),
        "M = 0": (P, 0, ok, P, 2),
        "M > 2^30": (P, (1 << 30) + 1, ok, P, 2),
        "K > 2^30": (P, 128, _nv(256, (1 << 30) + 64), P, 2),
        "X misaligned": (P + 2, 128, ok, P, 3),
        "Y misaligned": (P, 128, ok, P + 2, 3),
        "Y null": (P, 128, ok, None, 1),
        "X null": (None, 128, ok, P, 1),
    }
    for name, (X, M, w, Y, want) in cases.items():
        assert both(X, M, w, Y) == (want, want), name


def test_valid_call_without_gpu_reports_cuda_or_device_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    P = 0x7F0000000000
    w = _nv(256, 256)
    st = lib.mq_prefill_linear(P, None, 128, ctypes.byref(w), 0, None, None, P, None, None, ctypes.c_void_p(P),
                               ctypes.c_size_t(1 << 30), None)
    assert st in (7, 8)


def test_binding_raises_when_library_missing(tmp_path):
    saved = mqb._lib
    try:
        mqb._lib = None
        with pytest.raises(FileNotFoundError):
            mqb.load(str(tmp_path / "nope.so"))
    finally:
        mqb._lib = saved
