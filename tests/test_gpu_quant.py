"""GPU quantizer (tensor amax + Eq. 2 / Eq. 3 block quantizer) vs the oracle:
codes, block scales and the tensor scale must be bit-exact."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import nvfp4_host, require_gpu, scales_from_layout, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check_quant(x_bits, t, alpha_expected=None):
    codes, scales, alpha = nvfp4_host(t)
    if alpha_expected is None:
        _, alpha_expected, _ = oracle.tensor_alpha(x_bits)
    assert np.float32(alpha) == np.float32(alpha_expected)
    rc, rs = oracle.quantize(x_bits, alpha_expected)
    assert np.array_equal(scales, rs), f"{int((scales != rs).sum())} scale mismatches"
    assert np.array_equal(codes, rc), f"{int((codes != rc).sum())} code byte mismatches"


@pytest.mark.parametrize("M,K,kind", [(128, 256, "normal"), (200, 320, "heavy"), (1, 64, "heavy"),
                                      (129, 4096, "heavy"), (513, 1088, "heavy")])
def test_quantize_activation_bit_exact(M, K, kind):
    x = wl.normal_bf16(M, K, 1.0, 3) if kind == "normal" else wl.heavy_tailed_bf16(M, K, 5)
    t = mq.quantize_activation(to_dev(x))
    torch.cuda.synchronize()
    _check_quant(x, t)


@pytest.mark.parametrize("M,K", [(7, 2048), (64, 2304), (128, 4096), (8, 4352)])
def test_small_activation_launch_shapes_bit_exact(M, K):
    """Small activations are quantized in one launch: up to 16 tiles of 128 x 256 by one
    thread-block cluster exchanging the block maxima through distributed shared memory (8, 9
    and 16 CTAs here, 16 being the non-portable maximum), 17 tiles by the cooperative launch.
    Codes, scales and alpha are bit-exact either way."""
    x = wl.heavy_tailed_bf16(M, K, 17 + M)
    t = mq.quantize_activation(to_dev(x))
    torch.cuda.synchronize()
    _check_quant(x, t)


def test_nonfinite_input_in_a_cluster_quantization():
    """A NaN in a 16-tile activation (one cluster): reported as MQ_ERR_NONFINITE, excluded from
    the tensor amax; the other rows' codes and scales match the oracle with that alpha."""
    x = wl.heavy_tailed_bf16(32, 4096, 23)
    x[17, 3001] = 0x7FC0
    ws = mq.workspace(32, 4096)
    t = mq.quantize_activation(to_dev(x), ws=ws)
    assert mq.async_status(ws) == 5
    amax, ax, bad = oracle.tensor_alpha(x)
    assert bad
    codes, scales, alpha = nvfp4_host(t)
    assert np.float32(alpha) == np.float32(ax)
    ok = np.arange(32) != 17
    rc, rs = oracle.quantize(x[ok], ax)
    assert np.array_equal(codes[ok], rc)
    assert np.array_equal(scales[ok], rs)


def test_tiny_workload_quantization():
    """The tiny 128x256x256 workload: X ~ N(0,1), W ~ N(0, 0.02^2), seed 0."""
    p = wl.tiny().projections[0]
    x, w = wl.make_x(p), wl.make_w(p)
    _check_quant(x, mq.quantize_activation(to_dev(x)))
    _check_quant(w, mq.quantize_weight(to_dev(w)))


def test_golden_blocks_on_gpu():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "handworked_blocks.json")))
    x = np.concatenate([wl.f32_to_bf16_bits(np.asarray(b["x"], np.float32)) for b in g["blocks"]])[None, :]
    t = mq.quantize_activation(to_dev(x))
    codes, scales, alpha = nvfp4_host(t)
    assert alpha == 1.0
    for i, b in enumerate(g["blocks"]):
        assert scales[0, i] == b["sigma_code"], b["name"]
        got = [(int(codes[0, 8 * i + j // 2]) >> (4 * (j % 2))) & 15 for j in range(16)]
        assert got == b["codes"], b["name"]


def test_every_e2m1_tie_and_e4m3_midpoint():
    """Blocks built so that |x|/(alpha sigma) hits every E2M1 tie and the block
    quotient hits E4M3 midpoints (alpha = 1 via a 2688 anchor)."""
    rng = np.random.default_rng(1)
    grid = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = (grid[1:] + grid[:-1]) / 2
    rows = []
    anchor = np.zeros(16, np.float32)
    anchor[0] = 2688.0
    rows.append(anchor)
    for m in mids[mids * 6 < 2000][::2]:
        blk = np.zeros(16, np.float32)
        blk[0] = m * 6           # amax_b / 6 = midpoint (not always BF16-exact; rounding is part of the test)
        ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) * m
        blk[1:8] = ties
        blk[8:15] = -ties
        blk[15] = rng.standard_normal() * m
        rows.append(blk)
    v = np.concatenate(rows)
    pad = (-len(v)) % 64
    v = np.concatenate([v, np.zeros(pad, np.float32)]).reshape(1, -1)
    x = wl.f32_to_bf16_bits(v)
    _check_quant(x, mq.quantize_activation(to_dev(x)))


@pytest.mark.parametrize("alpha", [0.125, 0.1, 1.0 / 6.0, 0.0371, 3.3e-3, 7.5])
def test_block_scale_rounding_near_e4m3_midpoints(alpha):
    """Block maxima placed on and next to every E4M3 rounding midpoint times
    alpha*6 (the BF16 values nearest to it and two BF16 steps either side), for
    several static tensor scales: the block-scale code must match the oracle's
    Pi_E4M3(fl32(amax_b / fl32(alpha*6))) exactly, ties included."""
    a32 = np.float32(alpha)
    aq = np.float32(a32 * np.float32(6.0))
    grid = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = (grid[1:] + grid[:-1]) / 2
    rng = np.random.default_rng(int(alpha * 1e4))
    blocks = []
    for m in mids:
        centre = wl.f32_to_bf16_bits(np.array([m * float(aq)], np.float32))[0]
        for d in (-2, -1, 0, 1, 2):
            b = int(centre) + d
            if not 0 < b < 0x7F80:
                continue
            amax_b = wl.bf16_bits_to_f32(np.array([b], np.uint16))[0]
            blk = (rng.uniform(-1, 1, 16) * amax_b).astype(np.float32)
            blk[rng.integers(16)] = -amax_b if d % 2 else amax_b
            blocks.append(blk)
    v = np.concatenate(blocks)
    v = np.concatenate([v, np.zeros((-len(v)) % 64, np.float32)]).reshape(-1, 64)
    x = wl.f32_to_bf16_bits(v)
    # block maxima must survive the BF16 rounding of the filler values
    t = mq.quantize_activation(to_dev(x), alpha_static=torch.tensor([float(a32)], device="cuda"))
    _check_quant(x, t, alpha_expected=float(a32))


def test_static_alpha_and_saturation():
    x = wl.heavy_tailed_bf16(256, 512, 8)
    alpha = np.float32(0.01)   # far too small: many blocks clip at sigma = 448 and codes at 6
    t = mq.quantize_activation(to_dev(x), alpha_static=torch.tensor([alpha], device="cuda"))
    _check_quant(x, t, alpha_expected=float(alpha))
    _, scales, _ = nvfp4_host(t)
    assert (scales == 0x7E).any()


def test_zero_and_negative_zero_and_tiny():
    x = np.zeros((128, 256), np.uint16)
    x[0, 1] = 0x8000                       # -0.0
    x[1, :16] = wl.f32_to_bf16_bits(np.full(16, 2.0 ** -12, np.float32))
    x[2, :] = wl.f32_to_bf16_bits(np.full(256, -1e-30, np.float32))
    t = mq.quantize_activation(to_dev(x))
    _check_quant(x, t)
    z = mq.quantize_activation(to_dev(np.zeros((64, 64), np.uint16)))
    assert float(z.alpha.cpu()[0]) == 1.0


def test_weight_quantization_and_gate_up_interleave():
    I, K = 256, 512
    w = wl.normal_bf16(2 * I, K, 0.02, 77)
    plain = mq.quantize_weight(to_dev(w))
    _check_quant(w, plain)
    inter = mq.quantize_weight(to_dev(w), gate_up_interleave=True)
    perm = np.empty(2 * I, np.int64)
    for r in range(2 * I):
        c, t = divmod(r, 32)
        perm[r] = 16 * c + t if t < 16 else I + 16 * c + (t - 16)
    codes, scales, alpha = nvfp4_host(inter)
    _, a_ref, _ = oracle.tensor_alpha(w)
    rc, rs = oracle.quantize(w, a_ref)
    assert alpha == a_ref
    assert np.array_equal(codes, rc[perm]) and np.array_equal(scales, rs[perm])


@pytest.mark.parametrize("rows,K,kind", [(128, 256, "heavy"), (200, 1088, "heavy"), (1, 64, "heavy"),
                                         (512, 4096, "weights"), (2048, 12288, "heavy")])
def test_scale_search_bit_exact(rows, K, kind):
    """Opt-in per-block scale search: codes, scales and alpha bit-exact against the oracle's
    search (same binary32 error arithmetic, same tie rule); small inputs take the single-launch
    path, the largest the amax-kernel path."""
    x = wl.normal_bf16(rows, K, 0.02, 91) if kind == "weights" else wl.heavy_tailed_bf16(rows, K, 93)
    t = mq.quantize(to_dev(x), scale_search=True)
    torch.cuda.synchronize()
    codes, scales, alpha = nvfp4_host(t)
    _, a_ref, _ = oracle.tensor_alpha(x)
    assert np.float32(alpha) == np.float32(a_ref)
    rc, rs = oracle.quantize(x, a_ref, search=True)
    assert np.array_equal(scales, rs), f"{int((scales != rs).sum())} scale mismatches"
    assert np.array_equal(codes, rc), f"{int((codes != rc).sum())} code byte mismatches"
    plain_c, plain_s = oracle.quantize(x, a_ref)
    print(f"scale search {rows}x{K}: {100.0 * float((rs != plain_s).mean()):.1f} % of blocks moved")


def test_scale_search_golden_blocks_static_alpha_and_interleave():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scale_search_blocks.json")))
    x = np.concatenate([wl.f32_to_bf16_bits(np.asarray(b["x"], np.float32)) for b in g["blocks"]])[None, :]
    x = np.concatenate([x, np.zeros((1, 64 - x.shape[1] % 64 if x.shape[1] % 64 else 0), np.uint16)], axis=1)
    t = mq.quantize(to_dev(x), alpha_static=torch.ones(1, device="cuda"), scale_search=True)
    torch.cuda.synchronize()
    codes, scales, alpha = nvfp4_host(t)
    assert alpha == 1.0
    for i, b in enumerate(g["blocks"]):
        assert scales[0, i] == b["sigma_code_search"], b["name"]
        got = [(int(codes[0, 8 * i + j // 2]) >> (4 * (j % 2))) & 15 for j in range(16)]
        assert got == b["codes"], b["name"]
    # gate/up interleave with the search
    I, K = 128, 512
    w = wl.normal_bf16(2 * I, K, 0.02, 78)
    inter = mq.quantize(to_dev(w), gate_up_interleave=True, scale_search=True)
    perm = np.empty(2 * I, np.int64)
    for r in range(2 * I):
        c, t_ = divmod(r, 32)
        perm[r] = 16 * c + t_ if t_ < 16 else I + 16 * c + (t_ - 16)
    codes, scales, alpha = nvfp4_host(inter)
    _, a_ref, _ = oracle.tensor_alpha(w)
    rc, rs = oracle.quantize(w, a_ref, search=True)
    assert np.array_equal(codes, rc[perm]) and np.array_equal(scales, rs[perm])


def test_gemm_with_searched_weights_matches_oracle():
    """The GEMM consumes searched scales like any others: parity against the oracle's
    block-scaled matmul on the searched weight."""
    from gpu_helpers import gemm_check
    x = wl.heavy_tailed_bf16(256, 1024, 95)
    w = wl.normal_bf16(512, 1024, 0.02, 96)
    Wq = mq.quantize(to_dev(w), scale_search=True)
    y = mq.prefill_linear(to_dev(x), Wq)
    torch.cuda.synchronize()
    ax = oracle.tensor_alpha(x)[1]
    aw = oracle.tensor_alpha(w)[1]
    y64, sabs = oracle.nvfp4_linear_rows((*oracle.quantize(x, ax), ax), (*oracle.quantize(w, aw, search=True), aw))
    from gpu_helpers import to_host_bits
    gemm_check(to_host_bits(y), y64, sabs)


def test_unswizzle_matches_layout_mapping_and_padding_is_zero():
    x = wl.heavy_tailed_bf16(200, 320, 9)
    t = mq.quantize_activation(to_dev(x))
    dev_rm = mq.unswizzle_scales(t).cpu().numpy()
    buf = t.scales.cpu().numpy()
    assert np.array_equal(dev_rm, scales_from_layout(buf, 200, 320))
    mask = np.zeros(buf.size, bool)
    atoms = 8
    r = np.arange(200)[:, None]
    kb = np.arange(20)[None, :]
    off = ((r // 128) * atoms + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (kb % 4)
    mask[off.ravel()] = True
    assert not buf[~mask].any(), "padding rows / atoms must hold zero scales"


def test_nonfinite_input_is_reported():
    x = wl.heavy_tailed_bf16(128, 256, 2)
    x[5, 7] = 0x7FC0
    ws = mq.workspace()
    mq.quantize_activation(to_dev(x), ws=ws)
    assert mq.async_status(ws) == 5        # MQ_ERR_NONFINITE
    assert mq.async_status(ws) == 0        # cleared
    mq.quantize_activation(to_dev(wl.heavy_tailed_bf16(128, 256, 2)), ws=ws)
    assert mq.async_status(ws) == 0


def test_repeated_amax_on_one_workspace():
    """The amax pass resets its block counter: back-to-back calls on one workspace stay exact."""
    ws = mq.workspace()
    for seed in range(4):
        x = wl.heavy_tailed_bf16(300, 1024, 100 + seed)
        t = mq.quantize_activation(to_dev(x), ws=ws)
        torch.cuda.synchronize()
        _check_quant(x, t)
    assert mq.async_status(ws) == 0


def test_e2m1_conversion_instruction_matches_definition():
    """Every FP32 value in [-8, 8]: the hardware E2M1 rounding equals the comparison-chain definition."""
    assert mq.selftest_e2m1() == (0, 0)


def _interleave_perm(n_rows):
    """Stored row r of a gate/up-interleaved weight -> source row (16-row groups, gate then up)."""
    half = n_rows // 2
    perm = np.empty(n_rows, np.int64)
    for r in range(n_rows):
        c, t = divmod(r, 32)
        perm[r] = 16 * c + t if t < 16 else half + 16 * c + (t - 16)
    return perm


@pytest.mark.parametrize("M,K,interleave", [(2048, 4096, False), (4096, 2048, True), (4173, 16448, False),
                                            (16384, 4096, True)])
def test_lean_quantization_paths_bit_exact(M, K, interleave):
    """The lean tile loop: alone for 128 x 256-aligned tensors of more tiles than SMs (2048 x 4096,
    and a 4096 x 2048 gate/up weight whose interleave maps each warp's 16 rows onto 16 consecutive
    source rows), and for inner tiles beside the regular loop's edge tiles from 2048 tiles (4173 x
    16448: 33 x 65 tiles with a partial last row block and column chunk; a 16384 x 4096 gate/up
    weight).  Codes, scales and alpha bit-exact against the oracle on the first and last 128-row
    blocks and one row in every 128-row block between."""
    x = wl.heavy_tailed_bf16(M, K, 31 + M) if not interleave else wl.normal_bf16(M, K, 0.02, 37 + M)
    X = to_dev(x)
    t = mq.quantize_weight(X, gate_up_interleave=True) if interleave else mq.quantize_activation(X)
    torch.cuda.synchronize()
    codes, scales, alpha = nvfp4_host(t)
    _, a_ref, _ = oracle.tensor_alpha(x)
    assert np.float32(alpha) == np.float32(a_ref)
    rows = np.unique(np.concatenate([np.arange(128), np.arange(M - (M % 128 or 128) - 128, M),
                                     np.arange(128, M, 128) + 37 % 128]))
    rows = rows[rows < M]
    src = _interleave_perm(M)[rows] if interleave else rows
    rc, rs = oracle.quantize(x[src], a_ref)
    assert np.array_equal(scales[rows], rs), f"{int((scales[rows] != rs).sum())} scale mismatches"
    assert np.array_equal(codes[rows], rc), f"{int((codes[rows] != rc).sum())} code byte mismatches"
