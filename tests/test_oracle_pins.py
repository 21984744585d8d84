"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one oracle function against something the format
definitions or the mathematics fix: library decoders of the same format,
exhaustive enumeration, brute force on tiny inputs, hand-worked blocks
(tests/golden/handworked_blocks.json), closed forms of the matmul on
grid-valued inputs, and invariants of Eq. 2 / Eq. 3 of "Mix-Quant: Quantized
Prefilling, Precise Decoding for Agentic LLMs", section 3.3.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1_POS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP FP4 E2M1 magnitudes


def bf16(vals):
    return wl.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


# ------------------------------------------------------------------ formats

def test_e2m1_decode_table():
    vals = [oracle.e2m1_value(c) for c in range(16)]
    assert vals[:8] == E2M1_POS
    assert vals[8:] == [-v for v in E2M1_POS]
    assert math.copysign(1.0, vals[8]) == -1.0        # code 0x8 is -0


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(mine[~nan], ref[~nan])


def test_e4m3_decode_landmarks():
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0x08) == 2.0 ** -6      # smallest normal
    assert oracle.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9  # largest subnormal


def _finite_e4m3_sorted():
    return [(oracle.e4m3_value(c), c) for c in range(0x7F)]


def test_e4m3_round_matches_torch_rne():
    """Pi_E4M3 (Eq. 3) = torch's float32 -> float8_e4m3fn cast (RNE) on [0, 448]."""
    rng = np.random.default_rng(11)
    s = np.exp2(rng.uniform(-14, 9, 200000)).astype(np.float32)
    grid = np.array([v for v, _ in _finite_e4m3_sorted()], dtype=np.float64)
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)          # every tie, exact in fp32
    s = np.concatenate([s, mids, grid.astype(np.float32), [0.0, 448.0]]).astype(np.float32)
    s = s[s <= 448.0]
    ref = torch.from_numpy(s).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_round(float(v)) for v in s], dtype=np.uint8)
    assert np.array_equal(mine, ref)


def test_e4m3_round_saturates():
    for v in (448.0, 449.0, 463.9, 464.0, 1e6, float("inf")):
        assert oracle.e4m3_round(v) == 0x7E


def test_e2m1_round_brute_force():
    """Pi_FP4 magnitude = brute-force nearest of the 8 magnitudes, ties to even index."""
    rng = np.random.default_rng(3)
    m = np.concatenate([rng.uniform(0, 7, 20000), np.linspace(0, 6.5, 2601),
                        [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]]).astype(np.float32)
    for v in m:
        x = float(v)
        d = [abs(p - x) for p in E2M1_POS]
        best = min(d)
        cands = [i for i, di in enumerate(d) if di == best]
        want = 7 if x >= 6.0 else ([i for i in cands if i % 2 == 0] or cands)[0]
        assert oracle.e2m1_round(x) == want, x


def test_e2m1_tie_table():
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for m, idx in ties.items():
        assert oracle.e2m1_round(m) == idx


def test_bf16_rounding_known_values():
    one = 1.0
    cases = {
        one: 0x3F80,
        one + 2.0 ** -8: 0x3F80,            # tie -> even
        one + 3 * 2.0 ** -8: 0x3F82,        # tie -> even (up)
        one + 2.0 ** -8 + 2.0 ** -30: 0x3F81,
        -2.0: 0xC000,
        2.0 ** -133: 0x0001,                # smallest subnormal
        2.0 ** -134: 0x0000,                # tie with 0 -> even (0)
        3 * 2.0 ** -134: 0x0002,            # tie between 1 and 2 quanta -> 2
        (2 - 2.0 ** -7) * 2.0 ** 127: 0x7F7F,
        (2 - 2.0 ** -8) * 2.0 ** 127: 0x7F80,  # rounds to +inf
    }
    for v, bits in cases.items():
        assert int(oracle.round_bf16(np.array([v]))[0]) == bits, v


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(100000) * np.exp2(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(oracle.round_bf16(v.astype(np.float64)), ref)


# ------------------------------------------------------------- Eq. 2 / 3

def _golden_row():
    g = json.load(open(os.path.join(GOLDEN, "handworked_blocks.json")))
    x = np.concatenate([bf16(b["x"]) for b in g["blocks"]])[None, :]
    return g, x


def test_handworked_blocks():
    g, x = _golden_row()
    amax, alpha, bad = oracle.tensor_alpha(x)
    assert (amax, alpha, bad) == (2688.0, g["alpha"], False)
    codes, scales = oracle.quantize(x, alpha)
    xhat = oracle.dequantize(codes, scales, alpha)[0]
    for i, b in enumerate(g["blocks"]):
        assert scales[0, i] == b["sigma_code"], b["name"]
        assert oracle.e4m3_value(int(scales[0, i])) == b["sigma"]
        got = []
        for j in range(16):
            byte = int(codes[0, i * 8 + j // 2])
            got.append(byte & 15 if j % 2 == 0 else byte >> 4)
        assert got == b["codes"], b["name"]
        assert list(xhat[16 * i:16 * i + 16]) == [float(v) for v in b["xhat"]], b["name"]


def test_nibble_order_even_k_low():
    x = np.zeros((1, 16), dtype=np.uint16)
    x[0, :2] = bf16([6.0, -3.0])     # amax 6; alpha = 6/2688
    _, alpha, _ = oracle.tensor_alpha(x)
    codes, _ = oracle.quantize(x, alpha)
    assert codes[0, 0] == 0x7 | (0xD << 4)


def test_tensor_alpha_special_cases():
    z = np.zeros((4, 32), dtype=np.uint16)
    assert oracle.tensor_alpha(z) == (0.0, 1.0, False)
    x = bf16(np.linspace(-3, 5, 64)).reshape(2, 32)
    x[1, 3] = 0x7FC0  # NaN
    amax, _, bad = oracle.tensor_alpha(x)
    assert bad and amax == 5.0
    x[1, 3] = 0xFF80  # -inf
    assert oracle.tensor_alpha(x)[2]


def test_alpha_prevents_global_saturation():
    """With alpha = amax/(6*448) the block holding the tensor amax gets sigma = 448 and no block exceeds it."""
    for seed in range(5):
        x = wl.heavy_tailed_bf16(64, 256, seed)
        amax, alpha, _ = oracle.tensor_alpha(x)
        _, scales = oracle.quantize(x, alpha)
        sig = np.array([oracle.e4m3_value(int(c)) for c in np.unique(scales)])
        assert sig.max() == 448.0
        flat = np.abs(wl.bf16_bits_to_f32(x)).reshape(64, -1, 16).max(axis=2)
        r, b = np.unravel_index(np.argmax(flat), flat.shape)
        assert scales[r, b] == 0x7E


def test_block_scale_is_nearest_e4m3_of_exact_quotient():
    """Eq. 3 in fp32 picks the E4M3 value nearest to the exact quotient amax_b/(6 alpha).

    The only allowed difference is at a near-tie: when the exact quotient lies
    within a few fp32 ulps of the midpoint of two E4M3 neighbours, the two
    fp32 roundings (of alpha*6 and of the quotient) may land on the tie and
    pick the even neighbour.  Both candidates are then the two neighbours.
    """
    x = wl.heavy_tailed_bf16(256, 256, 7)
    amax, alpha, _ = oracle.tensor_alpha(x)
    _, scales = oracle.quantize(x, alpha)
    grid = _finite_e4m3_sorted()
    vals = [Fraction(v) for v, _ in grid]
    xf = np.abs(wl.bf16_bits_to_f32(x)).reshape(256, 16, 16).max(axis=2)
    a6 = Fraction(float(np.float32(alpha))) * 6
    near_ties = 0
    for r in range(256):
        for b in range(16):
            q = Fraction(float(xf[r, b])) / a6
            best = min(grid, key=lambda vc: (abs(Fraction(vc[0]) - q), vc[1] & 1))
            want = best[1] if q < 448 else 0x7E
            if scales[r, b] == want:
                continue
            # must be a near-tie between two adjacent E4M3 values
            i = int(np.searchsorted(np.array([float(v) for v in vals]), float(q)))
            lo, hi = vals[i - 1], vals[i]
            mid = (lo + hi) / 2
            assert abs(q - mid) <= mid * Fraction(1, 2 ** 21), (float(q), float(mid))
            assert int(scales[r, b]) in (grid[i - 1][1], grid[i][1])
            near_ties += 1
    assert near_ties < 0.02 * 256 * 16


def test_elements_on_grid_and_error_bound():
    """Every xhat = +-alpha*sigma*v, and |x - xhat| <= d*(half local step) for normal unsaturated scales."""
    x = wl.heavy_tailed_bf16(128, 512, 9)
    _, alpha, _ = oracle.tensor_alpha(x)
    codes, scales = oracle.quantize(x, alpha)
    xhat = oracle.dequantize(codes, scales, alpha)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    sig = np.vectorize(oracle.e4m3_value)(scales.astype(np.int64)).repeat(16, axis=1)
    d = (np.float32(alpha) * sig.astype(np.float32)).astype(np.float64)   # fl32(alpha*sigma)
    d_exact = np.float64(np.float32(alpha)) * sig                         # alpha*sigma, exact in fp64
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(d_exact > 0, xhat / np.where(d_exact > 0, d_exact, 1.0), 0.0)
    assert np.all(np.isin(np.abs(v), E2M1_POS))
    # half the local grid step at |x|/d
    m = np.where(d > 0, np.abs(xf) / d, 0.0)
    half = np.where(m <= 2.0, 0.25, np.where(m <= 4.0, 0.5, 1.0))
    normal = sig >= 2.0 ** -6
    err = np.abs(xf - xhat)
    bound = d * half * (1 + 2.0 ** -20) + np.abs(xf) * 2.0 ** -22
    clipped = m > 6.0
    ok = (err <= bound) | ~normal | clipped
    assert ok.all()
    # clipped elements: rounding sigma to E4M3 costs at most 2^-4 relative, so |x|/d <= 6.4
    assert np.all(m[normal] <= 6.0 * (1 + 2.0 ** -4) + 1e-6)


def test_frobenius_error_bound():
    x = wl.heavy_tailed_bf16(64, 1024, 4)
    _, alpha, _ = oracle.tensor_alpha(x)
    c, s = oracle.quantize(x, alpha)
    xhat = oracle.dequantize(c, s, alpha)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    amax_b = np.abs(xf).reshape(64, -1, 16).max(axis=2)
    assert np.sum((xf - xhat) ** 2) <= 16 * np.sum((1.0625 * amax_b / 6) ** 2)


def test_requantize_is_idempotent():
    """Re-quantizing xhat of blocks whose max code is +-6 returns the same codes and scales."""
    x = wl.heavy_tailed_bf16(32, 256, 12)
    x[0, 0] = bf16([2688.0])[0]          # amax = 6*448 -> alpha = 1, so xhat = sigma*v is BF16-exact
    amax, alpha, _ = oracle.tensor_alpha(x)
    assert amax == 2688.0 and alpha == 1.0
    c, s = oracle.quantize(x, alpha)
    xhat = oracle.dequantize(c, s, alpha)
    xh = oracle.round_bf16(xhat)
    assert np.array_equal(oracle.bf16_to_f64(xh), xhat)
    c2, s2 = oracle.quantize(xh, alpha)
    lo, hi = c & 15, c >> 4
    mags = np.stack([lo & 7, hi & 7], axis=-1).reshape(32, -1, 16)
    full = mags.max(axis=2) == 7
    assert np.array_equal(s2[full], s[full])
    cm = c.reshape(32, -1, 8)
    assert np.array_equal(c2.reshape(32, -1, 8)[full], cm[full])


def test_rtn_quotient_reading_agrees_with_exact_division():
    """|x| * fl(1/fl(alpha*sigma)) picks the same code as the exact quotient except at near-ties."""
    x = wl.heavy_tailed_bf16(256, 512, 21)
    _, alpha, _ = oracle.tensor_alpha(x)
    c, s = oracle.quantize(x, alpha)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    sig = np.vectorize(oracle.e4m3_value)(s.astype(np.int64)).repeat(16, axis=1)
    d = np.float64(np.float32(np.float32(alpha) * sig.astype(np.float32)))
    m = np.where(d > 0, np.abs(xf) / np.where(d > 0, d, 1), 0)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    idx = np.searchsorted(mids, m, side="left")
    tie = np.isin(m, mids)
    idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)   # exact ties -> even index
    idx = np.minimum(idx, 7)
    lo, hi = c & 15, c >> 4
    got = np.stack([lo & 7, hi & 7], axis=-1).reshape(idx.shape)
    frac = np.mean(got != idx)
    assert frac <= 1e-5


# ------------------------------------------------------------------ matmuls

def _grid_matrix(rows, K, rng, with_anchor):
    """Values on the E2M1 grid, each 16-block holding a +-6, so sigma = 1 when alpha = 1."""
    v = rng.choice(np.array(E2M1_POS + [-p for p in E2M1_POS[1:]]), size=(rows, K))
    v = v.reshape(rows, K // 16, 16)
    v[:, :, 0] = rng.choice([6.0, -6.0], size=(rows, K // 16))
    v = v.reshape(rows, K)
    if with_anchor:                        # one block [2688, 0...] makes amax = 6*448 -> alpha = 1
        v[0, :16] = 0.0
        v[0, 0] = 2688.0
    return v


def test_gemm_closed_form_on_grid_inputs():
    rng = np.random.default_rng(17)
    M, N, K = 24, 40, 256
    xv = _grid_matrix(M, K, rng, True)
    wv = _grid_matrix(N, K, rng, True)
    xb, wb = bf16(xv), bf16(wv)
    ax, aw = oracle.tensor_alpha(xb)[1], oracle.tensor_alpha(wb)[1]
    assert ax == 1.0 and aw == 1.0
    xq = (*oracle.quantize(xb, ax), ax)
    wq = (*oracle.quantize(wb, aw), aw)
    y, sabs = oracle.nvfp4_linear_rows(xq, wq)
    # exact: every value is a multiple of 1/2, so 4*x*w sums are integers
    xi = [[int(Fraction(v) * 2) for v in row] for row in xv]
    wi = [[int(Fraction(v) * 2) for v in row] for row in wv]
    for m in range(M):
        for n in range(N):
            exact = Fraction(sum(a * b for a, b in zip(xi[m], wi[n])), 4)
            assert y[m, n] == float(exact)
            assert sabs[m, n] == float(Fraction(sum(abs(a * b) for a, b in zip(xi[m], wi[n])), 4))
    assert np.array_equal(oracle.round_bf16(y), oracle.round_bf16(np.array(y)))


def test_gemm_tensor_scales_multiply_out():
    """Scaling X by 2^e scales alpha_x by 2^e and leaves codes/scales unchanged (exact)."""
    x = wl.heavy_tailed_bf16(16, 128, 30)
    w = wl.normal_bf16(8, 128, 0.02, 31)
    xs = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(x) * np.float32(8.0))
    a1, a2 = oracle.tensor_alpha(x)[1], oracle.tensor_alpha(xs)[1]
    assert a2 == 8 * a1
    c1, s1 = oracle.quantize(x, a1)
    c2, s2 = oracle.quantize(xs, a2)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    aw = oracle.tensor_alpha(w)[1]
    wq = (*oracle.quantize(w, aw), aw)
    y1, _ = oracle.nvfp4_linear_rows((c1, s1, a1), wq)
    y2, _ = oracle.nvfp4_linear_rows((c2, s2, a2), wq)
    assert np.array_equal(8 * y1, y2)


def test_bf16_linear_exact_on_small_integers():
    rng = np.random.default_rng(2)
    xi = rng.integers(-8, 9, size=(5, 64))
    wi = rng.integers(-8, 9, size=(7, 64))
    y = oracle.bf16_linear_rows(bf16(xi), bf16(wi))
    assert np.array_equal(y, (xi @ wi.T).astype(np.float64))


def test_nvfp4_vs_bf16_error_is_bounded_by_quantization_error():
    """|Y_nvfp4 - Y_exact| <= |X - Xhat||W| + |Xhat||W - What| row by row (Cauchy-Schwarz)."""
    x = wl.heavy_tailed_bf16(32, 512, 40)
    w = wl.normal_bf16(48, 512, 0.02, 41)
    ax, aw = oracle.tensor_alpha(x)[1], oracle.tensor_alpha(w)[1]
    xq = (*oracle.quantize(x, ax), ax)
    wq = (*oracle.quantize(w, aw), aw)
    y, _ = oracle.nvfp4_linear_rows(xq, wq)
    yb = oracle.bf16_linear_rows(x, w)
    xf, wf = oracle.bf16_to_f64(x), oracle.bf16_to_f64(w)
    xh, wh = oracle.dequantize(*xq), oracle.dequantize(*wq)
    ex = np.linalg.norm(xf - xh, axis=1)[:, None] * np.linalg.norm(wf, axis=1)[None, :]
    ew = np.linalg.norm(xh, axis=1)[:, None] * np.linalg.norm(wf - wh, axis=1)[None, :]
    assert np.all(np.abs(y - yb) <= (ex + ew) * (1 + 1e-9))
    assert oracle.rel_frobenius(y, yb) < 0.2


def test_silu_mul_against_torch():
    rng = np.random.default_rng(8)
    g = rng.standard_normal(50000) * 6
    u = rng.standard_normal(50000) * 3
    h = oracle.bf16_to_f64(oracle.silu_mul(g, u))
    gf = torch.from_numpy(g.astype(np.float32).astype(np.float64))
    ref = (torch.nn.functional.silu(gf) * torch.from_numpy(u.astype(np.float32).astype(np.float64))).numpy()
    assert np.all(np.abs(h - ref) <= oracle.bf16_ulp(ref) * 0.5 + np.abs(ref) * 2.0 ** -22)
    assert oracle.silu_mul(np.array([0.0]), np.array([5.0]))[0] == 0


def test_bf16_ulp():
    assert oracle.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert oracle.bf16_ulp(np.array([3.0]))[0] == 2.0 ** -6
    assert oracle.bf16_ulp(np.array([0.0]))[0] == 2.0 ** -133


@pytest.mark.parametrize("mutation", ["drop_sign", "ties_away"])
def test_pins_catch_planted_mistakes(mutation):
    """A plausible slip in the encode step is caught by the hand-worked golden blocks."""
    g, x = _golden_row()
    _, alpha, _ = oracle.tensor_alpha(x)
    codes, _ = oracle.quantize(x, alpha)
    lo, hi = codes & 15, codes >> 4
    got = np.stack([lo, hi], axis=-1).reshape(-1)
    want = np.concatenate([b["codes"] for b in g["blocks"]])
    assert np.array_equal(got, want)
    if mutation == "drop_sign":
        planted = got & 7
    else:  # round ties away from zero instead of to even
        xf = np.abs(wl.bf16_bits_to_f32(x[0]).astype(np.float64))
        planted = got.copy()
        for i, v in enumerate(xf[16:32]):   # block B has alpha = sigma = 1
            planted[16 + i] = (got[16 + i] & 8) | int(np.argmin([abs(p - v) - 1e-9 * p for p in E2M1_POS]))
    assert not np.array_equal(planted, want)


# ------------------------------------------------------------------ opt-in scale search

def test_scale_search_handworked_blocks():
    g = json.load(open(os.path.join(GOLDEN, "scale_search_blocks.json")))
    for b in g["blocks"]:
        x = bf16(b["x"]).reshape(1, 16)
        assert np.array_equal(wl.bf16_bits_to_f32(x).ravel(), np.asarray(b["x"], np.float32)), b["name"]
        c0, s0 = oracle.quantize(x, g["alpha"])
        c1, s1 = oracle.quantize(x, g["alpha"], search=True)
        assert int(s0[0, 0]) == b["sigma_code_rne"], b["name"]
        assert int(s1[0, 0]) == b["sigma_code_search"], b["name"]
        got = [(int(c1[0, j // 2]) >> (4 * (j % 2))) & 15 for j in range(16)]
        assert got == b["codes"], b["name"]


def test_scale_search_never_worse_than_eq3_and_stays_next_to_it():
    """Exact (FP64) block error of the searched scale <= that of the Eq. 3 scale, up to the
    binary32 rounding of the search metric; the chosen code is c0 - 1, c0 or c0 + 1."""
    for seed in range(3):
        x = wl.heavy_tailed_bf16(96, 512, 40 + seed)
        _, alpha, _ = oracle.tensor_alpha(x)
        c0, s0 = oracle.quantize(x, alpha)
        c1, s1 = oracle.quantize(x, alpha, search=True)
        assert np.all(np.abs(s1.astype(np.int64) - s0.astype(np.int64)) <= 1)
        xf = wl.bf16_bits_to_f32(x).astype(np.float64)
        e0 = ((oracle.dequantize(c0, s0, alpha) - xf) ** 2).reshape(96, -1, 16).sum(axis=2)
        e1 = ((oracle.dequantize(c1, s1, alpha) - xf) ** 2).reshape(96, -1, 16).sum(axis=2)
        assert np.all(e1 <= e0 * (1 + 2.0 ** -18) + 1e-30)
        assert e1.sum() < e0.sum()                     # the search does help on heavy-tailed data
        changed = s1 != s0
        assert changed.any() and np.all(e1[changed] < e0[changed] * (1 + 2.0 ** -18))


def test_scale_search_output_is_on_the_grid_of_its_scale():
    """With the searched scale the codes are still Eq. 2's nearest grid points (the same invariant
    as the Eq. 3 path: |x - xhat| <= half the local step unless clipped)."""
    x = wl.heavy_tailed_bf16(64, 512, 7)
    _, alpha, _ = oracle.tensor_alpha(x)
    codes, scales = oracle.quantize(x, alpha, search=True)
    xhat = oracle.dequantize(codes, scales, alpha)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    sig = np.vectorize(oracle.e4m3_value)(scales.astype(np.int64)).repeat(16, axis=1)
    d = (np.float32(alpha) * sig.astype(np.float32)).astype(np.float64)
    d_exact = np.float64(np.float32(alpha)) * sig
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(d_exact > 0, xhat / np.where(d_exact > 0, d_exact, 1.0), 0.0)
    assert np.all(np.isin(np.abs(v), E2M1_POS))
    m = np.where(d > 0, np.abs(xf) / d, 0.0)
    half = np.where(m <= 2.0, 0.25, np.where(m <= 4.0, 0.5, 1.0))
    normal = sig >= 2.0 ** -6
    err = np.abs(xf - xhat)
    bound = d * half * (1 + 2.0 ** -20) + np.abs(xf) * 2.0 ** -22
    assert np.all((err <= bound) | ~normal | (m > 6.0))


# ------------------------------------------------------------------ RMSNorm feeding the quantizer

def test_rmsnorm_matches_torch_within_one_bf16_ulp():
    x = wl.heavy_tailed_bf16(64, 1024, 51)
    g = wl.normal_bf16(1, 1024, 1.0, 52)[0]
    h, rstd = oracle.rmsnorm(x, g, 1e-6)
    xf = torch.from_numpy(wl.bf16_bits_to_f32(x).astype(np.float64))
    gf = torch.from_numpy(wl.bf16_bits_to_f32(g).astype(np.float64))
    ref = torch.nn.functional.rms_norm(xf, (1024,), weight=gf, eps=1e-6).numpy()
    ref_bf = oracle.bf16_to_f64(oracle.round_bf16(ref))
    mine = oracle.bf16_to_f64(h)
    ulp = oracle.bf16_ulp(ref_bf)
    assert np.all(np.abs(mine - ref_bf) <= ulp)
    assert np.mean(mine == ref_bf) > 0.99
    r64 = 1.0 / np.sqrt((xf.numpy() ** 2).mean(axis=1) + 1e-6)
    assert np.allclose(rstd, r64, rtol=2.0 ** -22, atol=0)


def test_rmsnorm_closed_forms():
    g = wl.normal_bf16(1, 256, 1.0, 53)[0]
    # constant rows of 2 (eps 0): ms = 4, rstd = 0.5 exactly, h = gamma exactly
    x = wl.f32_to_bf16_bits(np.full((2, 256), 2.0, np.float32))
    h, r = oracle.rmsnorm(x, g, 0.0)
    assert np.all(r == 0.5) and np.array_equal(h[0], g) and np.array_equal(h[1], g)
    # +-3 rows: ms = 9, rstd = fl32(1/3), fl32(3 * fl32(1/3)) = 1, so h = +-gamma exactly
    x = wl.f32_to_bf16_bits(np.tile(np.array([3.0, -3.0], np.float32), 128)[None, :])
    h, r = oracle.rmsnorm(x, g, 0.0)
    assert r[0] == np.float32(1.0 / 3.0)
    sign = np.tile(np.array([0, 0x8000], np.uint16), 128)
    assert np.array_equal(h[0], g ^ sign)


# ------------------------------------------------------------------ RoPE on the K projection

def _rope_f64(yk, pos, cs):
    k, _ = oracle.kv_rope_rows(yk, np.zeros_like(yk), pos, cs)
    return oracle.bf16_to_f64(k)


def test_rope_identity_at_position_zero_and_norm_preserved():
    rng = np.random.default_rng(71)
    cs = wl.rope_cos_sin(64)
    yk = rng.standard_normal((4, 256))
    k0 = _rope_f64(yk, np.zeros(4, np.int64), cs)
    assert np.array_equal(k0, oracle.bf16_to_f64(oracle.round_bf16(yk)))
    # each (i, i+64) pair is rotated: its norm is kept (up to the BF16 rounding of the output)
    kr = _rope_f64(yk, np.array([1, 7, 33, 63]), cs).reshape(4, 2, 2, 64)
    y = yk.reshape(4, 2, 2, 64)
    n_in = y[:, :, 0] ** 2 + y[:, :, 1] ** 2
    n_out = kr[:, :, 0] ** 2 + kr[:, :, 1] ** 2
    assert np.allclose(n_out, n_in, rtol=2 ** -6, atol=1e-3)


def test_rope_scores_depend_only_on_relative_position():
    """The defining property of rotary embeddings: <R(p) q, R(p') k> depends on p - p' only
    (checked on the un-rounded rotation; the oracle's output differs from it by BF16 rounding)."""
    rng = np.random.default_rng(72)
    cs = wl.rope_cos_sin(512).astype(np.float64)
    q, k = rng.standard_normal(128), rng.standard_normal(128)

    def rot(v, p):
        c, s = cs[p, :64], cs[p, 64:]
        return np.concatenate([v[:64] * c - v[64:] * s, v[64:] * c + v[:64] * s])
    for p, pp, delta in [(10, 3, 100), (200, 50, 7), (5, 5, 300)]:
        a = rot(q, p) @ rot(k, pp)
        b = rot(q, p + delta) @ rot(k, pp + delta)
        assert abs(a - b) < 2e-5 * (1 + abs(a))
    # the oracle computes exactly that rotation before rounding to BF16
    yk = rng.standard_normal((3, 128))
    pos = np.array([3, 100, 511])
    mine = _rope_f64(yk, pos, cs.astype(np.float32))
    ref = np.stack([rot(yk[i], pos[i]) for i in range(3)])
    cs32 = cs.astype(np.float32).astype(np.float64)
    ref32 = np.stack([np.concatenate([yk[i, :64] * cs32[p, :64] - yk[i, 64:] * cs32[p, 64:],
                                      yk[i, 64:] * cs32[p, :64] + yk[i, :64] * cs32[p, 64:]])
                      for i, p in enumerate(pos)])
    assert np.array_equal(mine, oracle.bf16_to_f64(oracle.round_bf16(ref32)))
    assert np.allclose(mine, ref, rtol=2 ** -7, atol=1e-6)
    # and the property holds for the oracle's own (BF16) outputs, which a sign or index slip
    # in its rotation would break
    cs32 = cs.astype(np.float32)
    qs = rng.standard_normal((1, 128)) * 4
    ks = rng.standard_normal((1, 128)) * 4
    for p, pp, delta in [(10, 3, 100), (200, 50, 7), (30, 400, 60)]:
        a = _rope_f64(qs, np.array([p]), cs32)[0] @ _rope_f64(ks, np.array([pp]), cs32)[0]
        b = _rope_f64(qs, np.array([p + delta]), cs32)[0] @ _rope_f64(ks, np.array([pp + delta]), cs32)[0]
        assert abs(a - b) < 0.02 * np.linalg.norm(qs) * np.linalg.norm(ks) ** 1, (p, pp, a, b)
        if delta >= 60:   # shifting only one side does change the score, well beyond the rounding noise
            c = _rope_f64(qs, np.array([p]), cs32)[0] @ _rope_f64(ks, np.array([pp + delta]), cs32)[0]
            assert abs(a - c) > 10 * abs(a - b)


def test_rope_is_complex_multiplication_by_the_position_phase():
    """Rotary embedding read as complex arithmetic: pairing channel i with i + 64 as
    z_i = k_i + j k_{i+64}, position p multiplies z_i by exp(j p f_i), f_i = 1e6^(-2i/128).
    numpy's complex product (from angles in float64, not the table) fixes the rotation's
    direction and pairing, which the relative-position property alone does not: rotating
    the other way, or pairing i with i + 1, keeps that property but fails here."""
    rng = np.random.default_rng(73)
    cs = wl.rope_cos_sin(4096)
    f = 1.0e6 ** (-2.0 * np.arange(64) / 128)
    yk = rng.standard_normal((6, 256))                        # two heads
    pos = np.array([0, 1, 2, 17, 1000, 4095])
    mine = _rope_f64(yk, pos, cs).reshape(6, 2, 128)
    z = yk.reshape(6, 2, 2, 64)
    zc = (z[:, :, 0] + 1j * z[:, :, 1]) * np.exp(1j * pos[:, None, None] * f[None, None, :])
    ref = np.concatenate([zc.real, zc.imag], axis=2)           # [6, 2, 128]
    bound = oracle.bf16_ulp(ref) + 1e-6 * (np.abs(z[:, :, 0]) + np.abs(z[:, :, 1])).repeat(2, axis=2)
    assert np.all(np.abs(mine - ref) <= bound)
    # closed form at position 1, frequency 0 (f_0 = 1): e_0 turns into (cos 1, sin 1)
    e0 = np.zeros((1, 128))
    e0[0, 0] = 1.0
    r = _rope_f64(e0, np.array([1]), cs)[0]
    assert r[0] == oracle.bf16_to_f64(oracle.round_bf16(np.array([np.cos(1.0)])))[0]
    assert r[64] == oracle.bf16_to_f64(oracle.round_bf16(np.array([np.sin(1.0)])))[0]
    assert np.count_nonzero(r) == 2


@pytest.mark.parametrize("mistake", ["opposite_direction", "adjacent_pairs"])
def test_rope_pin_catches_planted_mistakes(monkeypatch, mistake):
    """Plant a plausible slip in the oracle's rotation (CPU only) and check that the
    complex-multiplication pin fails: rotating by -p f_i (sin sign flipped), or pairing
    channel i with i + 1 instead of i + 64."""
    orig = oracle.kv_rope_rows

    def planted(yk, yv, positions, cos_sin, head_dim=128):
        yk = np.asarray(yk, dtype=np.float64)
        if mistake == "opposite_direction":
            cs = np.array(cos_sin, dtype=np.float32)
            cs[:, head_dim // 2:] *= -1
            return orig(yk, yv, positions, cs, head_dim)
        M, n = yk.shape
        k = yk.reshape(M, n // head_dim, head_dim // 2, 2).transpose(0, 1, 3, 2).reshape(M, n)
        kr, v = orig(k, yv, positions, cos_sin, head_dim)
        return kr.reshape(M, n // head_dim, 2, head_dim // 2).transpose(0, 1, 3, 2).reshape(M, n), v

    monkeypatch.setattr(oracle, "kv_rope_rows", planted)
    with pytest.raises(AssertionError):
        test_rope_is_complex_multiplication_by_the_position_phase()


def test_rmsnorm_eps_enters_under_the_root_and_the_mean_divides_by_k():
    """Closed forms where eps is as large as the mean square, so that eps outside the root
    (1/(sqrt(ms) + eps)) or a mean over K - 1 would change the result far beyond rounding."""
    K = 256
    g = wl.f32_to_bf16_bits(np.ones(K, np.float32))
    # x = 2^-10 everywhere, eps = 2^-20: ms = 2^-20 exactly, ms + eps = 2^-19, rstd = 2^9.5
    x = wl.f32_to_bf16_bits(np.full((1, K), 2.0 ** -10, np.float32))
    h, r = oracle.rmsnorm(x, g, 2.0 ** -20)
    assert r[0] == np.float32(2.0 ** 9.5)
    t = np.float32(np.float32(2.0 ** -10) * np.float32(2.0 ** 9.5))        # fl32(x * rstd), gamma = 1
    assert np.all(h[0] == oracle.round_bf16(np.array([float(t)]))[0])
    # one non-zero element 16 in a row of K: ms = 256 / K = 1 exactly, eps = 3 -> rstd = 1/2
    x = np.zeros((1, K), np.float32)
    x[0, 5] = 16.0
    h, r = oracle.rmsnorm(wl.f32_to_bf16_bits(x), g, 3.0)
    assert r[0] == np.float32(0.5)
    assert wl.bf16_bits_to_f32(h)[0, 5] == 8.0 and np.count_nonzero(wl.bf16_bits_to_f32(h)) == 1


# ------------------------------------------------------------------ the error metric behind every tolerance gate

def test_rel_frobenius_closed_forms():
    """Closed forms of ||y - y_ref||_F / ||y_ref||_F (exact in binary64 for these integers):
    a doubled reference gives exactly 1; an error orthogonal to the reference gives
    ||e|| / ||y_ref|| (12/5 here) and NOT ||e|| / ||y|| (12/13), its square (144/25) or its
    root; the norm runs over all elements of a matrix (1/sqrt(26)), not per row; a zero
    reference gives 0 for a zero output and +inf otherwise."""
    y_ref = np.array([0.0, 3.0, 4.0])
    assert oracle.rel_frobenius(y_ref, y_ref) == 0.0
    assert oracle.rel_frobenius(2.0 * y_ref, y_ref) == 1.0
    assert oracle.rel_frobenius(y_ref + np.array([12.0, 0.0, 0.0]), y_ref) == 12.0 / 5.0
    assert oracle.rel_frobenius(y_ref, y_ref + np.array([12.0, 0.0, 0.0])) == 12.0 / 13.0   # not symmetric
    m_ref = np.array([[3.0, 4.0], [0.0, 1.0]])
    m = m_ref + np.array([[0.0, 0.0], [1.0, 0.0]])
    assert abs(oracle.rel_frobenius(m, m_ref) - 1.0 / math.sqrt(26.0)) <= 1e-16
    assert oracle.rel_frobenius(np.zeros(4), np.zeros(4)) == 0.0
    assert oracle.rel_frobenius(np.array([0.0, 1e-30, 0.0, 0.0]), np.zeros(4)) == math.inf


@pytest.mark.parametrize("mistake", ["divide_by_output_norm", "no_root", "squared", "per_row_mean",
                                     "absolute_on_zero_reference"])
def test_rel_frobenius_pin_catches_planted_mistakes(monkeypatch, mistake):
    """Plant a plausible slip in the metric (CPU only) and check the closed forms catch it."""
    def planted(y, y_ref):
        y = np.asarray(y, dtype=np.float64)
        y_ref = np.asarray(y_ref, dtype=np.float64)
        d = y - y_ref
        if mistake == "divide_by_output_norm":
            return float(np.linalg.norm(d) / np.linalg.norm(y))
        if mistake == "no_root":
            return float(np.sum(d * d) / np.sum(y_ref * y_ref))
        if mistake == "squared":
            return float(np.linalg.norm(d) / np.linalg.norm(y_ref)) ** 2
        if mistake == "per_row_mean":
            yr, dr = np.atleast_2d(y_ref), np.atleast_2d(d)
            return float(np.mean(np.linalg.norm(dr, axis=-1) / np.linalg.norm(yr, axis=-1)))
        den = np.linalg.norm(y_ref)
        return float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))

    monkeypatch.setattr(oracle, "rel_frobenius", planted)
    with pytest.raises(AssertionError):
        test_rel_frobenius_closed_forms()
