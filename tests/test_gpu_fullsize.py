"""Parity at the workloads' full sizes, in the launch configuration the
benchmark uses.  Quantization is checked bit-exactly on sampled rows (and
on whole weights); GEMM outputs on sampled rows that the FP64 oracle
computes one by one, with the tolerance of gpu_helpers.gemm_check.  The
sample holds one row of every 128-row block (and the first and last rows),
so every M-block of the CTA-pair tile schedule is compared; the 8192-token
k projection is compared on its whole output.

Workloads (seeded synthetic stand-ins for the paper's prefill activations,
Qwen3-8B layer shapes):
  * 8192-token projections: q (K=4096, N=4096), k (N=1024), up (N=12288),
    down (K=12288, N=4096);
  * 32768-token fused MLP: gate+up (K=4096, N=2*12288) -> SiLU-mul ->
    NVFP4 h -> down (K=12288, N=4096);
  * phase-aware pair on one BF16 master weight (K=4096, N=12288): NVFP4
    prefill at 16384 tokens and BF16 decode at 1/8/32/64 tokens;
  * ragged multi-turn prefill: 8 sequences, 131072 tokens, one MLP.
"""
import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import (block_rows, gemm_check, nvfp4_host, require_gpu, silu_mul_check, to_dev, to_host_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _dev_rows_quant(t, rows):
    codes = t.codes[torch.as_tensor(rows, device=t.codes.device)].cpu().numpy()
    rm = mq.unswizzle_scales(t).cpu().numpy()[rows]
    return codes, rm, float(t.alpha.cpu()[0])


def _check_activation(x_bits, Xq, rows):
    _, ax, _ = oracle.tensor_alpha(x_bits)
    codes, scales, alpha = _dev_rows_quant(Xq, rows)
    assert np.float32(alpha) == np.float32(ax)
    rc, rs = oracle.quantize(x_bits[rows], ax)
    assert np.array_equal(scales, rs) and np.array_equal(codes, rc)
    return ax, rc, rs


def _check_weight(w_bits, Wq):
    codes, scales, alpha = nvfp4_host(Wq)
    _, aw, _ = oracle.tensor_alpha(w_bits)
    assert alpha == aw
    rc, rs = oracle.quantize(w_bits, aw)
    assert np.array_equal(scales, rs), f"{int((scales != rs).sum())} weight scale mismatches"
    assert np.array_equal(codes, rc), f"{int((codes != rc).sum())} weight code mismatches"
    return rc, rs, aw


def test_qwen3_8b_projections_M8192():
    w = wl.qwen3_8b_projections(8192)
    groups = {}
    for p in w.projections:
        groups.setdefault(p.x_group, []).append(p)
    ws = mq.workspace()
    for g, ps in groups.items():
        x = wl.make_x(ps[0])
        Xq = mq.quantize_activation(to_dev(x), ws=ws)
        rows = block_rows(x.shape[0], seed=len(g))       # one row in every 128-row block
        ax, xc, xs = _check_activation(x, Xq, rows)
        for p in ps:
            wb = wl.make_w(p)
            Wq = mq.quantize_weight(to_dev(wb), ws=ws)
            y = mq.prefill_linear(W=Wq, Xq=Xq, ws=ws)
            torch.cuda.synchronize()
            wc, wsc, aw = _check_weight(wb, Wq)
            if p.name == "k_proj":
                # the smallest projection (8192 x 1024 x 4096, 68.7 GFLOP): its whole output vs the oracle,
                # with the whole activation's codes and scales bit-exact
                ax, xc_all, xs_all = _check_activation(x, Xq, np.arange(x.shape[0]))
                y64, sabs = oracle.nvfp4_linear_rows((xc_all, xs_all, ax), (wc, wsc, aw))
                rel, mx, bmax = gemm_check(to_host_bits(y), y64, sabs)
                del xc_all, xs_all
            else:
                y64, sabs = oracle.nvfp4_linear_rows((xc, xs, ax), (wc, wsc, aw))
                rel, mx, bmax = gemm_check(to_host_bits(y[torch.as_tensor(rows, device=y.device)]), y64, sabs)
            print(f"{p.name}: rel-Frobenius {rel:.2e}, max-abs {mx:.3e} (bound max {bmax:.3e})")
            del y, Wq, y64, sabs
    assert mq.async_status(ws) == 0


def _mlp(x, wgu, wdn, rows, ws):
    """Run the fused MLP on the GPU with a calibrated alpha_h (amax of h / (6*448)
    from an unfused-equivalent calibration pass) and check it on `rows`."""
    M, I = x.shape[0], wdn.shape[1]
    X = to_dev(x)
    Wgu = mq.quantize_weight(to_dev(wgu), gate_up_interleave=True, ws=ws)
    Wdn = mq.quantize_weight(to_dev(wdn), ws=ws)
    h_dbg = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    one = torch.ones(1, device="cuda")
    mq.prefill_linear(X, Wgu, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=one, h_debug=h_dbg, ws=ws)
    amax_h = float(h_dbg.float().abs().max())            # calibration: amax of h
    alpha_h = np.float32(amax_h / 2688.0) if amax_h > 0 else np.float32(1.0)
    ah = torch.tensor([float(alpha_h)], device="cuda")
    H = mq.prefill_linear(X, Wgu, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=ah, h_debug=h_dbg, ws=ws)
    H.alpha.copy_(ah)
    y = mq.prefill_linear(W=Wdn, Xq=H, ws=ws)
    torch.cuda.synchronize()
    assert mq.async_status(ws) == 0
    ridx = torch.as_tensor(rows, device="cuda")

    # gate/up GEMM + SiLU-mul on the sampled rows
    ax = oracle.tensor_alpha(x)[1]
    xc, xs = oracle.quantize(x[rows], ax)
    awgu = oracle.tensor_alpha(wgu)[1]
    g64, gs = oracle.nvfp4_linear_rows((xc, xs, ax), (*oracle.quantize(wgu, awgu), awgu))
    h_gpu = to_host_bits(h_dbg[ridx])
    rel_h, mx_h, bmax_h = silu_mul_check(h_gpu, g64[:, :I], g64[:, I:], gs[:, :I], gs[:, I:])
    del g64, gs
    # h codes / scales: bit-exact vs the oracle quantizing the GPU's own h with alpha_h
    hc, hs, _ = _dev_rows_quant(H, rows)
    rc, rs = oracle.quantize(h_gpu, float(alpha_h))
    assert np.array_equal(hs, rs) and np.array_equal(hc, rc)
    # down projection on the sampled rows of the NVFP4 h
    awd = oracle.tensor_alpha(wdn)[1]
    y64, sabs = oracle.nvfp4_linear_rows((rc, rs, float(alpha_h)), (*oracle.quantize(wdn, awd), awd))
    rel, mx, bmax = gemm_check(to_host_bits(y[ridx]), y64, sabs)
    # end-to-end vs the unquantized BF16 MLP (reported, not gated beyond sanity)
    yb = oracle.bf16_linear_rows(x, wgu, rows)
    hb = oracle.silu_mul(yb[:, :I], yb[:, I:])
    yb2 = oracle.bf16_linear_rows(hb, wdn)
    e2e = oracle.rel_frobenius(oracle.bf16_to_f64(to_host_bits(y[ridx])), yb2)
    print(f"MLP M={M}: h rel {rel_h:.2e}, max-abs {mx_h:.3e} (bound max {bmax_h:.3e}); down rel-Frobenius {rel:.2e}, max-abs {mx:.3e} "
          f"(bound max {bmax:.3e}); NVFP4-vs-BF16 MLP error {e2e:.3f}")
    assert e2e < 0.5
    return y


def test_fused_mlp_M32768():
    x = wl.heavy_tailed_bf16(32768, 4096, 3000)
    wgu, wdn = wl.mlp_weights(3000)
    rows = block_rows(32768, seed=3)         # one row in every 128-row block
    _mlp(x, wgu, wdn, rows, mq.workspace(x.shape[0], x.shape[1]))


def test_ragged_multiturn_131072_tokens():
    x, off = wl.ragged_heavy_tailed_bf16(wl.RAGGED_LENGTHS, 4096, 5000)
    assert x.shape[0] == 131072
    wgu, wdn = wl.mlp_weights(5000)
    # one row in every 128-row block, plus every sequence's first and last token
    bounds = [int(off[i]) for i in range(len(wl.RAGGED_LENGTHS))] + [int(off[i + 1]) - 1
                                                                      for i in range(len(wl.RAGGED_LENGTHS))]
    rows = block_rows(x.shape[0], seed=5, extra=bounds)
    _mlp(x, wgu, wdn, rows, mq.workspace(x.shape[0], x.shape[1]))


def test_phase_aware_pair_shared_master_weight():
    """NVFP4 prefill at 16384 tokens and BF16 decode at 1/8/32/64 tokens on one BF16 master weight."""
    wmaster = wl.normal_bf16(12288, 4096, 0.02, 4001)
    ws = mq.workspace()
    Wd = to_dev(wmaster)
    Wq = mq.quantize_weight(Wd, ws=ws)
    wc, wsc, aw = _check_weight(wmaster, Wq)
    x = wl.heavy_tailed_bf16(16384, 4096, 4000)
    rows = block_rows(16384, seed=4)
    y = mq.prefill_linear(to_dev(x), Wq, ws=mq.workspace(16384, 4096))
    torch.cuda.synchronize()
    ax = oracle.tensor_alpha(x)[1]
    y64, sabs = oracle.nvfp4_linear_rows((*oracle.quantize(x[rows], ax), ax), (wc, wsc, aw))
    gemm_check(to_host_bits(y[torch.as_tensor(rows, device="cuda")]), y64, sabs)
    # NVFP4-vs-BF16 output error: GPU value equals the oracle's within 1e-3
    ybf = oracle.bf16_linear_rows(x, wmaster, rows)
    err_gpu = oracle.rel_frobenius(oracle.bf16_to_f64(to_host_bits(y[torch.as_tensor(rows, device='cuda')])), ybf)
    err_ref = oracle.rel_frobenius(oracle.bf16_to_f64(oracle.round_bf16(y64)), ybf)
    print(f"NVFP4-vs-BF16 relative error: GPU {err_gpu:.4f}, oracle {err_ref:.4f}")
    assert abs(err_gpu - err_ref) < 1e-3
    for M in (1, 8, 32, 64):
        xd = wl.heavy_tailed_bf16(M, 4096, 4100 + M)
        yd = mq.decode_linear(to_dev(xd), Wd, ws=ws)
        torch.cuda.synchronize()
        ref = oracle.bf16_linear_rows(xd, wmaster)
        sab = np.abs(oracle.bf16_to_f64(xd)) @ np.abs(oracle.bf16_to_f64(wmaster)).T
        yr = oracle.bf16_to_f64(oracle.round_bf16(ref))
        yg = oracle.bf16_to_f64(to_host_bits(yd))
        ulp = np.maximum(oracle.bf16_ulp(yr), oracle.bf16_ulp(yg))
        assert np.all(np.abs(yg - yr) <= ulp + 2.0 ** -16 * sab)
    # the transposed orientation of the same 4096 x 12288 master (K = 12288, N = 4096)
    wt = wl.normal_bf16(4096, 12288, 0.02, 4002)
    xd = wl.heavy_tailed_bf16(64, 12288, 4003)
    yd = mq.decode_linear(to_dev(xd), to_dev(wt), ws=ws)
    torch.cuda.synchronize()
    ref = oracle.bf16_to_f64(oracle.round_bf16(oracle.bf16_linear_rows(xd, wt)))
    assert oracle.rel_frobenius(oracle.bf16_to_f64(to_host_bits(yd)), ref) < 1e-3
    assert mq.async_status(ws) == 0
