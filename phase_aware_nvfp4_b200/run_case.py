"""Run one operation of the library on seeded synthetic data, for profiling.

    python -m phase_aware_nvfp4_b200.run_case quant  --M 8192  --K 12288 [--iters 3]
    python -m phase_aware_nvfp4_b200.run_case gemm   --M 8192  --N 12288 --K 4096
    python -m phase_aware_nvfp4_b200.run_case mlp    --M 8192  --N 24576 --K 4096
    python -m phase_aware_nvfp4_b200.run_case decode --M 1     --N 24576 --K 4096
    python -m phase_aware_nvfp4_b200.run_case kv_rope --M 8192 --N 2048  --K 4096

Inputs are prepared (and weights quantized) before the profiled calls; each
iteration then launches only the operation named:

* ``quant``: activation quantization of a heavy-tailed BF16 X [M, K]
  (tensor amax, then E4M3 block scales and E2M1 codes);
* ``gemm``: the block-scaled NVFP4 GEMM with the BF16 epilogue, X already
  quantized;
* ``mlp``: the gate/up GEMM with the fused SiLU-mul + NVFP4 requantization
  epilogue (N = 2 x intermediate size, interleaved gate/up rows);
* ``decode``: the BF16 decode GEMM Y = X W^T (M <= 256);
* ``decode_nvfp4``: the uniform-NVFP4 decode (tokens quantized on the fly,
  NVFP4 weight; M <= 128);
* ``rmsnorm_quant``: RMSNorm fused with the NVFP4 quantization of its output;
* ``kv_rope``: the K/V projection (N = 2 x heads x 128, X already quantized)
  with RoPE on the K heads and the BF16 KV-cache write in the GEMM epilogue;
  positions uniform in [0, 40960), slots a permutation of the tokens.

Prints the mean CUDA-event time per iteration.  The data recipe is the one the
tests and the benchmark use (Student-t(3) activations with 1 % outlier
channels scaled x20; N(0, 0.02^2) weights).
"""
from __future__ import annotations

import argparse
import sys

import numpy as np


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("op", choices=["quant", "gemm", "mlp", "decode", "decode_nvfp4", "rmsnorm_quant", "kv_rope"])
    ap.add_argument("--M", type=int, default=8192)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    a = ap.parse_args(argv)

    import torch
    from . import mixquant as mq
    from . import workloads as wl

    dev = torch.device("cuda", 0)

    def dev_bf16(x):
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)

    X = dev_bf16(wl.heavy_tailed_bf16(a.M, a.K, 11))
    ws = mq.workspace(a.M, a.K, device=dev)
    if a.op == "rmsnorm_quant":
        gam = dev_bf16(wl.normal_bf16(1, a.K, 1.0, 13)[0])
        Xq = mq.nvfp4_empty(a.M, a.K, dev)
        run = lambda: mq.rmsnorm_quantize(X, gam, 1e-6, out=Xq, ws=ws)
    elif a.op == "quant":
        Xq = mq.nvfp4_empty(a.M, a.K, dev)
        run = lambda: mq.quantize_activation(X, out=Xq, ws=ws)
    elif a.op in ("gemm", "mlp"):
        W = dev_bf16(wl.normal_bf16(a.N, a.K, 0.02, 12))
        Wq = mq.quantize_weight(W, gate_up_interleave=(a.op == "mlp"), ws=ws)
        del W
        Xq = mq.quantize_activation(X, ws=ws)
        if a.op == "gemm":
            Y = torch.empty((a.M, a.N), dtype=torch.bfloat16, device=dev)
            run = lambda: mq.prefill_linear(W=Wq, Xq=Xq, Y=Y, ws=ws)
        else:
            H = mq.nvfp4_empty(a.M, a.N // 2, dev)
            ah = torch.full((1,), 0.25, dtype=torch.float32, device=dev)
            run = lambda: mq.prefill_linear(W=Wq, Xq=Xq, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=ah, H=H, ws=ws)
    elif a.op == "kv_rope":
        if a.N % 256 != 0:
            raise SystemExit("kv_rope needs N = 2 x heads x 128")
        heads, max_pos = a.N // 256, 40960
        Wq = mq.quantize_weight(dev_bf16(wl.normal_bf16(a.N, a.K, 0.02, 12)), ws=ws)
        Xq = mq.quantize_activation(X, ws=ws)
        cs = torch.from_numpy(wl.rope_cos_sin(max_pos)).to(dev)
        rng = np.random.default_rng(14)
        pos = torch.from_numpy(rng.integers(0, max_pos, size=a.M).astype(np.int32)).to(dev)
        slots = torch.from_numpy(rng.permutation(a.M).astype(np.int64)).to(dev)
        kc = torch.empty((a.M, heads, 128), dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        run = lambda: mq.prefill_kv_rope(W=Wq, Xq=Xq, n_kv_heads=heads, positions=pos, cos_sin=cs, slots=slots,
                                         k_cache=kc, v_cache=vc, ws=ws)
    elif a.op == "decode":
        W = dev_bf16(wl.normal_bf16(a.N, a.K, 0.02, 12))
        Y = torch.empty((a.M, a.N), dtype=torch.bfloat16, device=dev)
        wsd = mq.decode_workspace(a.M, a.N, a.K, device=dev)
        run = lambda: mq.decode_linear(X, W, Y=Y, ws=wsd)
    else:
        Wq = mq.quantize_weight(dev_bf16(wl.normal_bf16(a.N, a.K, 0.02, 12)), ws=ws)
        Y = torch.empty((a.M, a.N), dtype=torch.bfloat16, device=dev)
        wsd = mq.decode_workspace(a.M, a.N, a.K, device=dev)
        run = lambda: mq.decode_linear_nvfp4(X, Wq, Y=Y, ws=wsd)
    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        run()
    e1.record()
    torch.cuda.synchronize()
    st = mq.async_status(ws)
    if st == 0 and a.op in ("decode", "decode_nvfp4"):
        st = mq.async_status(wsd)
    ms = e0.elapsed_time(e1) / max(1, a.iters)
    flops = 2.0 * a.M * a.N * a.K if a.op in ("gemm", "mlp", "kv_rope", "decode", "decode_nvfp4") else 0.0
    rate = f", {flops / (ms * 1e-3) / 1e12:.0f} TFLOP/s" if flops else ""
    print(f"{a.op} M={a.M} N={a.N} K={a.K}: {ms * 1e3:.1f} us per call{rate} (status {mq.STATUS_NAMES.get(st, st)})")
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
