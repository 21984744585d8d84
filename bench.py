#!/usr/bin/env python
"""Benchmark of the NVFP4 prefill linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {mixquant,reference}]

One step = one prefill pass over the linear projections of a Qwen3-8B-shaped
transformer layer at M = 8192 tokens (the four projection shapes of the
workload: q-proj K=4096 N=4096 and k-proj K=4096 N=1024 on the attention
input, up-proj K=4096 N=12288 on the MLP input, down-proj K=12288 N=4096 on
the MLP intermediate).  Every activation is quantized on the fly (dynamic
tensor amax + NVFP4 block quantizer, once per distinct input), then each
projection runs the tcgen05 block-scaled FP4 GEMM with a BF16 output.  The
weights are quantized once, before timing (offline, as the method does).

The metric is prefill-linear TFLOP/s counting 2*M*N*K per projection over
the time of quantization + GEMM.  L2 (126 MB) is flushed before every timed
step by a 512 MiB write followed by a 256 MiB read (the read evicts the dirty
lines of the write, so the timed kernels start on a cold L2 without paying
for the flush buffer's write-back); the flush is outside the per-step CUDA
events.  The timed steps carry no events between their kernels (an event
between two kernels would keep the second from launching while the first
drains); the per-kernel times behind the rooflines come from a second pass
of the same steps with an event around every kernel.

Multi-GPU: one process per GPU (torchrun), each rank runs its own independent
prefill batch -- the linear layer is token-parallel, so there is no
data-path collective ("weak" scaling).  A barrier brackets the timed region
and the per-step time is the max over ranks.

--impl reference times the CPU oracle (oracle/), as it stands, on the host
cores, on a bounded sample of the same workload, and prints the same line
with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 prefill linear TFLOP/s (quant+GEMM) and fraction of B200 dense FP4 peak"
UNIT = "TFLOP/s"
FP4_PER_BF16 = 4.0          # nominal dense FP4 : dense BF16 tensor throughput on B200
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
GEMM_SOURCES = ("phase_aware_nvfp4_b200/csrc/mq_gemm.cu", "phase_aware_nvfp4_b200/csrc/mq_device.cuh")
QUANT_SOURCES = ("phase_aware_nvfp4_b200/csrc/mq_quant.cu", "phase_aware_nvfp4_b200/csrc/mq_device.cuh")
COUNTERS = os.path.join(ROOT, "profiles", "ncu_dram_bytes_gemm_and_quantizer_qwen3_8b_projections_M8192.json")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mixquant", choices=["mixquant", "reference"])
    ap.add_argument("--M", type=int, default=8192, help="prefill tokens per step (per rank)")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the decode / fused-MLP side measurements reported under 'extras'")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- helpers

def sources_sha(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0) or 0), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 0.0, "fallback"


def counters_for(kernel: str, sha: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source is unchanged since."""
    try:
        with open(COUNTERS) as f:
            d = json.load(f)
        k = d.get(kernel, {})
        if k.get("source_sha") == sha:
            return k
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005, pci=None, nvml=None):
        """index: NVML index to use when no NVML device matches `pci`, the
        (domain, bus, device) PCI address of the CUDA device being timed (NVML
        enumerates every GPU of the node, CUDA only the visible ones)."""
        self.period = period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.match = None
        self._stop = threading.Event()
        self._t = None
        try:
            if nvml is None:
                import pynvml as nvml
            nvml.nvmlInit()
            self.nv = nvml
            self.h, self.match = self._handle(nvml, index, pci)
            self.max_mhz = nvml.nvmlDeviceGetMaxClockInfo(self.h, nvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    @staticmethod
    def _handle(nv, index, pci):
        if pci is not None:
            try:
                for i in range(nv.nvmlDeviceGetCount()):
                    h = nv.nvmlDeviceGetHandleByIndex(i)
                    info = nv.nvmlDeviceGetPciInfo(h)
                    if (int(info.domain), int(info.bus), int(info.device)) == tuple(int(v) for v in pci):
                        return h, "pci"
            except Exception:
                pass
        return nv.nvmlDeviceGetHandleByIndex(index), "index"

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "nvml_device": self.match}


# ---------------------------------------------------------------- multi-rank aggregation

def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of every rank divided by the slowest rank's step time."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------- workload

def workload(M: int):
    from phase_aware_nvfp4_b200 import workloads as wl
    return wl.qwen3_8b_projections(M)


def groups_of(w):
    groups = {}
    for p in w.projections:
        groups.setdefault(p.x_group, []).append(p)
    return groups


def host_inputs(w):
    """Seeded BF16 inputs (numpy uint16): one X per input group, one W per projection."""
    from phase_aware_nvfp4_b200 import workloads as wl
    xs = {g: wl.make_x(ps[0]) for g, ps in groups_of(w).items()}
    ws = {p.name: wl.make_w(p) for p in w.projections}
    return xs, ws


# ---------------------------------------------------------------- oracle timing

def oracle_sample_step(w, xs, wq, rows_per_proj: int, cols_per_proj: int, rng):
    """One bounded oracle pass: for each projection, the tensor amax of X, the
    NVFP4 quantization of `rows_per_proj` sampled rows and the FP64 block-scaled
    matmul against `cols_per_proj` sampled weight rows.  Returns the FLOPs covered."""
    import oracle
    flops = 0
    for g, ps in groups_of(w).items():
        x = xs[g]
        _, ax, _ = oracle.tensor_alpha(x)
        rows = np.sort(rng.choice(x.shape[0], size=min(rows_per_proj, x.shape[0]), replace=False))
        xc, xsc = oracle.quantize(x[rows], ax)
        for p in ps:
            wc, wsc, aw = wq[p.name]
            cols = np.sort(rng.choice(p.N, size=min(cols_per_proj, p.N), replace=False))
            oracle.nvfp4_linear_rows((xc, xsc, ax), (wc[cols], wsc[cols], aw))
            flops += 2 * len(rows) * len(cols) * p.K
    return flops


def oracle_threads():
    import oracle
    n = oracle.num_threads()
    try:
        from threadpoolctl import threadpool_info
        n = max([n] + [int(i.get("num_threads", 1)) for i in threadpool_info()])
    except Exception:
        pass
    return n


def time_oracle(w, xs, wsh, budget_s: float, steps: int = 1, warmup: int = 0):
    """Oracle throughput in TFLOP/s on bounded samples sized to `budget_s` seconds per step."""
    import oracle
    wq = {}
    for p in w.projections:
        _, aw, _ = oracle.tensor_alpha(wsh[p.name])
        wq[p.name] = (*oracle.quantize(wsh[p.name], aw), aw)
    rng = np.random.default_rng(0)
    # calibrate the sample so one step costs about budget_s
    r, c = 16, 256
    t0 = time.perf_counter()
    oracle_sample_step(w, xs, wq, r, c, rng)
    t1 = time.perf_counter() - t0
    scale = max(1.0, budget_s / max(t1, 1e-3))
    r = int(min(w.projections[0].M, r * scale ** 0.5))
    c = int(min(4096, c * scale ** 0.5))
    for _ in range(warmup):
        oracle_sample_step(w, xs, wq, r, c, rng)
    tot_flops, tot_t = 0, 0.0
    for _ in range(max(1, steps)):
        t0 = time.perf_counter()
        tot_flops += oracle_sample_step(w, xs, wq, r, c, rng)
        tot_t += time.perf_counter() - t0
    return {"value": tot_flops / tot_t / 1e12, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"per step and projection: tensor amax of the full X, NVFP4 quantization of {r} of "
                      f"{w.projections[0].M} sampled activation rows, FP64 block-scaled matmul against {c} "
                      f"sampled weight rows (x all K); weights quantized before timing",
            "seconds": tot_t, "steps": max(1, steps)}


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(args.M)
    xs, wsh = host_inputs(w)
    per_step = max(0.05, min(2.0, 120.0 / max(1, args.steps + args.warmup)))
    res = time_oracle(w, xs, wsh, per_step, steps=args.steps, warmup=args.warmup)
    line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * res["seconds"] / res["steps"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w),
            "cpu_baseline": {k: res[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": res["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": w.name, "M": w.projections[0].M,
            "projections": [{"name": p.name, "K": p.K, "N": p.N} for p in w.projections],
            "activation": "Student-t(3), 1% channels x20, BF16", "weights": "N(0, 0.02^2), BF16",
            "l2": "flushed before every timed step: 512 MiB write, then 256 MiB read (cold, clean L2)",
            "quantization": "dynamic tensor amax per activation, once per distinct input"}


# ---------------------------------------------------------------- GPU arm

def _to_dev(torch, a, dev):
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)


class L2Flush:
    """Evicts L2 (126 MB): a 512 MiB write, then a 256 MiB read, so that the
    dirty lines of the write are written back before the timed work starts."""

    def __init__(self, torch, dev):
        self.w = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def _time_calls(torch, fn, reps, flush):
    """Mean device time (ms) of fn() over reps calls, L2 flushed before each.  One untimed call
    comes first, so first-launch costs (lazy loading of a kernel's module, tensor-map set-up)
    stay out of the mean."""
    fn()
    evs = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def _time_rotating(torch, calls, reps):
    """Mean device time (ms) of one call, cycling through `calls` (each on its
    own copy of the weights, together larger than L2, so every call streams
    its weights from HBM while the kernels' code and descriptors stay warm).
    A spin kernel before each call keeps the GPU busy while the host enqueues."""
    evs = []
    for i in range(reps):
        torch.cuda._sleep(200_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        calls[i % len(calls)]()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def _time_stream(torch, calls, reps):
    """Mean device time (ms) per call of `reps` calls issued back to back,
    cycling through `calls` as _time_rotating does: the decode of a layer stack,
    where each call's launch overlaps the previous call's tail."""
    # the GPU spins (~5 ms) while the host enqueues all the calls, so that the
    # timed span holds device work only, not host launch overhead
    torch.cuda._sleep(10_000_000)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(reps):
        calls[i % len(calls)]()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def _decode_pair(mq, torch, dev, wl, Wm, Wq, hbm_gbs, reps, seed):
    """BF16 decode and uniform-NVFP4 decode (tokens quantized on the fly) on one
    weight [N, K] and its NVFP4 copy at M = 1, 8, 32, 64 tokens, timed on
    rotating weight copies larger than L2 (weights cold, code warm): `ms` per
    isolated call (a spin kernel before each, so every call pays its launch
    and ramp), `ms_stream` per call of a back-to-back sequence.  HBM roofline
    bytes: 2NK + 2MK + 2MN (BF16) and 0.5625NK + 2MK + 2MN (NVFP4)."""
    N, K = Wm.shape
    n_bf = max(2, -(-(400 << 20) // (2 * N * K)))          # copies: together > 3 x L2
    n_q = max(2, -(-(400 << 20) // (N * K // 2)))
    Wm_copies = [Wm] + [Wm.clone() for _ in range(n_bf - 1)]
    Wq_copies = [Wq] + [mq.NVFP4Tensor(Wq.codes.clone(), Wq.scales.clone(), Wq.alpha.clone(), Wq.rows, Wq.cols)
                        for _ in range(n_q - 1)]
    dec, decq = {}, {}
    for M in (1, 8, 32, 64):
        x = _to_dev(torch, wl.heavy_tailed_bf16(M, K, seed + M), dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsd = mq.decode_workspace(M, N, K, device=dev)
        bf = [lambda W=W: mq.decode_linear(x, W, Y=y, ws=wsd) for W in Wm_copies]
        q4 = [lambda W=W: mq.decode_linear_nvfp4(x, W, Y=y, ws=wsd) for W in Wq_copies]
        for f in bf + q4:
            f()
        # the set-up above leaves the GPU idle for a while: ~50 ms of spinning first,
        # so the timed calls do not start on a clock that is still ramping up
        torch.cuda._sleep(100_000_000)
        ms = _time_rotating(torch, bf, 4 * reps)
        ms_s = _time_stream(torch, bf, 4 * reps)
        by = 2 * N * K + 2 * M * K + 2 * M * N
        gbs = by / (ms * 1e-3) / 1e9
        dec[str(M)] = {"ms": ms, "GB/s": gbs, "frac": gbs / hbm_gbs,
                       "ms_stream": ms_s, "frac_stream": by / (ms_s * 1e-3) / 1e9 / hbm_gbs}
        msq = _time_rotating(torch, q4, 4 * reps)
        msq_s = _time_stream(torch, q4, 4 * reps)
        byq = 0.5625 * N * K + 2 * M * K + 2 * M * N
        gbs = byq / (msq * 1e-3) / 1e9
        decq[str(M)] = {"ms": msq, "GB/s": gbs, "frac": gbs / hbm_gbs, "speedup_vs_bf16": ms / msq,
                        "ms_stream": msq_s, "frac_stream": byq / (msq_s * 1e-3) / 1e9 / hbm_gbs,
                        "speedup_vs_bf16_stream": ms_s / msq_s}
    del Wm_copies, Wq_copies
    return dec, decq


def measure_extras(mq, torch, dev, flush, hbm_gbs, fp4_peak, reps=10):
    """Side measurements of the other workloads (the main line is the projection step):

    * phase-aware pair on one BF16 master weight [12288, 4096]: BF16 decode at
      M = 1, 8, 32, 64 tokens (HBM roofline: 2NK + 2MK + 2MN bytes), the
      uniform-NVFP4 decode on its NVFP4 copy (0.5625 NK + 2MK + 2MN bytes;
      includes quantizing the tokens) -- both timed on rotating weight copies
      larger than L2 (weights cold, code warm) -- and NVFP4
      prefill (quantize + GEMM) at M = 16384, plus the NVFP4-vs-BF16 output
      error of the two paths on the first 64 prefill tokens;
    * fused MLP at M = 32768: activation quantization, gate/up GEMM with the
      SiLU-mul + NVFP4 requantization epilogue, down GEMM.
    """
    from phase_aware_nvfp4_b200 import workloads as wl
    out = {}
    N, K = 12288, 4096
    Wm = _to_dev(torch, wl.normal_bf16(N, K, 0.02, 4001), dev)
    ws = mq.workspace(16384, K, device=dev)
    Wq = mq.quantize_weight(Wm, ws=ws)
    dec, decq = _decode_pair(mq, torch, dev, wl, Wm, Wq, hbm_gbs, reps, seed=4000)
    # the other orientation of the same 4096 x 12288 master (K = 12288, N = 4096)
    Wt = _to_dev(torch, wl.normal_bf16(K, N, 0.02, 4002), dev)
    dec_t, decq_t = _decode_pair(mq, torch, dev, wl, Wt, mq.quantize_weight(Wt, ws=ws), hbm_gbs, reps, seed=4003)
    del Wt
    Mp = 16384
    X = _to_dev(torch, wl.heavy_tailed_bf16(Mp, K, 4000), dev)
    Xq = mq.nvfp4_empty(Mp, K, dev)
    Y = torch.empty((Mp, N), dtype=torch.bfloat16, device=dev)

    def prefill():
        mq.quantize_activation(X, out=Xq, ws=ws)
        mq.prefill_linear(W=Wq, Xq=Xq, Y=Y, ws=ws)
    for _ in range(3):
        prefill()
    ms = _time_calls(torch, prefill, reps, flush)
    yb = mq.decode_linear(X[:64], Wm, ws=ws)
    torch.cuda.synchronize()
    yq, yr = Y[:64].double(), yb.double()
    err = float(torch.linalg.norm(yq - yr) / torch.linalg.norm(yr))
    # opt-in per-block scale search on the same weight: cost and quantization error
    def dequant(t):
        rs = mq.unswizzle_scales(t).to(torch.float32)          # E4M3 codes, row-major [N, K/16]
        sig = rs.to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float32)
        c = t.codes.to(torch.int32)
        nib = torch.stack([c & 15, c >> 4], dim=-1).reshape(t.rows, t.cols)
        lut = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6], device=dev)
        return lut[nib] * sig.repeat_interleave(16, dim=1) * t.alpha
    wref = Wm.to(torch.float32)
    tp = mq.quantize(Wm, ws=ws)
    tsr = mq.quantize(Wm, scale_search=True, ws=ws)
    ms_p = _time_calls(torch, lambda: mq.quantize(Wm, out=tp, ws=ws), reps, flush)
    ms_s = _time_calls(torch, lambda: mq.quantize(Wm, scale_search=True, out=tsr, ws=ws), reps, flush)
    err_p = float(torch.linalg.norm(dequant(tp) - wref) / torch.linalg.norm(wref))
    err_s = float(torch.linalg.norm(dequant(tsr) - wref) / torch.linalg.norm(wref))
    moved = float((mq.unswizzle_scales(tp) != mq.unswizzle_scales(tsr)).float().mean())
    out["scale_search"] = {"weight": [N, K], "ms_eq3": ms_p, "ms_search": ms_s,
                           "GB/s_search": (2 + 0.5625) * N * K / (ms_s * 1e-3) / 1e9,
                           "rel_err_eq3": err_p, "rel_err_search": err_s, "blocks_moved": moved}
    # K/V projection with RoPE + KV-cache write in the epilogue vs the same GEMM with a plain BF16 output
    Hk, Mk = 8, 8192
    Xk = _to_dev(torch, wl.heavy_tailed_bf16(Mk, K, 70), dev)
    wsk = mq.workspace(Mk, K, device=dev)
    Xkq = mq.quantize_activation(Xk, ws=wsk)
    Wkv = mq.quantize_weight(_to_dev(torch, wl.normal_bf16(2 * Hk * 128, K, 0.02, 71), dev), ws=wsk)
    csk = torch.from_numpy(wl.rope_cos_sin(40960)).to(dev)
    posk = torch.randint(0, 40960, (Mk,), dtype=torch.int32, device=dev)
    slk = torch.randperm(Mk, device=dev)
    kck = torch.empty((Mk, Hk, 128), dtype=torch.bfloat16, device=dev)
    vck = torch.empty_like(kck)
    Yk = torch.empty((Mk, 2 * Hk * 128), dtype=torch.bfloat16, device=dev)
    ms_kv = _time_calls(torch, lambda: mq.prefill_kv_rope(W=Wkv, Xq=Xkq, n_kv_heads=Hk, positions=posk, cos_sin=csk,
                                                           slots=slk, k_cache=kck, v_cache=vck, ws=wsk), reps, flush)
    ms_plain = _time_calls(torch, lambda: mq.prefill_linear(W=Wkv, Xq=Xkq, Y=Yk, ws=wsk), reps, flush)
    fl_kv = 2 * Mk * 2 * Hk * 128 * K
    out["kv_rope"] = {"M": Mk, "K": K, "n_kv_heads": Hk, "ms_fused": ms_kv, "ms_plain_gemm": ms_plain,
                      "TFLOP/s_fused": fl_kv / (ms_kv * 1e-3) / 1e12, "TFLOP/s_plain": fl_kv / (ms_plain * 1e-3) / 1e12}
    del Xk, Xkq, kck, vck, Yk
    # RMSNorm -> NVFP4 fused (the producer of the q/k/v input) vs the unfused pair
    Mr = 8192
    Xr = _to_dev(torch, wl.heavy_tailed_bf16(Mr, K, 61), dev)
    gam = _to_dev(torch, wl.normal_bf16(1, K, 1.0, 62)[0], dev)
    wsr = mq.workspace(Mr, K, device=dev)
    tr = mq.rmsnorm_quantize(Xr, gam, 1e-6, ws=wsr)
    tu = mq.nvfp4_empty(Mr, K, dev)

    def unfused():   # torch's norm writes BF16 h, then the quantizer reads it (amax + quantize)
        h = torch.nn.functional.rms_norm(Xr, (K,), weight=gam, eps=1e-6)
        mq.quantize_activation(h, out=tu, ws=wsr)
    ms_f = _time_calls(torch, lambda: mq.rmsnorm_quantize(Xr, gam, 1e-6, out=tr, ws=wsr), reps, flush)
    ms_u = _time_calls(torch, unfused, reps, flush)
    gbs_f = (2 + 2 + 0.5625) * Mr * K / (ms_f * 1e-3) / 1e9
    out["rmsnorm_quantize"] = {"M": Mr, "K": K, "ms_fused": ms_f, "ms_unfused_torch_norm": ms_u,
                               "GB/s_fused": gbs_f, "frac_fused": gbs_f / hbm_gbs, "speedup": ms_u / ms_f}
    del Xr
    out["phase_aware_pair"] = {
        "weight": [N, K], "decode_bf16": dec,
        "roofline_decode": {"bound": "hbm", "kernel": "decode_bf16_kernel", "unit": "GB/s", "peak": hbm_gbs,
                            "achieved": dec["64"]["GB/s"], "frac": dec["64"]["frac"], "M": 64,
                            "frac_stream": dec["64"]["frac_stream"]},
        "decode_nvfp4": decq,
        "transposed_weight": [K, N], "decode_bf16_k12288": dec_t, "decode_nvfp4_k12288": decq_t,
        "prefill_nvfp4": {"M": Mp, "ms": ms, "TFLOP/s": 2 * Mp * N * K / (ms * 1e-3) / 1e12},
        "nvfp4_vs_bf16_rel_frobenius": err}
    del X, Xq, Y
    # fused MLP, M = 32768
    Mm = 32768
    wgu, wdn = wl.mlp_weights(3000)
    I = wdn.shape[1]
    Wgu = mq.quantize_weight(_to_dev(torch, wgu, dev), gate_up_interleave=True, ws=ws)
    Wdn = mq.quantize_weight(_to_dev(torch, wdn, dev), ws=ws)
    X = _to_dev(torch, wl.heavy_tailed_bf16(Mm, K, 3000), dev)
    wsm = mq.workspace(Mm, K, device=dev)
    Xq = mq.nvfp4_empty(Mm, K, dev)
    H = mq.nvfp4_empty(Mm, I, dev)
    Y = torch.empty((Mm, wdn.shape[0]), dtype=torch.bfloat16, device=dev)
    # static alpha_h, calibrated once (offline step): amax of h over this batch / (6 * 448)
    mq.quantize_activation(X, out=Xq, ws=wsm)
    h_dbg = torch.empty((Mm, I), dtype=torch.bfloat16, device=dev)
    one = torch.ones(1, dtype=torch.float32, device=dev)
    mq.prefill_linear(W=Wgu, Xq=Xq, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=one, H=H, h_debug=h_dbg, ws=wsm)
    amax_h = float(h_dbg.float().abs().max())
    del h_dbg
    ah = torch.full((1,), amax_h / 2688.0 if amax_h > 0 else 1.0, dtype=torch.float32, device=dev)
    H.alpha.copy_(ah)

    parts = {}

    def mlp(record=None):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        mq.quantize_activation(X, out=Xq, ws=wsm)
        e[1].record()
        mq.prefill_linear(W=Wgu, Xq=Xq, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=ah, H=H, ws=wsm)
        e[2].record()
        mq.prefill_linear(W=Wdn, Xq=H, Y=Y, ws=wsm)
        e[3].record()
        if record is not None:
            record.append(e)
    for _ in range(3):
        mlp()
    rec = []
    ms = _time_calls(torch, lambda: mlp(rec), reps, flush)
    q_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in rec]))
    gu_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in rec]))
    dn_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in rec]))
    fl_gu = 2 * Mm * wgu.shape[0] * K
    fl_dn = 2 * Mm * wdn.shape[0] * I
    out["fused_mlp"] = {"M": Mm, "gate_up": [wgu.shape[0], K], "down": [wdn.shape[0], I], "ms": ms,
                        "TFLOP/s": (fl_gu + fl_dn) / (ms * 1e-3) / 1e12,
                        "quant_ms": q_ms, "gate_up_silu_requant_ms": gu_ms, "down_ms": dn_ms,
                        "gate_up_TFLOP/s": fl_gu / (gu_ms * 1e-3) / 1e12,
                        "down_TFLOP/s": fl_dn / (dn_ms * 1e-3) / 1e12,
                        "gate_up_frac": fl_gu / (gu_ms * 1e-3) / 1e12 / fp4_peak}
    # the unfused MLP with a dynamic alpha_h (R9's alternative): gate/up GEMM writing BF16 h,
    # then the down projection quantizing h with amax|h| / 2688 (amax + quantize + GEMM)
    Hb = torch.empty((Mm, I), dtype=torch.bfloat16, device=dev)
    Y2 = torch.empty_like(Y)
    wsh = mq.workspace(Mm, I, device=dev)
    rec2 = []

    def mlp_unfused():
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        mq.quantize_activation(X, out=Xq, ws=wsm)
        e[1].record()
        mq.prefill_linear(W=Wgu, Xq=Xq, epilogue=mq.MQ_EPI_SILU_MUL_BF16, Y=Hb, ws=wsm)
        e[2].record()
        mq.prefill_linear(Hb, Wdn, Y=Y2, ws=wsh)
        e[3].record()
        rec2.append(e)
    for _ in range(3):
        mlp_unfused()
    rec2.clear()
    ms_u = _time_calls(torch, mlp_unfused, reps, flush)
    # NVFP4-vs-BF16 error of both on 64 tokens (BF16 reference through this library's BF16 GEMM)
    Wgu_bf = _to_dev(torch, wgu, dev)
    Wdn_bf = _to_dev(torch, wdn, dev)
    mlp()
    torch.cuda.synchronize()
    rows = torch.arange(0, Mm, Mm // 64, device=dev)
    g = mq.decode_linear(X[rows].contiguous(), Wgu_bf).float()
    hb = (torch.nn.functional.silu(g[:, :I]) * g[:, I:]).to(torch.bfloat16).contiguous()
    yb = mq.decode_linear(hb, Wdn_bf).double()

    def rel(yq):
        return float(torch.linalg.norm(yq[rows].double() - yb) / torch.linalg.norm(yb))
    out["fused_mlp"]["unfused_dynamic_alpha_h"] = {
        "ms": ms_u, "TFLOP/s": (fl_gu + fl_dn) / (ms_u * 1e-3) / 1e12,
        "gate_up_silu_bf16_ms": float(np.mean([e[1].elapsed_time(e[2]) for e in rec2])),
        "down_with_amax_quant_ms": float(np.mean([e[2].elapsed_time(e[3]) for e in rec2])),
        "speedup_of_fused_static": ms_u / ms,
        "nvfp4_vs_bf16_rel_frobenius": rel(Y2), "note": "64 tokens; the fused static-alpha_h path on the "
        "same tokens: see nvfp4_vs_bf16_rel_frobenius_fused_static"}
    out["fused_mlp"]["nvfp4_vs_bf16_rel_frobenius_fused_static"] = rel(Y)
    del Hb, Y2, wsh, Wgu_bf, Wdn_bf
    st = mq.async_status(wsm)
    if st != 0:
        raise RuntimeError(f"device error in the side measurements: {mq.STATUS_NAMES.get(st)}")
    return out


def measure_ragged_mlp(mq, torch, dev, fp4_peak, reps=3):
    """The ragged multi-turn prefill: 8 sequences of {2k, 4k, 8k, 8k, 16k, 16k, 32k, 42k}
    tokens (131072 in all, the 131K long context) through one Qwen3-8B MLP: dynamic
    activation quantization, gate/up GEMM with the SiLU-mul + NVFP4 requantization
    epilogue (static alpha_h calibrated once), down GEMM.  39.58 TFLOP per pass
    (2 * 131072 * (24576 * 4096 + 4096 * 12288)); the inputs (1 GB of X) are far
    larger than L2.  Per-sequence NVFP4-vs-BF16 output error on 32 sampled tokens
    of each sequence, the BF16 reference computed by the BF16 GEMM path of this
    library (decode_linear, 256 rows) with the SiLU-mul in FP32."""
    from phase_aware_nvfp4_b200 import workloads as wl
    x, off = wl.ragged_heavy_tailed_bf16(wl.RAGGED_LENGTHS, 4096, 5000)
    wgu, wdn = wl.mlp_weights(5000)
    M, K, I = x.shape[0], x.shape[1], wdn.shape[1]
    X = _to_dev(torch, x, dev)
    del x
    Wgu_bf = _to_dev(torch, wgu, dev)
    Wdn_bf = _to_dev(torch, wdn, dev)
    ws = mq.workspace(M, K, device=dev)
    Wgu = mq.quantize_weight(Wgu_bf, gate_up_interleave=True, ws=ws)
    Wdn = mq.quantize_weight(Wdn_bf, ws=ws)
    Xq = mq.nvfp4_empty(M, K, dev)
    H = mq.nvfp4_empty(M, I, dev)
    Y = torch.empty((M, wdn.shape[0]), dtype=torch.bfloat16, device=dev)
    # static alpha_h, calibrated once (offline): amax of h over this batch / (6 * 448)
    mq.quantize_activation(X, out=Xq, ws=ws)
    h_dbg = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
    one = torch.ones(1, dtype=torch.float32, device=dev)
    mq.prefill_linear(W=Wgu, Xq=Xq, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=one, H=H, h_debug=h_dbg, ws=ws)
    amax_h = float(h_dbg.float().abs().max())
    del h_dbg
    ah = torch.full((1,), amax_h / 2688.0 if amax_h > 0 else 1.0, dtype=torch.float32, device=dev)
    H.alpha.copy_(ah)
    rec = []

    def mlp():
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        mq.quantize_activation(X, out=Xq, ws=ws)
        e[1].record()
        mq.prefill_linear(W=Wgu, Xq=Xq, epilogue=mq.MQ_EPI_SILU_MUL_NVFP4, alpha_h=ah, H=H, ws=ws)
        e[2].record()
        mq.prefill_linear(W=Wdn, Xq=H, Y=Y, ws=ws)
        e[3].record()
        rec.append(e)
    mlp()
    torch.cuda.synchronize()
    rec.clear()
    for _ in range(reps):
        mlp()
    torch.cuda.synchronize()
    ms = float(np.mean([e[0].elapsed_time(e[3]) for e in rec]))
    q_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in rec]))
    gu_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in rec]))
    dn_ms = float(np.mean([e[2].elapsed_time(e[3]) for e in rec]))
    st = mq.async_status(ws)
    if st != 0:
        raise RuntimeError(f"device error in the ragged MLP: {mq.STATUS_NAMES.get(st)}")
    fl_gu, fl_dn = 2 * M * wgu.shape[0] * K, 2 * M * wdn.shape[0] * I
    tf = (fl_gu + fl_dn) / (ms * 1e-3) / 1e12
    # per-sequence NVFP4-vs-BF16 error on 32 sampled tokens per sequence
    rng = np.random.default_rng(5)
    rows = np.concatenate([np.sort(rng.choice(np.arange(off[i], off[i + 1]), 32, replace=False))
                           for i in range(len(wl.RAGGED_LENGTHS))])
    ridx = torch.as_tensor(rows, device=dev)
    g = mq.decode_linear(X[ridx].contiguous(), Wgu_bf).float()
    hb = (torch.nn.functional.silu(g[:, :I]) * g[:, I:]).to(torch.bfloat16).contiguous()
    yb = mq.decode_linear(hb, Wdn_bf).double()
    yq = Y[ridx].double()
    per_seq = []
    for i in range(len(wl.RAGGED_LENGTHS)):
        sl = slice(32 * i, 32 * (i + 1))
        per_seq.append(float(torch.linalg.norm(yq[sl] - yb[sl]) / torch.linalg.norm(yb[sl])))
    del X, Xq, H, Y, Wgu_bf, Wdn_bf
    return {"M": M, "lengths": list(wl.RAGGED_LENGTHS), "gate_up": [wgu.shape[0], K], "down": [wdn.shape[0], I],
            "flops": fl_gu + fl_dn, "ms": ms, "TFLOP/s": tf, "tokens_per_s": M / (ms * 1e-3),
            "frac": tf / fp4_peak, "quant_ms": q_ms, "gate_up_silu_requant_ms": gu_ms, "down_ms": dn_ms,
            "gate_up_TFLOP/s": fl_gu / (gu_ms * 1e-3) / 1e12, "down_TFLOP/s": fl_dn / (dn_ms * 1e-3) / 1e12,
            "nvfp4_vs_bf16_rel_frobenius_per_sequence": per_seq, "reps": reps,
            "l2": "inputs (1 GB) far larger than L2; no flush"}


def measure_library_gemm(torch, w, Wq, Xq, Y, flush, fp4_peak, reps=10):
    """Same-box context number: torch's block-scaled NVFP4 matmul (a library
    kernel) on the very operands the projection step quantized -- codes, E4M3
    block scales in the MMA scale layout (the "32_4_4" swizzle), and the FP32
    tensor scales -- timed like the step's GEMMs (L2 flushed before each call),
    with its output compared to the step's BF16 output as a cross-check."""
    import torch.nn.functional as F
    if not hasattr(torch, "float4_e2m1fn_x2") or not hasattr(F, "scaled_mm"):
        return {"unavailable": "this torch build has no NVFP4 scaled_mm"}
    ST, SW = F.ScalingType, F.SwizzleType

    def operands(t):
        rows, k16 = -(-t.rows // 128) * 128, -(-(t.cols // 16) // 4) * 4
        if t.scales.numel() != rows * k16:
            raise ValueError(f"scale buffer of {t.scales.numel()} bytes is not the library's {rows} x {k16}")
        return t.codes.view(torch.float4_e2m1fn_x2), t.scales.view(torch.float8_e4m3fn)

    out = {}
    for p in w.projections:
        xq, wq = Xq[p.x_group], Wq[p.name]
        try:
            a, sa = operands(xq)
            b, sb = operands(wq)

            def call(a=a, b=b, sa=sa, sb=sb, xq=xq, wq=wq):
                return F.scaled_mm(a, b.t(), [sa, xq.alpha], [ST.BlockWise1x16, ST.TensorWise],
                                   [sb, wq.alpha], [ST.BlockWise1x16, ST.TensorWise],
                                   swizzle_a=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE],
                                   swizzle_b=[SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE], output_dtype=torch.bfloat16)
            yl = call()
            torch.cuda.synchronize()
            yo = Y[p.name].double()
            rel = float(torch.linalg.norm(yl.double() - yo) / torch.linalg.norm(yo))
            del yl
            for _ in range(3):
                call()
            ms = _time_calls(torch, call, reps, flush)
            tf = p.flops / (ms * 1e-3) / 1e12
            out[p.name] = {"ms": ms, "TFLOP/s": tf, "frac": tf / fp4_peak, "rel_frobenius_vs_ours": rel}
        except Exception as e:     # the library's own argument checks; reported, not fatal
            out[p.name] = {"unavailable": f"{type(e).__name__}: {str(e).splitlines()[0][:200]}"}
    return out


def measure_e2e(torch, dist, world, dev, groups, xs_pin, X, Y, step, flops, K):
    """End to end through the public API with host buffers.  Every step copies
    its activations in from pinned host memory, runs the prefill pass and copies
    every output back to pinned host memory; all of it is inside the timed
    region.  The copies run on their own streams with two device buffer sets,
    so step i + 1's upload and step i - 1's download overlap step i's compute
    (PCIe is full duplex): the pipeline a serving loop would run."""
    Xb = [X, {g: torch.empty_like(t) for g, t in X.items()}]
    Yb = [Y, {n: torch.empty_like(t) for n, t in Y.items()}]
    y_pin = [{n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in Y.items()} for _ in range(2)]
    h2d = sum(t.numel() * 2 for t in xs_pin.values())
    d2h = sum(t.numel() * 2 for t in Y.values())
    ke = max(4, min(K, 20))
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def run(n_steps):
        ev = lambda: torch.cuda.Event(enable_timing=False)
        in_ready, x_free, y_ready, y_free = ([ev(), ev()] for _ in range(4))
        for b in range(2):   # every buffer starts free
            x_free[b].record(comp)
            y_free[b].record(comp)
        for i in range(n_steps):
            b = i % 2
            s_in.wait_event(x_free[b])
            with torch.cuda.stream(s_in):
                for g in groups:
                    Xb[b][g].copy_(xs_pin[g], non_blocking=True)
            in_ready[b].record(s_in)
            comp.wait_event(in_ready[b])
            comp.wait_event(y_free[b])
            step(False, Xs=Xb[b], Ys=Yb[b])
            x_free[b].record(comp)
            y_ready[b].record(comp)
            s_out.wait_event(y_ready[b])
            with torch.cuda.stream(s_out):
                for n in Y:
                    y_pin[b][n].copy_(Yb[b][n], non_blocking=True)
            y_free[b].record(s_out)
        for b in range(2):
            comp.wait_event(y_free[b])

    run(3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    s_in.wait_event(a)
    s_out.wait_event(a)
    run(ke)
    b.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / ke, dev)
    return {"value": whole_job_tflops(flops, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": ke,
            "h2d_GB/s": h2d / (e2e_ms * 1e-3) / 1e9, "d2h_GB/s": d2h / (e2e_ms * 1e-3) / 1e9,
            "pipeline": "upload, compute and download on three streams, two buffer sets: uploads and "
                        "downloads of neighbouring steps overlap each step's compute"}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from phase_aware_nvfp4_b200 import mixquant as mq

    w = workload(args.M)
    groups = groups_of(w)
    xs_h, ws_h = host_inputs(w)
    xs_pin = {g: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for g, x in xs_h.items()}
    X = {g: t.to(dev) for g, t in xs_pin.items()}
    Wd = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev) for n, a in ws_h.items()}
    ws = mq.workspace(device=dev)
    stream = torch.cuda.current_stream()

    # offline weight quantization (timed once, reported separately)
    Wq = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for p in w.projections:
        Wq[p.name] = mq.quantize_weight(Wd[p.name], ws=ws)
    e1.record()
    torch.cuda.synchronize()
    weight_quant_ms = e0.elapsed_time(e1)

    Xq = {g: mq.nvfp4_empty(args.M, ps[0].K, dev) for g, ps in groups.items()}
    Y = {p.name: torch.empty((p.M, p.N), dtype=torch.bfloat16, device=dev) for p in w.projections}
    flush = L2Flush(torch, dev)

    ev = {}

    def step(record: bool, i: int = 0, Xs=None, Ys=None):
        Xs = X if Xs is None else Xs
        Ys = Y if Ys is None else Ys
        for g, ps in groups.items():
            if record:
                ev[("q", g, i)][0].record()
            mq.quantize_activation(Xs[g], out=Xq[g], ws=ws)
            if record:
                ev[("q", g, i)][1].record()
            for p in ps:
                if record:
                    ev[("g", p.name, i)][0].record()
                mq.prefill_linear(W=Wq[p.name], Xq=Xq[g], Y=Ys[p.name], ws=ws)
                if record:
                    ev[("g", p.name, i)][1].record()

    for _ in range(args.warmup):
        flush()
        step(False)
    torch.cuda.synchronize()
    st = mq.async_status(ws)
    if st != 0:
        raise RuntimeError(f"device error during warm-up: {mq.STATUS_NAMES.get(st)}")

    K = args.steps
    for i in range(K):
        for g in groups:
            ev[("q", g, i)] = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        for p in w.projections:
            ev[("g", p.name, i)] = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    inst_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]

    # Timed region: K steps with events around each step only.  An event
    # recorded between two kernels would stop the second from launching while
    # the first drains (programmatic dependent launch), so the per-kernel
    # breakdown (roofline) comes from a second pass of K steps right after,
    # with events around every kernel; its step time is reported beside.
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local,
                      pci=(props.pci_domain_id, props.pci_bus_id, props.pci_device_id)) as clk:
        for i in range(K):
            flush()
            step_ev[i][0].record()
            step(False)
            step_ev[i][1].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        for i in range(K):
            flush()
            inst_ev[i][0].record()
            step(True, i)
            inst_ev[i][1].record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st = mq.async_status(ws)
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {mq.STATUS_NAMES.get(st)}")

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    ms = float(np.mean(step_ms))
    ms_instrumented = float(np.mean([a.elapsed_time(b) for a, b in inst_ev]))
    gemm_ms = {p.name: float(np.mean([ev[("g", p.name, i)][0].elapsed_time(ev[("g", p.name, i)][1])
                                      for i in range(K)])) for p in w.projections}
    quant_ms = {g: float(np.mean([ev[("q", g, i)][0].elapsed_time(ev[("q", g, i)][1]) for i in range(K)]))
                for g in groups}
    ms = max_over_ranks(ms, dev)

    flops = w.flops
    value = whole_job_tflops(flops, world, ms)
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = measured_peaks()
    fp4_peak = bf16_tf * FP4_PER_BF16
    gemm_flops = sum(p.flops for p in w.projections)
    gemm_total_ms = sum(gemm_ms.values())
    achieved = gemm_flops / (gemm_total_ms * 1e-3) / 1e12
    gsha = sources_sha(GEMM_SOURCES)
    cnt = counters_for("gemm_nvfp4", gsha)
    traffic = None
    if cnt is not None and "dram_bytes_per_launch" in cnt:
        traffic = float(np.mean(list(cnt["dram_bytes_per_launch"].values())))
    roofline = {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": achieved / fp4_peak, "traffic": traffic,
                "kernel": "gemm_nvfp4_pair_kernel<BF16 epilogue>",
                "peak_source": f"{peak_src} bf16_tflops (burst) x {FP4_PER_BF16:g} nominal FP4:BF16 ratio",
                "per_projection_tflops": {p.name: p.flops / (gemm_ms[p.name] * 1e-3) / 1e12
                                          for p in w.projections}}
    # quantizer: algorithmic bytes = amax read (2 B/elem) + quantize read (2) + codes/scales write (0.5625)
    q_bytes = {g: ps[0].M * ps[0].K * (2 + 2 + 0.5625) for g, ps in groups.items()}
    q_gbs = sum(q_bytes.values()) / (sum(quant_ms.values()) * 1e-3) / 1e9
    qcnt = counters_for("quantize_activation", sources_sha(QUANT_SOURCES))
    q_traffic = None
    if qcnt is not None and "dram_bytes_per_launch" in qcnt:
        q_traffic = float(np.mean(list(qcnt["dram_bytes_per_launch"].values())))
    roofline_quant = {"bound": "hbm", "achieved": q_gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": q_gbs / hbm_gbs,
                      "traffic": q_traffic, "kernel": "amax_kernel + quantize_kernel",
                      "bytes_per_elem": 4.5625, "ms": quant_ms}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4", "data": "synthetic", "config": config_of(w),
            "tokens_per_s": args.M * world / (ms * 1e-3),
            "fp4_peak_frac": value / world / fp4_peak,
            "roofline": roofline, "roofline_quant": roofline_quant,
            "gemm_ms": gemm_ms, "quant_ms": quant_ms, "weight_quant_ms_offline": weight_quant_ms,
            "breakdown": {"ms_per_step_with_kernel_events": ms_instrumented,
                          "note": "gemm_ms, quant_ms and the rooflines come from a second pass of the same K "
                                  "steps with events around every kernel; those events stop each kernel from "
                                  "launching while its predecessor drains, so the headline steps run without"},
            "gpu_launches": K * (2 * len(groups) + len(w.projections)),
            "clocks": clk.summary()}

    # end to end through the public API with host buffers: H2D of every
    # activation from pinned memory, the prefill pass, D2H of every output
    if not args.no_e2e:
        line["e2e"] = measure_e2e(torch, dist, world, dev, groups, xs_pin, X, Y, step, flops, K)

    if not args.no_extras:
        line["extras"] = measure_extras(mq, torch, dev, flush, hbm_gbs, fp4_peak)
        line["extras"]["library_nvfp4_gemm"] = measure_library_gemm(torch, w, Wq, Xq, Y, flush, fp4_peak)
        line["extras"]["ragged_mlp_131072"] = measure_ragged_mlp(mq, torch, dev, fp4_peak)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res = time_oracle(w, xs_h, ws_h, args.cpu_baseline_seconds, steps=1)
        line["cpu_baseline"] = {k: res[k] for k in ("value", "unit", "cores", "kind", "sample")}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
