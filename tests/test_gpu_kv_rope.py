"""K/V projection with RoPE and the KV-cache write fused into the NVFP4 GEMM epilogue
(mq_prefill_kv_rope) vs the oracle: block-scaled GEMM in FP64, rotate-half RoPE with the same
cos/sin table, BF16 K'/V at the token's cache slot."""
import numpy as np
import pytest
import torch

import oracle
from phase_aware_nvfp4_b200 import mixquant as mq
from phase_aware_nvfp4_b200 import workloads as wl

from gpu_helpers import GAMMA, require_gpu, to_dev, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _run(M, K, H, seed, max_pos=8192, extra_slots=37):
    rng = np.random.default_rng(seed)
    x = wl.heavy_tailed_bf16(M, K, seed)
    w = wl.normal_bf16(2 * H * 128, K, 0.02, seed + 1)
    pos = rng.integers(0, max_pos, size=M).astype(np.int32)
    num_slots = M + extra_slots
    slots = rng.permutation(num_slots)[:M].astype(np.int64)
    cs = wl.rope_cos_sin(max_pos)
    Wq = mq.quantize_weight(to_dev(w))
    kc = torch.zeros((num_slots, H, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros((num_slots, H, 128), dtype=torch.bfloat16, device="cuda")
    ws = mq.workspace(M, K)
    mq.prefill_kv_rope(to_dev(x), Wq, n_kv_heads=H, positions=torch.from_numpy(pos).cuda(),
                       cos_sin=torch.from_numpy(cs).cuda(), slots=torch.from_numpy(slots).cuda(), k_cache=kc,
                       v_cache=vc, ws=ws)
    torch.cuda.synchronize()
    assert mq.async_status(ws) == 0
    return x, w, pos, slots, cs, kc, vc, num_slots


def _check(x, w, pos, slots, cs, kc, vc, num_slots, rows):
    M = x.shape[0]
    H = w.shape[0] // 256
    ax, aw = oracle.tensor_alpha(x)[1], oracle.tensor_alpha(w)[1]
    y64, sabs = oracle.nvfp4_linear_rows((*oracle.quantize(x, ax), ax), (*oracle.quantize(w, aw), aw), rows)
    n = H * 128
    k_ref, v_ref = oracle.kv_rope_rows(y64[:, :n], y64[:, n:], pos[rows], cs)
    k_gpu = to_host_bits(kc[torch.from_numpy(slots[rows]).cuda()].reshape(len(rows), n))
    v_gpu = to_host_bits(vc[torch.from_numpy(slots[rows]).cuda()].reshape(len(rows), n))
    # bound: BF16 ulp + the FP32 accumulation bound carried through the rotation + binary32 rotation rounding
    csr = cs[pos[rows]].astype(np.float64)
    c = np.tile(np.concatenate([csr[:, :64], csr[:, :64]], axis=1), (1, H))
    s = np.tile(np.concatenate([csr[:, 64:], csr[:, 64:]], axis=1), (1, H))
    sk = sabs[:, :n].reshape(len(rows), H, 2, 64)
    s_swap = np.concatenate([sk[:, :, 1], sk[:, :, 0]], axis=2).reshape(len(rows), n)
    s_rot = sabs[:, :n] * np.abs(c) + s_swap * np.abs(s)
    for got, ref, sb in ((k_gpu, k_ref, s_rot), (v_gpu, v_ref, sabs[:, n:])):
        g, r = oracle.bf16_to_f64(got), oracle.bf16_to_f64(ref)
        ulp = np.maximum(oracle.bf16_ulp(r), oracle.bf16_ulp(g))
        bound = ulp + GAMMA * sb + 2.0 ** -20 * (np.abs(r) + sb * 0)
        err = np.abs(g - r)
        assert oracle.rel_frobenius(g, r) < 2e-3
        assert np.all(err <= bound), float((err - bound).max())
    # cache rows that no token maps to stay untouched
    free = np.setdiff1d(np.arange(num_slots), slots)
    assert not torch.any(kc[torch.from_numpy(free).cuda()].view(torch.int16) != 0)
    assert not torch.any(vc[torch.from_numpy(free).cuda()].view(torch.int16) != 0)


@pytest.mark.parametrize("M,K,H", [(300, 512, 2), (64, 256, 1), (129, 1024, 3)])
def test_kv_rope_vs_oracle(M, K, H):
    """M > 128 runs the CTA-pair kernel, M <= 128 the single-CTA kernel; ragged M in both."""
    x, w, pos, slots, cs, kc, vc, ns = _run(M, K, H, 80 + M)
    _check(x, w, pos, slots, cs, kc, vc, ns, np.arange(M))


def test_kv_rope_qwen3_8b_kv_projection_8192_tokens():
    """Qwen3-8B K/V shapes: 8 KV heads of 128 on a 4096 hidden size; sampled tokens."""
    x, w, pos, slots, cs, kc, vc, ns = _run(8192, 4096, 8, 90, max_pos=40960)
    rows = np.sort(np.random.default_rng(91).choice(8192, 48, replace=False))
    _check(x, w, pos, slots, cs, kc, vc, ns, rows)


def test_kv_rope_bad_position_is_reported():
    H, K, M = 1, 256, 16
    x = wl.heavy_tailed_bf16(M, K, 92)
    w = wl.normal_bf16(2 * H * 128, K, 0.02, 93)
    Wq = mq.quantize_weight(to_dev(w))
    cs = torch.from_numpy(wl.rope_cos_sin(64)).cuda()
    pos = torch.zeros(M, dtype=torch.int32, device="cuda")
    pos[3] = 64                                                # out of range
    slots = torch.arange(M, dtype=torch.int64, device="cuda")
    kc = torch.zeros((M, H, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ws = mq.workspace(M, K)
    mq.prefill_kv_rope(to_dev(x), Wq, n_kv_heads=H, positions=pos, cos_sin=cs, slots=slots, k_cache=kc,
                       v_cache=vc, ws=ws)
    assert mq.async_status(ws) == 9                           # MQ_ERR_INDEX
    torch.cuda.synchronize()
    assert not torch.any(kc[3].view(torch.int16) != 0)          # the bad token was not written
    assert torch.any(kc[2].view(torch.int16) != 0)


def test_kv_rope_pair_kernel_skips_bad_tokens_only():
    """CTA-pair kernel (M > 128), one K/V tile row with a position past the table and one with a
    negative slot: the call reports MQ_ERR_INDEX, those two tokens write nothing, and every other
    token's K'/V rows still match the oracle (the tile's index loads run one tile ahead)."""
    M, K, H, max_pos = 300, 512, 3, 4096
    rng = np.random.default_rng(94)
    x = wl.heavy_tailed_bf16(M, K, 95)
    w = wl.normal_bf16(2 * H * 128, K, 0.02, 96)
    pos = rng.integers(0, max_pos, size=M).astype(np.int32)
    num_slots = M + 11
    slots = rng.permutation(num_slots)[:M].astype(np.int64)
    bad_pos_row, bad_slot_row = 17, 250
    freed = slots[bad_slot_row]
    pos[bad_pos_row] = max_pos
    slots[bad_slot_row] = -1
    cs = wl.rope_cos_sin(max_pos)
    Wq = mq.quantize_weight(to_dev(w))
    kc = torch.zeros((num_slots, H, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ws = mq.workspace(M, K)
    mq.prefill_kv_rope(to_dev(x), Wq, n_kv_heads=H, positions=torch.from_numpy(pos).cuda(),
                       cos_sin=torch.from_numpy(cs).cuda(), slots=torch.from_numpy(slots).cuda(), k_cache=kc,
                       v_cache=vc, ws=ws)
    torch.cuda.synchronize()
    assert mq.async_status(ws) == 9                           # MQ_ERR_INDEX
    good = np.setdiff1d(np.arange(M), [bad_pos_row, bad_slot_row])
    # the two skipped tokens' rows: the bad-position token's own slot and the slot the
    # bad-slot token would have had are both left at zero
    for sl in (slots[bad_pos_row], freed):
        assert not torch.any(kc[int(sl)].view(torch.int16) != 0)
        assert not torch.any(vc[int(sl)].view(torch.int16) != 0)
    slots_chk = slots.copy()
    slots_chk[bad_slot_row] = freed
    _check(x, w, pos, slots_chk, cs, kc, vc, num_slots, good)
