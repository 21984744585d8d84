// mq_gemm.cu -- block-scaled NVFP4 x NVFP4 GEMM on sm_100a tensor cores.
//
// Y[M, N] = alpha_a * alpha_b * sum_k (sigma_a q_a)[m, k] (sigma_b q_b)[n, k]
// with FP32 accumulation in TMEM and a BF16 (or fused SiLU-mul + NVFP4
// requantize) epilogue: the prefill linear layer of "Mix-Quant: Quantized
// Prefilling, Precise Decoding for Agentic LLMs", section 3.3 (NVFP4 W4A4
// prefill; Eq. 2 gives xhat = alpha * sigma * q, so the matmul of the
// dequantized operands factors into the block-scaled MMA times the two
// tensor scales).
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: per K stage, A and B code tiles by tensor-map
//               TMA (128-byte swizzle), and the A/B scale atoms by bulk copy,
//               all completing on one mbarrier.
//   warp 1      TMEM owner and MMA issuer: copies the stage's scale atoms to
//               TMEM (tcgen05.cp) and issues 4 x tcgen05.mma kind::mxf4nvf4
//               (128 x 256 x 64 each) per stage; commits free the stage and,
//               at the end of a tile, signal the epilogue.
//   warps 2-5   epilogue: drain the 128 x 256 FP32 accumulator from TMEM
//               (one row per thread), release it to the MMA warp, then apply
//               the tensor scales and store BF16 (or SiLU-mul -> NVFP4).
// Stage = 256 K-elements (128 bytes per row, one swizzle row); 4 stages in
// flight.  TMEM: accumulator in columns [0, 256), scale factors in the 48
// columns from 256 (per stage: 4 x 4 columns for A, 4 x 8 columns for B, one
// 32-bit column per 32 rows per MMA).
#include "mq_device.cuh"

namespace mq {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;                  // K elements per stage
constexpr int BK_BYTES = BK / 2;         // packed FP4 bytes per row per stage
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK_BYTES;   // 16 KiB
constexpr int B_STAGE = BN * BK_BYTES;   // 32 KiB
constexpr int SFA_STAGE = 2048;          // 1 row block x 4 atoms
constexpr int SFB_STAGE = 4096;          // 2 row blocks x 4 atoms
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_STAGE;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // + barriers + alignment slack
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
// One scale-factor region (SFA 16 columns + SFB 32 columns per stage), rewritten
// every stage: copies and MMAs from one thread execute in issue order, so the
// copies of stage s+1 land after the MMAs of stage s have read stage s's
// scales.  (Alternating two regions measured slower: with a commit per stage
// the pipe then serialises the copies behind the previous stage's MMAs.)
constexpr uint32_t TMEM_SF = 256;
constexpr uint32_t IDESC = idesc_nvfp4(BM, BN);

struct Params {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* alpha_a;
    const float* alpha_b;
    int M, N, K;
    int num_m_blk, num_n_blk, num_tiles, k_stages;
    int n_fastest;      // tile order: 1 = n-block varies fastest, 0 = m-block fastest
    int sfa_atoms, sfb_atoms, sfb_rowblks;
    void* y;
    uint8_t* h_codes;
    uint8_t* h_scales;
    const float* h_alpha;
    uint16_t* h_debug;
    int h_atoms;
    const int32_t* positions;
    const float* cos_sin;
    int64_t max_pos;
    const int64_t* slots;
    uint16_t* k_cache;
    uint16_t* v_cache;
    int64_t num_slots;
    int n_heads;
    WsControl* ctrl;
};

// Tile index -> (m block, n block).  The block index of the operand with
// more bytes varies slowest: the CTAs resident at one time then share a few
// of its blocks and sweep all blocks of the smaller operand, which stays in
// L2, instead of every wave re-reading the larger one from HBM.
__device__ __forceinline__ void tile_coords(const Params& p, int tile, int& m_blk, int& n_blk)
{
    if (p.n_fastest) {
        n_blk = tile % p.num_n_blk;
        m_blk = tile / p.num_n_blk;
    } else {
        m_blk = tile % p.num_m_blk;
        n_blk = tile / p.num_m_blk;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

// Fused MLP epilogue for one 32-column chunk of a row: columns 0..15 are
// gate values and 16..31 the matching up values (the weight rows were
// interleaved in 16-row groups when quantized).  Produces 16 values of
// h = bf16(silu(g) * u) and quantizes them as one NVFP4 block with the
// static tensor scale alpha_h (Eq. 2 / Eq. 3 with alpha = alpha_h).
// h = bf16(silu(g) * u) of one 32-column chunk (16 gate columns, then the 16
// matching up columns), with g, u = fl(acc * fl(alpha_x * alpha_w)); returns
// the 16 values (exactly representable in BF16) and their |h| maximum.
__device__ __forceinline__ float silu_mul_chunk(const uint32_t (&acc)[32], float alpha_ab, float (&h)[16])
{
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const float g = __fmul_rn(__uint_as_float(acc[j]), alpha_ab);
        const float u = __fmul_rn(__uint_as_float(acc[16 + j]), alpha_ab);
        const float sg = __fdiv_rn(g, 1.0f + expf(-g));
        const float hv = __bfloat162float(__float2bfloat16_rn(__fmul_rn(sg, u)));
        h[j] = hv;
        amax = fmaxf(amax, fabsf(hv));
    }
    return amax;
}

__device__ __forceinline__ void silu_mul_quant_chunk(const uint32_t (&acc)[32], float alpha_ab, float alpha_h,
                                                     float alpha_h_qmax, uint32_t (&codes)[2], uint32_t& scale,
                                                     uint32_t (&hbits)[8])
{
    float h[16];
    const float amax = silu_mul_chunk(acc, alpha_ab, h);
#pragma unroll
    for (int j = 0; j < 8; ++j) hbits[j] = pack_bf16x2(h[2 * j], h[2 * j + 1]);
    const uint32_t sc = e4m3_round_sat(__fdiv_rn(amax, alpha_h_qmax));
    const float d = __fmul_rn(alpha_h, e4m3_to_float(sc));
    const float enc = (d == 0.0f) ? 0.0f : __fdiv_rn(1.0f, d);
    const float h0[8] = {h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7]};
    const float h1[8] = {h[8], h[9], h[10], h[11], h[12], h[13], h[14], h[15]};
    codes[0] = e2m1x8_encode(h0, enc);
    codes[1] = e2m1x8_encode(h1, enc);
    scale = sc;
}

struct EpiScales {
    float alpha_ab, alpha_h, alpha_h_qmax;
};

template <int EPI>
__device__ __forceinline__ EpiScales epi_scales(const Params& p)
{
    EpiScales e;
    e.alpha_ab = __fmul_rn(*p.alpha_a, *p.alpha_b);
    e.alpha_h = 1.0f;
    e.alpha_h_qmax = 6.0f;
    if (EPI == 1) {
        e.alpha_h = *p.h_alpha;
        e.alpha_h_qmax = __fmul_rn(e.alpha_h, 6.0f);
    }
    return e;
}

// Epilogue of one 256-column accumulator row block: this thread owns output
// row `row` and TMEM lane t_row.  Drains the 256 FP32 accumulators into
// registers, calls release() (the accumulator may then be overwritten by the
// next tile's MMAs), and only then stores BF16 Y, or (EPI 1) SiLU-mul ->
// NVFP4 h codes + scales (+ optional BF16 h).
// KV epilogue (EPI 2) for one token and one 128-column head: the projection
// columns are K heads 0..H-1 then V heads 0..H-1.  Values are
// fl(acc * fl(alpha_x*alpha_w)); K heads are rotated (rotate-half RoPE: pairs i,
// i+64 with c = cos_sin[pos][i], s = cos_sin[pos][64+i], k'_i = fl(fl(k_i c) -
// fl(k_{i+64} s)), k'_{i+64} = fl(fl(k_{i+64} c) + fl(k_i s))), then rounded to
// BF16 and stored at cache[slot][head][0..127].  A position or slot out of
// range posts kErrIndex and the row is not written.  acc[c][j] = column 32c + j.
__device__ __forceinline__ void kv_rope_store(const Params& p, float alpha_ab, int64_t m, int hh,
                                              uint32_t (&acc)[4][32])
{
    if (m >= p.M) return;
    const int32_t pos = __ldg(p.positions + m);
    const int64_t slot = __ldg(p.slots + m);
    if (pos < 0 || pos >= p.max_pos || slot < 0 || slot >= p.num_slots) {
        post_error(p.ctrl, kErrIndex);
        return;
    }
    const bool is_k = hh < p.n_heads;
    const int head = is_k ? hh : hh - p.n_heads;
    if (is_k) {
        const float4* cs = reinterpret_cast<const float4*>(p.cos_sin + (int64_t)pos * 128);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 cv = __ldg(cs + 8 * c + q);        // cos of frequencies 32c + 4q .. + 3
                const float4 sv = __ldg(cs + 16 + 8 * c + q);   // sin of the same
                const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
                const float ss[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int j = 4 * q + t;
                    const float a = __fmul_rn(__uint_as_float(acc[c][j]), alpha_ab);
                    const float b = __fmul_rn(__uint_as_float(acc[c + 2][j]), alpha_ab);
                    acc[c][j] = __float_as_uint(__fsub_rn(__fmul_rn(a, cc[t]), __fmul_rn(b, ss[t])));
                    acc[c + 2][j] = __float_as_uint(__fadd_rn(__fmul_rn(b, cc[t]), __fmul_rn(a, ss[t])));
                }
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[c][j] = __float_as_uint(__fmul_rn(__uint_as_float(acc[c][j]), alpha_ab));
    }
    uint4* dst = reinterpret_cast<uint4*>((is_k ? p.k_cache : p.v_cache) + (slot * p.n_heads + head) * 128);
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int j = 8 * q;
            dst[4 * c + q] = make_uint4(pack_bf16x2(__uint_as_float(acc[c][j]), __uint_as_float(acc[c][j + 1])),
                                        pack_bf16x2(__uint_as_float(acc[c][j + 2]), __uint_as_float(acc[c][j + 3])),
                                        pack_bf16x2(__uint_as_float(acc[c][j + 4]), __uint_as_float(acc[c][j + 5])),
                                        pack_bf16x2(__uint_as_float(acc[c][j + 6]), __uint_as_float(acc[c][j + 7])));
        }
}

template <int EPI, class Release>
__device__ __forceinline__ void epilogue_tile(const Params& p, const EpiScales& es, uint32_t t_row, int64_t row,
                                              int n_blk, Release release)
{
    if (EPI == 2) {
        // two heads per 256-column tile; TMEM is released after the second head's loads
        uint32_t acc[4][32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_row + 128 * h + 32 * c, acc[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_wait_ld(acc[c]);
            if (h == 1) {
                tc_fence_before();
                release();
            }
            kv_rope_store(p, es.alpha_ab, row, 2 * n_blk + h, acc);
        }
        return;
    }
    const int lane_ok = row < p.M;
    if (EPI == 3) {
        // SiLU-mul with a BF16 h output [M, N/2] in p.y (the unfused MLP path)
        uint32_t hb[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + 32 * c, r);
            tmem_wait_ld(r);
            float h[16];
            (void)silu_mul_chunk(r, es.alpha_ab, h);
#pragma unroll
            for (int j = 0; j < 8; ++j) hb[8 * c + j] = pack_bf16x2(h[2 * j], h[2 * j + 1]);
        }
        tc_fence_before();
        release();
        const int hN = p.N / 2;
        const int hcol0 = n_blk * (BN / 2);
        if (lane_ok && hcol0 < hN) {
            const int nch = min(8, (hN - hcol0) / 16);
            uint16_t* hrow = static_cast<uint16_t*>(p.y) + row * (int64_t)hN + hcol0;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < nch) {
                    reinterpret_cast<uint4*>(hrow)[2 * c] = make_uint4(hb[8 * c], hb[8 * c + 1], hb[8 * c + 2], hb[8 * c + 3]);
                    reinterpret_cast<uint4*>(hrow)[2 * c + 1] =
                        make_uint4(hb[8 * c + 4], hb[8 * c + 5], hb[8 * c + 6], hb[8 * c + 7]);
                }
        }
        return;
    }
    if (EPI == 0) {
        uint32_t out[128];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + 32 * c, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                out[16 * c + j] = pack_bf16x2(__fmul_rn(__uint_as_float(r[2 * j]), es.alpha_ab),
                                              __fmul_rn(__uint_as_float(r[2 * j + 1]), es.alpha_ab));
        }
        tc_fence_before();
        release();
        if (lane_ok) {
            uint16_t* yrow = static_cast<uint16_t*>(p.y) + row * (int64_t)p.N + (int64_t)n_blk * BN;
            const int ncols = min(BN, p.N - n_blk * BN);
#pragma unroll
            for (int q = 0; q < 32; ++q)
                if (8 * q < ncols)
                    reinterpret_cast<uint4*>(yrow)[q] = make_uint4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
        }
    } else {
        uint32_t codes[16];
        uint32_t scl[8];
        uint32_t hb[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + 32 * c, r);
            tmem_wait_ld(r);
            uint32_t cc[2], hbits[8];
            silu_mul_quant_chunk(r, es.alpha_ab, es.alpha_h, es.alpha_h_qmax, cc, scl[c], hbits);
            codes[2 * c] = cc[0];
            codes[2 * c + 1] = cc[1];
#pragma unroll
            for (int j = 0; j < 8; ++j) hb[8 * c + j] = hbits[j];
        }
        tc_fence_before();
        release();
        const int hN = p.N / 2;
        const int hcol0 = n_blk * (BN / 2);  // first h column of this tile
        if (lane_ok && hcol0 < hN) {
            const int nch = min(8, (hN - hcol0) / 16);
            uint8_t* crow = p.h_codes + row * (int64_t)(hN / 2) + hcol0 / 2;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < nch) *reinterpret_cast<uint2*>(crow + 8 * c) = make_uint2(codes[2 * c], codes[2 * c + 1]);
#pragma unroll
            for (int g = 0; g < 2; ++g)
                if (4 * g < nch) {
                    const int kb = hcol0 / 16 + 4 * g;
                    const uint32_t v = scl[4 * g] | (scl[4 * g + 1] << 8) | (scl[4 * g + 2] << 16) | (scl[4 * g + 3] << 24);
                    *reinterpret_cast<uint32_t*>(p.h_scales + sf_offset(row, kb, p.h_atoms)) = v;
                }
            if (p.h_debug != nullptr) {
                uint16_t* hrow = p.h_debug + row * (int64_t)hN + hcol0;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (c < nch) {
                        reinterpret_cast<uint4*>(hrow)[2 * c] = make_uint4(hb[8 * c], hb[8 * c + 1], hb[8 * c + 2], hb[8 * c + 3]);
                        reinterpret_cast<uint4*>(hrow)[2 * c + 1] =
                            make_uint4(hb[8 * c + 4], hb[8 * c + 5], hb[8 * c + 6], hb[8 * c + 7]);
                    }
            }
        }
    }
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* acc_full = empty_bar + STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* mma_done = acc_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 128);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
    }
    if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // set-up done: wait for the previous kernel of the stream (its outputs may
    // be this GEMM's operands or scales), and let the next one get scheduled
    grid_dep_wait();
    grid_dep_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // Whole warp (warp-uniform values); one elected lane issues the copies.
        {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_parity[STAGES];
            bool issued[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                int m_blk, n_blk;
                tile_coords(p, tile, m_blk, n_blk);
                const bool two_sfb = (2 * n_blk + 1) < p.sfb_rowblks;
                const uint32_t tx = A_STAGE + B_STAGE + SFA_STAGE + (two_sfb ? SFB_STAGE : SFB_STAGE / 2);
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!warp_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&full_bar[stage], tx);
                        tma_load_2d(smem + OFF_A + stage * A_STAGE, &tmap_a, &full_bar[stage], ks * BK_BYTES,
                                    m_blk * BM);
                        tma_load_2d(smem + OFF_B + stage * B_STAGE, &tmap_b, &full_bar[stage], ks * BK_BYTES,
                                    n_blk * BN);
                        bulk_load(smem + OFF_SFA + stage * SFA_STAGE,
                                  p.sfa + ((int64_t)m_blk * p.sfa_atoms + ks * 4) * 512, SFA_STAGE, &full_bar[stage]);
                        bulk_load(smem + OFF_SFB + stage * SFB_STAGE,
                                  p.sfb + ((int64_t)(2 * n_blk) * p.sfb_atoms + ks * 4) * 512, 2048, &full_bar[stage]);
                        if (two_sfb)
                            bulk_load(smem + OFF_SFB + stage * SFB_STAGE + 2048,
                                      p.sfb + ((int64_t)(2 * n_blk + 1) * p.sfb_atoms + ks * 4) * 512, 2048,
                                      &full_bar[stage]);
                    }
                    __syncwarp();
                    issued[stage] = true;
                    issued_parity[stage] = phase;
                    if (++stage == STAGES) stage = 0, phase ^= 1u;
                }
            }
            if (!ok) {
                if (lane == 0) {
                    post_error(p.ctrl, kErrTimeout);
                    *abort_flag = 1;
                }
                // let every copy already in flight land before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s]) (void)mbar_wait(&full_bar[s], issued_parity[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Whole warp; descriptors formed once and advanced by (offset >> 4)
        // in their 14-bit start-address field; one elected lane issues.
        {
            const uint64_t a_desc0 = sdesc_kmajor_sw128(smem_u32(smem + OFF_A));
            const uint64_t b_desc0 = sdesc_kmajor_sw128(smem_u32(smem + OFF_B));
            const uint64_t sfa_desc0 = sdesc_sf_block(smem_u32(smem + OFF_SFA));
            const uint64_t sfb_desc0 = sdesc_sf_block(smem_u32(smem + OFF_SFB));
            const uint32_t sfa_tmem = tmem_base + TMEM_SF;
            const uint32_t sfb_tmem = sfa_tmem + 16;
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, next_ready = false;
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                if (!warp_wait(acc_empty, acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!next_ready && !warp_wait(&full_bar[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    {   // look at the next ring stage now; its result is used next iteration
                        const int ns = (stage + 1 == STAGES) ? 0 : stage + 1;
                        next_ready = warp_test(&full_bar[ns], ns == 0 ? (phase ^ 1u) : phase);
                    }
                    const uint64_t a_d = a_desc0 + (uint64_t)((stage * A_STAGE) >> 4);
                    const uint64_t b_d = b_desc0 + (uint64_t)((stage * B_STAGE) >> 4);
                    const uint64_t sfa_d = sfa_desc0 + (uint64_t)((stage * SFA_STAGE) >> 4);
                    const uint64_t sfb_d = sfb_desc0 + (uint64_t)((stage * SFB_STAGE) >> 4);
                    // per k-block: its scale copies, then its MMA
                    if (elect_one()) {
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) {
                            tmem_cp_32x128b_x4(sfa_tmem + 4 * kb, sfa_d + (uint64_t)((kb * 512) >> 4));
                            tmem_cp_32x128b_x4(sfb_tmem + 8 * kb, sfb_d + (uint64_t)((kb * 512) >> 4));
                            tmem_cp_32x128b_x4(sfb_tmem + 8 * kb + 4, sfb_d + (uint64_t)((2048 + kb * 512) >> 4));
                            umma_nvfp4(tmem_base, a_d + (uint64_t)((kb * 32) >> 4), b_d + (uint64_t)((kb * 32) >> 4),
                                       IDESC, sfa_tmem + 4 * kb, sfb_tmem + 8 * kb, (ks | kb) != 0 ? 1u : 0u);
                        }
                        tc_commit(&empty_bar[stage]);
                    }
                    __syncwarp();
                    if (++stage == STAGES) stage = 0, phase ^= 1u;
                }
                if (!ok) break;
                if (elect_one()) tc_commit(acc_full);
                __syncwarp();
                acc_phase ^= 1u;
            }
            if (!ok && lane == 0) {
                post_error(p.ctrl, kErrTimeout);
                *abort_flag = 1;
            }
            // every MMA / copy issued above has finished before TMEM is freed
            if (elect_one()) tc_commit(mma_done);
            __syncwarp();
            (void)mbar_wait(mma_done, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int lg = warp & 3;  // TMEM lane group this warp may access
        EpiScales es = epi_scales<EPI>(p);
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            int m_blk, n_blk;
            tile_coords(p, tile, m_blk, n_blk);
            if (*abort_flag || !mbar_wait(acc_full, acc_phase)) {
                post_error(p.ctrl, kErrTimeout);
                *abort_flag = 1;
                break;
            }
            acc_phase ^= 1u;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(32 * lg) << 16);
            const int64_t row = (int64_t)m_blk * BM + 32 * lg + lane;
            epilogue_tile<EPI>(p, es, t_row, row, n_blk, [&] { mbar_arrive(acc_empty); });
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ==========================================================================
// CTA-pair kernel: 256 x 256 output tile per cluster of two CTAs
// ==========================================================================
//
// Each CTA of the pair loads its own 128 rows of A, its own 128 of the 256
// rows of B, the scale atoms of its A rows and all 256 rows of B scales; all
// loads signal the full barrier of the leader CTA (rank 0).  The leader
// alone issues the pair MMAs (tcgen05 cta_group::2, 256 x 256 x 64): each SM
// multiplies its A rows by the whole B tile, half of which it receives from
// the peer, and accumulates its 128 x 256 quarter... half of the tile in its
// own TMEM.  Per CTA and stage this moves 38 KB instead of 54 KB for the
// same FLOPs per SM, and five stages fit in shared memory.
constexpr int P_STAGES = 5;
constexpr int P_B_STAGE = 128 * BK_BYTES;  // this CTA's half of the B tile
constexpr int P_STAGE_BYTES = A_STAGE + P_B_STAGE + SFA_STAGE + SFB_STAGE;
constexpr int P_OFF_A = 0;
constexpr int P_OFF_B = P_OFF_A + P_STAGES * A_STAGE;
constexpr int P_OFF_SFA = P_OFF_B + P_STAGES * P_B_STAGE;
constexpr int P_OFF_SFB = P_OFF_SFA + P_STAGES * SFA_STAGE;
constexpr int P_STG_BYTES = 32 * 64 * 2;   // one warp's 32-row x 64-column BF16 output subtile
constexpr int P_OFF_STG = P_OFF_SFB + P_STAGES * SFB_STAGE;   // 8 epilogue warps x 1 buffer
constexpr int P_OFF_BAR = P_OFF_STG + 8 * P_STG_BYTES;
constexpr int P_SMEM_BYTES = P_OFF_BAR + 256 + 1024;
constexpr uint32_t P_IDESC = idesc_nvfp4(2 * BM, BN);
static_assert(P_SMEM_BYTES <= 232448, "pair kernel shared memory");
// Pair kernel warps: 0 TMA producer, 1 MMA issuer, 2-9 epilogue (warp w drains
// TMEM lane group w % 4, accumulator columns [128 * ((w - 2) / 4), + 128)).
constexpr int P_NUM_THREADS = 320;
constexpr int P_EPI_WARPS = 8;

// Pair-kernel epilogue: eight warps drain the 128 x 256 FP32 accumulator,
// two per TMEM lane group, each taking 32 rows x one 128-column half, so the
// accumulator is released after four TMEM loads per warp instead of eight.
// The release is per warp: every lane has waited for its loads, the warp
// synchronises and lane 0 arrives on the leader CTA's acc_empty barrier.
template <class Barrier>
__device__ __forceinline__ void release_acc_warp(int lane, Barrier arrive)
{
    tc_fence_before();
    __syncwarp();
    if (lane == 0) arrive();
}

// BF16 half-tile through shared memory: after the release, the warp writes
// its 32 rows x 128 columns as two 64-column subtiles into its 4 KiB staging
// buffer (128-byte swizzle) and stores each with one TMA tile store; the
// buffer is reused once the previous store has finished reading it.  Full
// 128-byte lines reach global memory instead of 16-byte pieces of 32 rows,
// which keeps the L1 / shared-memory port free for the tensor cores.  Only
// warp-level synchronisation is used, so a warp that leaves early (wait
// timeout) cannot block the others.  (x0, y0): first output column and first
// row of this warp's 32 x 128 block.
template <class Barrier>
__device__ __forceinline__ void epilogue_half_bf16_tma(const EpiScales& es, uint32_t t_col, int lane, uint8_t* stg,
                                                       const CUtensorMap* tmap_y, int32_t x0, int32_t y0,
                                                       Barrier arrive)
{
    // all four TMEM loads in flight, one wait, then release: the accumulator is
    // handed back to the MMA warp after one load latency instead of four
    uint32_t acc[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_col + 32 * c, acc[c]);
    tmem_wait_ld(acc[0]);
#pragma unroll
    for (int c = 1; c < 4; ++c) tmem_wait_ld(acc[c]);
    release_acc_warp(lane, arrive);
    uint32_t out[64];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 16; ++j)
            out[16 * c + j] = pack_bf16x2(__fmul_rn(__uint_as_float(acc[c][2 * j]), es.alpha_ab),
                                          __fmul_rn(__uint_as_float(acc[c][2 * j + 1]), es.alpha_ab));
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        // the store that last read the buffer is done reading it
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        uint8_t* rowp = stg + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int w = 32 * q + 4 * j;
            *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                make_uint4(out[w], out[w + 1], out[w + 2], out[w + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmap_y, stg, x0 + 64 * q, y0);
            bulk_commit_group();
        }
    }
}

// Unfused MLP half-tile (EPI 3): the warp's 32 rows x 128 accumulator columns
// are four 32-column gate/up chunks = 64 columns of h = bf16(silu(g) * u),
// written as one 32 x 64 BF16 subtile through the staging buffer with one TMA
// store (x0 = first h column, y0 = first row).
template <class Barrier>
__device__ __forceinline__ void epilogue_half_silu_bf16(const EpiScales& es, uint32_t t_col, int lane, uint8_t* stg,
                                                        const CUtensorMap* tmap_y, int32_t x0, int32_t y0,
                                                        Barrier arrive)
{
    uint32_t acc[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_col + 32 * c, acc[c]);
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_wait_ld(acc[c]);
    release_acc_warp(lane, arrive);
    uint32_t hb[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float h[16];
        (void)silu_mul_chunk(acc[c], es.alpha_ab, h);
#pragma unroll
        for (int j = 0; j < 8; ++j) hb[8 * c + j] = pack_bf16x2(h[2 * j], h[2 * j + 1]);
    }
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
    uint8_t* rowp = stg + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = make_uint4(hb[4 * j], hb[4 * j + 1], hb[4 * j + 2], hb[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmap_y, stg, x0, y0);
        bulk_commit_group();
    }
}

// KV half-tile (EPI 2) of the pair kernel.  The tile's 256 columns are two
// 128-column heads, A (columns 0..127) and B (128..255); the warp of half h
// takes frequencies 32h .. 32h + 31 of both heads, i.e. accumulator columns
// 32h + {0, 64, 128, 192} + 0..31, so the cos/sin values it needs (the 32
// tokens' rows at those frequencies) serve both heads.  Same arithmetic as
// kv_rope_store; the global traffic of a warp goes through its 4 KiB staging
// buffer (rows swizzled by 16-byte chunk, chunk ^ row % 8, so the row-wise and
// the column-wise passes are free of bank conflicts):
//   - the cos/sin values come in two chunks of 16 frequencies: per chunk the
//     warp loads 32 rows x (64 B of cos + 64 B of sin) with 16-byte loads,
//     eight lanes per row (kv_stage_cos_sin; the first chunk is staged before
//     the accumulator wait, so its latency overlaps the tile's MMAs), and each
//     lane then reads its own token's values;
//   - each rotated pair of columns is rounded to BF16 at once, and the result
//     leaves head by head: each lane writes its token's two 64-byte pieces
//     (columns 32h .. 32h + 31 and 64 + 32h .. 64 + 32h + 31 of the head row),
//     then the warp stores four lanes per piece.
// pos / slot / valid: this lane's token (loaded before the accumulator wait).
__device__ __forceinline__ void kv_stage_cos_sin(const Params& p, uint8_t* stg, int lane, int32_t pos, int ch)
{
    const int sub = lane >> 3, piece = lane & 7;
#pragma unroll 4
    for (int j = 0; j < 8; ++j) {
        const int r = sub + 4 * j;
        const int32_t pr = __shfl_sync(0xFFFFFFFFu, pos, r);
        const float* src =
            p.cos_sin + (int64_t)pr * 128 + (piece < 4 ? 16 * ch + 4 * piece : 64 + 16 * ch + 4 * (piece - 4));
        *reinterpret_cast<float4*>(stg + r * 128 + ((piece ^ (r & 7)) << 4)) =
            __ldg(reinterpret_cast<const float4*>(src));
    }
    __syncwarp();
}

template <class Barrier>
__device__ __forceinline__ void epilogue_half_kv(const Params& p, float alpha_ab, uint32_t t_col, int lane,
                                                 uint8_t* stg, int half, int n_blk, int32_t pos, int64_t slot,
                                                 bool valid, Barrier arrive)
{
    uint32_t acc[4][32];   // [head A low, head A high, head B low, head B high][frequency 32 half + j]
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_col + 64 * c, acc[c]);
    tmem_wait_ld(acc[0]);
#pragma unroll
    for (int c = 1; c < 4; ++c) tmem_wait_ld(acc[c]);
    release_acc_warp(lane, arrive);

    // K heads come first, so head B is a K head only if head A is one
    const bool rot_a = 2 * n_blk < p.n_heads, rot_b = 2 * n_blk + 1 < p.n_heads;
    uint32_t out[4][16];   // BF16 pairs: out[c][w] holds frequencies 32 half + 2w, + 2w + 1 of stream c
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
        if (rot_a && ch > 0) kv_stage_cos_sin(p, stg, lane, pos, 2 * half + 1);   // chunk 2 half was staged before the wait
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float cc[4] = {1.f, 1.f, 1.f, 1.f}, ss[4] = {0.f, 0.f, 0.f, 0.f};
            if (rot_a) {
                // cos and sin of frequencies 32 half + 16 ch + 4 q .. + 3 from this token's staged row
                const float4 cv = *reinterpret_cast<const float4*>(stg + lane * 128 + ((q ^ (lane & 7)) << 4));
                const float4 sv = *reinterpret_cast<const float4*>(stg + lane * 128 + (((q + 4) ^ (lane & 7)) << 4));
                cc[0] = cv.x, cc[1] = cv.y, cc[2] = cv.z, cc[3] = cv.w;
                ss[0] = sv.x, ss[1] = sv.y, ss[2] = sv.z, ss[3] = sv.w;
            }
#pragma unroll
            for (int hd = 0; hd < 2; ++hd) {
                const bool rot = hd == 0 ? rot_a : rot_b;
                float lo[4], hi[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int j = 16 * ch + 4 * q + t;
                    const float a = __fmul_rn(__uint_as_float(acc[2 * hd][j]), alpha_ab);
                    const float b = __fmul_rn(__uint_as_float(acc[2 * hd + 1][j]), alpha_ab);
                    if (rot) {
                        lo[t] = __fsub_rn(__fmul_rn(a, cc[t]), __fmul_rn(b, ss[t]));
                        hi[t] = __fadd_rn(__fmul_rn(b, cc[t]), __fmul_rn(a, ss[t]));
                    } else {
                        lo[t] = a;
                        hi[t] = b;
                    }
                }
                const int w = 8 * ch + 2 * q;
                out[2 * hd][w] = pack_bf16x2(lo[0], lo[1]);
                out[2 * hd][w + 1] = pack_bf16x2(lo[2], lo[3]);
                out[2 * hd + 1][w] = pack_bf16x2(hi[0], hi[1]);
                out[2 * hd + 1][w + 1] = pack_bf16x2(hi[2], hi[3]);
            }
        }
        __syncwarp();   // the next chunk's loads (or the stores) overwrite the staging rows
    }
    const int sub = lane >> 3, piece = lane & 7;
    // destination column of this lane's 16-byte piece: low half (pieces 0..3)
    // or high half (4..7) of the head row, at the warp's 32 frequencies
    const int col = (piece < 4 ? 0 : 64) + 32 * half + 8 * (piece & 3);
#pragma unroll
    for (int hd = 0; hd < 2; ++hd) {
        const int hh = 2 * n_blk + hd;
        const bool is_k = hh < p.n_heads;
        const int head = is_k ? hh : hh - p.n_heads;
        uint16_t* cache = is_k ? p.k_cache : p.v_cache;
        // this token's two pieces: staged chunks 0..3 = low, 4..7 = high
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint32_t* o = out[2 * hd + (q >> 2)] + 4 * (q & 3);
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((q ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = sub + 4 * j;
            const int64_t sr = __shfl_sync(0xFFFFFFFFu, slot, r);
            const int vr = __shfl_sync(0xFFFFFFFFu, valid ? 1 : 0, r);
            if (vr) {
                uint4* dst = reinterpret_cast<uint4*>(cache + (sr * p.n_heads + head) * 128 + col);
                *dst = *reinterpret_cast<const uint4*>(stg + r * 128 + ((piece ^ (r & 7)) << 4));
            }
        }
        __syncwarp();
    }
}

// Fused MLP half-tile (EPI 1): accumulator columns [128*half, 128*half + 128)
// are four 32-column chunks (16 gate + 16 up each) = 64 h columns = one
// 64-wide group of four NVFP4 blocks, whose four scale bytes form one 32-bit
// word of the scale layout.
template <class Barrier>
__device__ __forceinline__ void epilogue_half_mlp(const Params& p, const EpiScales& es, uint32_t t_col, int half,
                                                  int64_t row, int n_blk, int lane, Barrier arrive)
{
    // drain the raw accumulator first and release TMEM, so the next tile's
    // MMAs run while this warp does the SiLU-mul and requantization
    uint32_t acc[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_col + 32 * c, acc[c]);
    tmem_wait_ld(acc[0]);
#pragma unroll
    for (int c = 1; c < 4; ++c) tmem_wait_ld(acc[c]);
    release_acc_warp(lane, arrive);
    uint32_t codes[8];
    uint32_t scl[4];
    uint32_t hb[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t cc[2], hbits[8];
        silu_mul_quant_chunk(acc[c], es.alpha_ab, es.alpha_h, es.alpha_h_qmax, cc, scl[c], hbits);
        codes[2 * c] = cc[0];
        codes[2 * c + 1] = cc[1];
#pragma unroll
        for (int j = 0; j < 8; ++j) hb[8 * c + j] = hbits[j];
    }
    const int hN = p.N / 2;
    const int hcol0 = n_blk * (BN / 2) + 64 * half;   // first h column of this half
    const int nch = min(4, (hN - hcol0) / 16);
    if (row < p.M && nch > 0) {
        uint8_t* crow = p.h_codes + row * (int64_t)(hN / 2) + hcol0 / 2;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c < nch) *reinterpret_cast<uint2*>(crow + 8 * c) = make_uint2(codes[2 * c], codes[2 * c + 1]);
        const uint32_t v = scl[0] | (scl[1] << 8) | (scl[2] << 16) | (scl[3] << 24);
        *reinterpret_cast<uint32_t*>(p.h_scales + sf_offset(row, hcol0 / 16, p.h_atoms)) = v;
        if (p.h_debug != nullptr) {
            uint16_t* hrow = p.h_debug + row * (int64_t)hN + hcol0;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (c < nch) {
                    reinterpret_cast<uint4*>(hrow)[2 * c] = make_uint4(hb[8 * c], hb[8 * c + 1], hb[8 * c + 2], hb[8 * c + 3]);
                    reinterpret_cast<uint4*>(hrow)[2 * c + 1] =
                        make_uint4(hb[8 * c + 4], hb[8 * c + 5], hb[8 * c + 6], hb[8 * c + 7]);
                }
        }
    }
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_NUM_THREADS, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                           const __grid_constant__ CUtensorMap tmap_y, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + P_OFF_BAR);
    uint64_t* empty_bar = full_bar + P_STAGES;
    uint64_t* acc_full = empty_bar + P_STAGES;
    uint64_t* acc_empty = acc_full + 1;   // used in the leader: both CTAs' epilogues arrive
    uint64_t* mma_done = acc_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * P_EPI_WARPS);   // one arrival per epilogue warp of both CTAs
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
        prefetch_tensormap(&tmap_sfa);
        prefetch_tensormap(&tmap_sfb);
        if (EPI == 0 || EPI == 3) prefetch_tensormap(&tmap_y);
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    cluster_barrier();   // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // set-up done: wait for the previous kernel of the stream (its outputs may
    // be this GEMM's operands or scales), and let the next one get scheduled
    grid_dep_wait();
    grid_dep_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        // Whole warp, warp-uniform values; one elected lane issues the copies.
        {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const uint32_t full0 = map_to_cta(smem_u32(&full_bar[0]), 0);
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int m_blk, n_blk;
                tile_coords(p, tile, m_blk, n_blk);
                const int a_row = m_blk * 2 * BM + (int)rank * BM;
                const int b_row = n_blk * BN + (int)rank * 128;
                const int sfa_row = (m_blk * 2 + (int)rank) * p.sfa_atoms;
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!warp_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (elect_one()) {
                        if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * P_STAGE_BYTES);
                        const uint32_t bar = full0 + 8u * (uint32_t)stage;
                        tma_load_2d_pair(smem + P_OFF_A + stage * A_STAGE, &tmap_a, bar, ks * BK_BYTES, a_row);
                        tma_load_2d_pair(smem + P_OFF_B + stage * P_B_STAGE, &tmap_b, bar, ks * BK_BYTES, b_row);
                        tma_load_2d_pair(smem + P_OFF_SFA + stage * SFA_STAGE, &tmap_sfa, bar, 0, sfa_row + ks * 4);
                        tma_load_3d_pair(smem + P_OFF_SFB + stage * SFB_STAGE, &tmap_sfb, bar, 0, ks * 4, 2 * n_blk);
                    }
                    __syncwarp();
                    if (++stage == P_STAGES) stage = 0, phase ^= 1u;
                }
            }
            if (!ok && lane == 0) {
                post_error(p.ctrl, kErrTimeout);
                *abort_flag = 1;
            }
            // Every load issued above has landed before this CTA may leave:
            // the stage it last filled is released by the leader only after
            // the MMAs that read it (and so after the copy completed).
            if (ok) {
                for (int s = 0; s < P_STAGES; ++s) {
                    (void)mbar_wait(&empty_bar[stage], phase ^ 1u);
                    if (++stage == P_STAGES) stage = 0, phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader CTA)
        // The whole warp runs the loop, so every address and descriptor is
        // warp-uniform; one elected lane issues the copies, MMAs and commits.
        // Descriptors are formed once and advanced by adding (offset >> 4) to
        // their 14-bit start-address field (shared addresses stay below 256 KB,
        // so the field never carries into its neighbours).
        if (leader) {
            const uint64_t a_desc0 = sdesc_kmajor_sw128(smem_u32(smem + P_OFF_A));
            const uint64_t b_desc0 = sdesc_kmajor_sw128(smem_u32(smem + P_OFF_B));
            const uint64_t sfa_desc0 = sdesc_sf_block(smem_u32(smem + P_OFF_SFA));
            const uint64_t sfb_desc0 = sdesc_sf_block(smem_u32(smem + P_OFF_SFB));
            const uint32_t sfa_tmem = tmem_base + TMEM_SF;
            const uint32_t sfb_tmem = sfa_tmem + 16;
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, next_ready = false;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                if (!warp_wait(acc_empty, acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!next_ready && !warp_wait(&full_bar[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    {   // look at the next ring stage now; its result is used next iteration
                        const int ns = (stage + 1 == P_STAGES) ? 0 : stage + 1;
                        next_ready = warp_test(&full_bar[ns], ns == 0 ? (phase ^ 1u) : phase);
                    }
                    const uint64_t a_d = a_desc0 + (uint64_t)((stage * A_STAGE) >> 4);
                    const uint64_t b_d = b_desc0 + (uint64_t)((stage * P_B_STAGE) >> 4);
                    const uint64_t sfa_d = sfa_desc0 + (uint64_t)((stage * SFA_STAGE) >> 4);
                    const uint64_t sfb_d = sfb_desc0 + (uint64_t)((stage * SFB_STAGE) >> 4);
                    if (elect_one()) {
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) {
                            tmem_cp_32x128b_x4_pair(sfa_tmem + 4 * kb, sfa_d + (uint64_t)((kb * 512) >> 4));
                            tmem_cp_32x128b_x4_pair(sfb_tmem + 8 * kb, sfb_d + (uint64_t)((kb * 512) >> 4));
                            tmem_cp_32x128b_x4_pair(sfb_tmem + 8 * kb + 4, sfb_d + (uint64_t)((2048 + kb * 512) >> 4));
                            umma_nvfp4_pair(tmem_base, a_d + (uint64_t)((kb * 32) >> 4), b_d + (uint64_t)((kb * 32) >> 4),
                                            P_IDESC, sfa_tmem + 4 * kb, sfb_tmem + 8 * kb, (ks | kb) != 0 ? 1u : 0u);
                        }
                        tc_commit_pair_mc(&empty_bar[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == P_STAGES) stage = 0, phase ^= 1u;
                }
                if (!ok) break;
                if (elect_one()) tc_commit_pair_mc(acc_full, 0x3);
                __syncwarp();
                acc_phase ^= 1u;
            }
            if (!ok && lane == 0) {
                post_error(p.ctrl, kErrTimeout);
                *abort_flag = 1;
            }
            if (elect_one()) tc_commit_pair(mma_done);
            __syncwarp();
            (void)mbar_wait(mma_done, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int lg = warp & 3;
        const int half = (warp - 2) >> 2;
        EpiScales es = epi_scales<EPI>(p);
        const uint32_t leader_acc_empty = map_to_cta(smem_u32(acc_empty), 0);
        // column offset of this warp's accumulator half: 128 columns of the tile,
        // or (KV) 32 columns in each of the four 64-column quarters
        const uint32_t t_col = tmem_base + ((uint32_t)(32 * lg) << 16) + (uint32_t)(EPI == 2 ? 32 * half : 128 * half);
        uint8_t* stg = smem + P_OFF_STG + (warp - 2) * P_STG_BYTES;
        auto arrive = [&] { mbar_arrive_cluster(leader_acc_empty); };
        uint32_t acc_phase = 0;
        // KV epilogue: this lane's token position and cache slot for a tile,
        // loaded one tile ahead (the loads of the next tile are in flight
        // during this tile's epilogue) and checked at the top of the tile: an
        // out-of-range one posts kErrIndex and the token is not written
        int32_t nx_pos = -1;
        int64_t nx_slot = -1;
        bool nx_in = false;
        auto kv_fetch = [&](int t) {
            int mb, nb;
            tile_coords(p, t, mb, nb);
            const int64_t m = (int64_t)mb * 2 * BM + (int64_t)rank * BM + 32 * lg + lane;
            nx_in = m < p.M;
            if (nx_in) {
                nx_pos = __ldg(p.positions + m);
                nx_slot = __ldg(p.slots + m);
            }
        };
        if (EPI == 2 && pair < p.num_tiles) kv_fetch(pair);
        for (int tile = pair; tile < p.num_tiles; tile += npairs) {
            int m_blk, n_blk;
            tile_coords(p, tile, m_blk, n_blk);
            int32_t kv_pos = 0;
            int64_t kv_slot = 0;
            bool kv_valid = false;
            if (EPI == 2 && nx_in) {
                kv_valid = nx_pos >= 0 && nx_pos < p.max_pos && nx_slot >= 0 && nx_slot < p.num_slots;
                if (kv_valid) {
                    kv_pos = nx_pos;
                    kv_slot = nx_slot;
                } else {
                    post_error(p.ctrl, kErrIndex);
                }
            }
            if (EPI == 2 && 2 * n_blk < p.n_heads) kv_stage_cos_sin(p, stg, lane, kv_pos, 2 * half);
            if (!warp_wait(acc_full, acc_phase, abort_flag)) {
                if (lane == 0) {
                    post_error(p.ctrl, kErrTimeout);
                    *abort_flag = 1;
                }
                break;
            }
            acc_phase ^= 1u;
            tc_fence_after();
            if (EPI == 2 && tile + npairs < p.num_tiles) kv_fetch(tile + npairs);
            const int64_t row0 = (int64_t)m_blk * 2 * BM + (int64_t)rank * BM + 32 * lg;
            if (EPI == 0) {
                epilogue_half_bf16_tma(es, t_col, lane, stg, &tmap_y, n_blk * BN + 128 * half, (int32_t)row0, arrive);
            } else if (EPI == 1) {
                epilogue_half_mlp(p, es, t_col, half, row0 + lane, n_blk, lane, arrive);
            } else if (EPI == 3) {
                epilogue_half_silu_bf16(es, t_col, lane, stg, &tmap_y, n_blk * (BN / 2) + 64 * half, (int32_t)row0,
                                        arrive);
            } else {
                epilogue_half_kv(p, es.alpha_ab, t_col, lane, stg, half, n_blk, kv_pos, kv_slot, kv_valid, arrive);
            }
        }
        // every output store has finished before the CTA may leave
        if ((EPI == 0 || EPI == 3) && lane == 0) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_barrier();   // no CTA leaves while its peer may still read its smem or TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ==========================================================================
// Wide CTA-pair kernel (BF16 epilogue): 256 x 384 output tile per pair
// ==========================================================================
//
// The same pipeline with a 384-column tile: per k-block two pair MMAs share
// the A operand, one over tile columns 0..255 (N = 256: B rows 0..127 from
// the leader, 128..255 from its peer) and one over columns 256..383 (N = 128:
// rows 256..319 from the leader, 320..383 from its peer).  Per SM and k-block
// that is 128 rows of A and 192 rows of B for 128 x 384 products, against 128
// and 128 for 128 x 256 in the square tile: a sixth fewer operand bytes per
// FLOP, and with a quarter fewer tile changes the accumulator hand-over to the
// epilogue is paid less often.  TMEM: accumulator columns 0..383, scale
// factors from 384 (A: 4 columns per k-block, B: 12).  Shared memory: four
// 48 KiB stages.  A tile narrower than 384 (the last one, when N % 384 == 256)
// issues only the N = 256 MMA.
constexpr int W_STAGES = 4;
constexpr int W_B0 = 128 * BK_BYTES;                 // B rows for the N = 256 MMA
constexpr int W_B1 = 64 * BK_BYTES;                  // B rows for the N = 128 MMA
constexpr int W_B_STAGE = W_B0 + W_B1;               // 24 KiB
constexpr int W_SFB_STAGE = 3 * 2048;                // three 128-row blocks x 4 atoms
constexpr int W_STAGE_BYTES = A_STAGE + W_B_STAGE + SFA_STAGE + W_SFB_STAGE;
constexpr int W_OFF_A = 0;
constexpr int W_OFF_B = W_OFF_A + W_STAGES * A_STAGE;
constexpr int W_OFF_SFA = W_OFF_B + W_STAGES * W_B_STAGE;
constexpr int W_OFF_SFB = W_OFF_SFA + W_STAGES * SFA_STAGE;
constexpr int W_OFF_STG = W_OFF_SFB + W_STAGES * W_SFB_STAGE;
constexpr int W_OFF_BAR = W_OFF_STG + 8 * P_STG_BYTES;
constexpr int W_SMEM_BYTES = W_OFF_BAR + 256 + 1024;
constexpr int WN = 384;
constexpr uint32_t W_TMEM_SF = 384;
constexpr uint32_t W_IDESC0 = idesc_nvfp4(2 * BM, 256);
constexpr uint32_t W_IDESC1 = idesc_nvfp4(2 * BM, 128);
static_assert(W_SMEM_BYTES <= 232448, "wide pair kernel shared memory");

// Epilogue of the wide kernel: warp (lane group lg, half) drains accumulator
// columns [192 half, 192 half + ncols) (ncols is 192, or 64 for the second
// half of a 256-wide tile), releases the accumulator, and stores 64-column
// BF16 subtiles through its staging buffer.
template <class Barrier>
__device__ __forceinline__ void epilogue_wide_bf16(const EpiScales& es, uint32_t t_col, int ncols, int lane,
                                                   uint8_t* stg, const CUtensorMap* tmap_y, int32_t x0, int32_t y0,
                                                   Barrier arrive)
{
    // one 32-column load at a time, packed to BF16 at once: the packed row
    // (96 registers) and one raw chunk stay within the register budget
    uint32_t out[96];
#pragma unroll
    for (int c = 0; c < 6; ++c) {
        if (32 * c < ncols) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_col + 32 * c, r);
            tmem_wait_ld(r);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                out[16 * c + j] = pack_bf16x2(__fmul_rn(__uint_as_float(r[2 * j]), es.alpha_ab),
                                              __fmul_rn(__uint_as_float(r[2 * j + 1]), es.alpha_ab));
        }
    }
    release_acc_warp(lane, arrive);
#pragma unroll
    for (int q = 0; q < 3; ++q) {
        if (64 * q >= ncols) break;
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        uint8_t* rowp = stg + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int w = 32 * q + 4 * j;
            *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                make_uint4(out[w], out[w + 1], out[w + 2], out[w + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmap_y, stg, x0 + 64 * q, y0);
            bulk_commit_group();
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_NUM_THREADS, 1)
    gemm_nvfp4_wide_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ CUtensorMap tmap_b64, const __grid_constant__ CUtensorMap tmap_sfa,
                           const __grid_constant__ CUtensorMap tmap_sfb3, const __grid_constant__ CUtensorMap tmap_y,
                           const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + W_OFF_BAR);
    uint64_t* empty_bar = full_bar + W_STAGES;
    uint64_t* acc_full = empty_bar + W_STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* mma_done = acc_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * P_EPI_WARPS);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
        prefetch_tensormap(&tmap_b64);
        prefetch_tensormap(&tmap_sfa);
        prefetch_tensormap(&tmap_sfb3);
        prefetch_tensormap(&tmap_y);
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    cluster_barrier();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dep_wait();
    grid_dep_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        const uint32_t full0 = map_to_cta(smem_u32(&full_bar[0]), 0);
        for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
            int m_blk, n_blk;
            tile_coords(p, tile, m_blk, n_blk);
            const int a_row = m_blk * 2 * BM + (int)rank * BM;
            const int n0 = n_blk * WN;
            const int sfa_row = (m_blk * 2 + (int)rank) * p.sfa_atoms;
            for (int ks = 0; ks < p.k_stages; ++ks) {
                if (!warp_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * W_STAGE_BYTES);
                    const uint32_t bar = full0 + 8u * (uint32_t)stage;
                    uint8_t* sb = smem + W_OFF_B + stage * W_B_STAGE;
                    tma_load_2d_pair(smem + W_OFF_A + stage * A_STAGE, &tmap_a, bar, ks * BK_BYTES, a_row);
                    tma_load_2d_pair(sb, &tmap_b, bar, ks * BK_BYTES, n0 + (int)rank * 128);
                    tma_load_2d_pair(sb + W_B0, &tmap_b64, bar, ks * BK_BYTES, n0 + 256 + (int)rank * 64);
                    tma_load_2d_pair(smem + W_OFF_SFA + stage * SFA_STAGE, &tmap_sfa, bar, 0, sfa_row + ks * 4);
                    tma_load_3d_pair(smem + W_OFF_SFB + stage * W_SFB_STAGE, &tmap_sfb3, bar, 0, ks * 4, 3 * n_blk);
                }
                __syncwarp();
                if (++stage == W_STAGES) stage = 0, phase ^= 1u;
            }
        }
        if (!ok && lane == 0) {
            post_error(p.ctrl, kErrTimeout);
            *abort_flag = 1;
        }
        if (ok) {
            for (int s = 0; s < W_STAGES; ++s) {
                (void)mbar_wait(&empty_bar[stage], phase ^ 1u);
                if (++stage == W_STAGES) stage = 0, phase ^= 1u;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader CTA)
        if (leader) {
            const uint64_t a_desc0 = sdesc_kmajor_sw128(smem_u32(smem + W_OFF_A));
            const uint64_t b_desc0 = sdesc_kmajor_sw128(smem_u32(smem + W_OFF_B));
            const uint64_t sfa_desc0 = sdesc_sf_block(smem_u32(smem + W_OFF_SFA));
            const uint64_t sfb_desc0 = sdesc_sf_block(smem_u32(smem + W_OFF_SFB));
            const uint32_t sfa_tmem = tmem_base + W_TMEM_SF;
            const uint32_t sfb_tmem = sfa_tmem + 16;
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true, next_ready = false;
            for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
                int m_blk, n_blk;
                tile_coords(p, tile, m_blk, n_blk);
                const bool wide = p.N - n_blk * WN > 256;   // else only the N = 256 MMA
                if (!warp_wait(acc_empty, acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!next_ready && !warp_wait(&full_bar[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    {
                        const int ns = (stage + 1 == W_STAGES) ? 0 : stage + 1;
                        next_ready = warp_test(&full_bar[ns], ns == 0 ? (phase ^ 1u) : phase);
                    }
                    const uint64_t a_d = a_desc0 + (uint64_t)((stage * A_STAGE) >> 4);
                    const uint64_t b0_d = b_desc0 + (uint64_t)((stage * W_B_STAGE) >> 4);
                    const uint64_t b1_d = b0_d + (uint64_t)(W_B0 >> 4);
                    const uint64_t sfa_d = sfa_desc0 + (uint64_t)((stage * SFA_STAGE) >> 4);
                    const uint64_t sfb_d = sfb_desc0 + (uint64_t)((stage * W_SFB_STAGE) >> 4);
                    if (elect_one()) {
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) {
                            const uint32_t acc = (ks | kb) != 0 ? 1u : 0u;
                            tmem_cp_32x128b_x4_pair(sfa_tmem + 4 * kb, sfa_d + (uint64_t)((kb * 512) >> 4));
                            tmem_cp_32x128b_x4_pair(sfb_tmem + 12 * kb, sfb_d + (uint64_t)((kb * 512) >> 4));
                            tmem_cp_32x128b_x4_pair(sfb_tmem + 12 * kb + 4, sfb_d + (uint64_t)((2048 + kb * 512) >> 4));
                            if (wide)
                                tmem_cp_32x128b_x4_pair(sfb_tmem + 12 * kb + 8,
                                                        sfb_d + (uint64_t)((4096 + kb * 512) >> 4));
                            umma_nvfp4_pair(tmem_base, a_d + (uint64_t)((kb * 32) >> 4), b0_d + (uint64_t)((kb * 32) >> 4),
                                            W_IDESC0, sfa_tmem + 4 * kb, sfb_tmem + 12 * kb, acc);
                            if (wide)
                                umma_nvfp4_pair(tmem_base + 256, a_d + (uint64_t)((kb * 32) >> 4),
                                                b1_d + (uint64_t)((kb * 32) >> 4), W_IDESC1, sfa_tmem + 4 * kb,
                                                sfb_tmem + 12 * kb + 8, acc);
                        }
                        tc_commit_pair_mc(&empty_bar[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == W_STAGES) stage = 0, phase ^= 1u;
                }
                if (!ok) break;
                if (elect_one()) tc_commit_pair_mc(acc_full, 0x3);
                __syncwarp();
                acc_phase ^= 1u;
            }
            if (!ok && lane == 0) {
                post_error(p.ctrl, kErrTimeout);
                *abort_flag = 1;
            }
            if (elect_one()) tc_commit_pair(mma_done);
            __syncwarp();
            (void)mbar_wait(mma_done, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int lg = warp & 3;
        const int half = (warp - 2) >> 2;
        EpiScales es = epi_scales<0>(p);
        const uint32_t leader_acc_empty = map_to_cta(smem_u32(acc_empty), 0);
        const uint32_t t_col = tmem_base + ((uint32_t)(32 * lg) << 16) + (uint32_t)(192 * half);
        uint8_t* stg = smem + W_OFF_STG + (warp - 2) * P_STG_BYTES;
        auto arrive = [&] { mbar_arrive_cluster(leader_acc_empty); };
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < p.num_tiles; tile += npairs) {
            int m_blk, n_blk;
            tile_coords(p, tile, m_blk, n_blk);
            if (!warp_wait(acc_full, acc_phase, abort_flag)) {
                if (lane == 0) {
                    post_error(p.ctrl, kErrTimeout);
                    *abort_flag = 1;
                }
                break;
            }
            acc_phase ^= 1u;
            tc_fence_after();
            const int64_t row0 = (int64_t)m_blk * 2 * BM + (int64_t)rank * BM + 32 * lg;
            const int width = min(WN, p.N - n_blk * WN);          // 384, or 256 for a last narrower tile
            const int ncols = min(192, width - 192 * half);       // 192 or 64
            epilogue_wide_bf16(es, t_col, ncols, lane, stg, &tmap_y, n_blk * WN + 192 * half, (int32_t)row0, arrive);
        }
        if (lane == 0) bulk_wait_group<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_barrier();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <int EPI>
cudaError_t launch_pair(int pairs, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsfa,
                        const CUtensorMap& tsfb, const CUtensorMap& ty, const Params& p, cudaStream_t s)
{
    auto k = gemm_nvfp4_pair_kernel<EPI>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(2 * pairs), dim3(P_NUM_THREADS), P_SMEM_BYTES, s, ta, tb, tsfa, tsfb, ty, p);
}

template <int EPI>
cudaError_t launch_single(int grid, const CUtensorMap& ta, const CUtensorMap& tb, const Params& p, cudaStream_t s)
{
    auto k = gemm_nvfp4_kernel<EPI>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, s, ta, tb, p);
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const GemmArgs& a, const DeviceInfo& di, cudaStream_t s)
{
    Params p{};
    p.sfa = a.a_scales;
    p.sfb = a.b_scales;
    p.alpha_a = a.a_alpha;
    p.alpha_b = a.b_alpha;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    const int num_n_blk = (int)((a.N + BN - 1) / BN);
    p.k_stages = (int)((a.K + BK - 1) / BK);
    p.sfa_atoms = (int)sf_atoms_per_rowblk(a.K);
    p.sfb_atoms = (int)sf_atoms_per_rowblk(a.K);
    p.sfb_rowblks = (int)sf_rowblks(a.N);
    p.y = a.y;
    p.h_codes = a.h_codes;
    p.h_scales = a.h_scales;
    p.h_alpha = a.h_alpha;
    p.h_debug = a.h_debug;
    p.h_atoms = (int)sf_atoms_per_rowblk(a.N / 2);
    p.positions = a.positions;
    p.cos_sin = a.cos_sin;
    p.max_pos = a.max_pos;
    p.slots = a.slots;
    p.k_cache = a.k_cache;
    p.v_cache = a.v_cache;
    p.num_slots = a.num_slots;
    p.n_heads = a.n_heads;
    p.ctrl = a.ctrl;

    CUtensorMap ta, tb;
    // A codes [M rows, K/2 bytes], B codes [N rows, K/2 bytes]: 128-byte-wide
    // boxes with the 128-byte swizzle the UMMA descriptors assume.
    if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, (uint64_t)(a.K / 2), (uint64_t)a.M,
                      (uint64_t)(a.K / 2), BK_BYTES, BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    if (a.M > BM) {
        // CTA-pair kernel: 256 x 256 tiles
        CUtensorMap tsfa, tsfb;
        if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_codes, (uint64_t)(a.K / 2), (uint64_t)a.N,
                          (uint64_t)(a.K / 2), BK_BYTES, 128, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        // scale buffers viewed as rows of one 512-byte atom (128 x u32); a box is 4 atoms
        const uint64_t a_atoms = (uint64_t)sf_rowblks(a.M) * (uint64_t)p.sfa_atoms;
        if (!make_tmap_2d(&tsfa, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.a_scales, 128, a_atoms, 512, 128, 4,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
        // B scales as [row blocks][atoms][128 x u32]: one box = 4 atoms of the two
        // 128-row blocks of a 256-row tile
        if (!make_tmap_3d(&tsfb, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.b_scales, 128, (uint64_t)p.sfb_atoms,
                          (uint64_t)p.sfb_rowblks, 512, (uint64_t)p.sfb_atoms * 512, 128, 4, 2))
            return cudaErrorInvalidValue;
        // output for the TMA-store epilogues, 64-column x 32-row boxes (one warp's
        // rows): Y [M, N] BF16 (EPI 0) or h [M, N/2] BF16 (EPI 3)
        CUtensorMap ty = tb;
        if (a.epilogue == 0 || a.epilogue == 3) {
            const uint64_t cols = a.epilogue == 0 ? (uint64_t)a.N : (uint64_t)a.N / 2;
            if (!make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, cols, (uint64_t)a.M, cols * 2, 64, 32,
                              CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        }
        p.num_m_blk = (int)((a.M + 2 * BM - 1) / (2 * BM));
        p.n_fastest = a.M > a.N;   // A (M rows) is the larger operand: sweep N fastest
        // 256 x 384 tiles (the last one 256 wide when N % 384 == 256) when they
        // do not cost more waves of the persistent grid than 256 x 256 tiles: a
        // wide tile does 1.5 times the work of a square one at ~3 % better
        // throughput (measured on the 8192 x 12288 x 4096 projection)
        const int pairs_avail = std::max(1, di.num_sms / 2);
        const int64_t waves_sq = ((int64_t)p.num_m_blk * num_n_blk + pairs_avail - 1) / pairs_avail;
        const int64_t waves_w = ((int64_t)p.num_m_blk * ((a.N + WN - 1) / WN) + pairs_avail - 1) / pairs_avail;
        if (a.epilogue == 0 && a.N >= 3072 && (a.N % WN == 0 || a.N % WN == 256) &&
            (double)waves_w * 1.5 * 0.97 < (double)waves_sq) {
            CUtensorMap tb64, tsfb3;
            if (!make_tmap_2d(&tb64, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_codes, (uint64_t)(a.K / 2), (uint64_t)a.N,
                              (uint64_t)(a.K / 2), BK_BYTES, 64, CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
            if (!make_tmap_3d(&tsfb3, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.b_scales, 128, (uint64_t)p.sfb_atoms,
                              (uint64_t)p.sfb_rowblks, 512, (uint64_t)p.sfb_atoms * 512, 128, 4, 3))
                return cudaErrorInvalidValue;
            p.num_n_blk = (int)((a.N + WN - 1) / WN);
            p.num_tiles = p.num_m_blk * p.num_n_blk;
            const int pairs = std::min(p.num_tiles, di.num_sms / 2);
            cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 W_SMEM_BYTES);
            if (e != cudaSuccess) return e;
            return launch_pdl(gemm_nvfp4_wide_kernel, dim3(2 * pairs), dim3(P_NUM_THREADS), W_SMEM_BYTES, s, ta, tb,
                              tb64, tsfa, tsfb3, ty, p);
        }
        p.num_n_blk = num_n_blk;
        p.num_tiles = p.num_m_blk * num_n_blk;
        const int pairs = std::min(p.num_tiles, di.num_sms / 2);
        switch (a.epilogue) {
            case 0: return launch_pair<0>(pairs, ta, tb, tsfa, tsfb, ty, p, s);
            case 1: return launch_pair<1>(pairs, ta, tb, tsfa, tsfb, ty, p, s);
            case 2: return launch_pair<2>(pairs, ta, tb, tsfa, tsfb, ty, p, s);
            case 3: return launch_pair<3>(pairs, ta, tb, tsfa, tsfb, ty, p, s);
        }
        return cudaErrorInvalidValue;
    }

    // single-CTA kernel for short activations (M <= 128): 128 x 256 tiles
    if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_codes, (uint64_t)(a.K / 2), (uint64_t)a.N,
                      (uint64_t)(a.K / 2), BK_BYTES, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    p.num_m_blk = (int)((a.M + BM - 1) / BM);
    p.num_n_blk = num_n_blk;
    p.num_tiles = p.num_m_blk * num_n_blk;
    p.n_fastest = 0;   // M <= 128: a single m block
    const int grid = std::min(p.num_tiles, di.num_sms);
    switch (a.epilogue) {
        case 0: return launch_single<0>(grid, ta, tb, p, s);
        case 1: return launch_single<1>(grid, ta, tb, p, s);
        case 2: return launch_single<2>(grid, ta, tb, p, s);
        case 3: return launch_single<3>(grid, ta, tb, p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace mq
