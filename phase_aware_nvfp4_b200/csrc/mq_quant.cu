// mq_quant.cu -- NVFP4 quantization on sm_100a: the tensor-level scale
// (tensor amax) and the block quantizer, after "Mix-Quant: Quantized
// Prefilling, Precise Decoding for Agentic LLMs", section 3.3, Eq. 2 and Eq. 3.
//
// Large tensors: an HBM-bound amax kernel, then the quantization kernel.
// Tensors of at most one 128 x 256 tile per SM: one cooperative launch of the
// quantization kernel takes the amax, hands alpha to every block through a
// bounded grid-wide wait, and quantizes (reading X back from L2), which saves
// a launch on the decode-sized inputs.
#include <mutex>

#include <map>
#include <utility>

#include "mq_device.cuh"

namespace mq {

// Grid-stride steps per loop trip of the amax pass (16: 2 us less than 4 per
// 64 MB activation, same at 201 MB and on the single-launch sizes).
#ifndef MQ_AMAX_UNROLL
#define MQ_AMAX_UNROLL 16
#endif
#ifndef MQ_AMAX_BLOCKS_PER_SM
#define MQ_AMAX_BLOCKS_PER_SM 4
#endif
constexpr int kAmaxThreads = 512;
constexpr int kAmaxUnroll = MQ_AMAX_UNROLL;

// Fast path: magnitude maximum including NaN/Inf (two operations per word).
// A maximum halfword >= 0x7F80 means a non-finite value was seen; only then
// is the thread's range scanned again with amax_accum.
__device__ __forceinline__ void amax_accum_fast(uint32_t w, uint32_t& mx)
{
    mx = max_u16x2(mx, w & 0x7FFF7FFFu);
}

__global__ void __launch_bounds__(kAmaxThreads, MQ_AMAX_BLOCKS_PER_SM) amax_kernel(const uint4* __restrict__ x, int64_t n_vec,
                                                            float* __restrict__ alpha_out, WsControl* ctrl,
                                                            uint32_t* __restrict__ partials)
{
    grid_dep_wait();   // X may be the previous kernel's output
    grid_dep_launch_dependents();
    uint32_t mx = 0, bad = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t i = i0;
    for (; i + (kAmaxUnroll - 1) * stride < n_vec; i += kAmaxUnroll * stride) {
        uint4 v[kAmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) v[u] = __ldg(x + i + u * stride);
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) {
            amax_accum_fast(v[u].x, mx);
            amax_accum_fast(v[u].y, mx);
            amax_accum_fast(v[u].z, mx);
            amax_accum_fast(v[u].w, mx);
        }
    }
    for (; i < n_vec; i += stride) {
        const uint4 v = __ldg(x + i);
        amax_accum_fast(v.x, mx);
        amax_accum_fast(v.y, mx);
        amax_accum_fast(v.z, mx);
        amax_accum_fast(v.w, mx);
    }
    if (max(mx & 0xFFFFu, mx >> 16) >= 0x7F80u) {
        // a NaN/Inf in this thread's range: rescan it for the finite maximum
        mx = 0;
        for (i = i0; i < n_vec; i += stride) {
            const uint4 v = __ldg(x + i);
            amax_accum(v.x, mx, bad);
            amax_accum(v.y, mx, bad);
            amax_accum(v.z, mx, bad);
            amax_accum(v.w, mx, bad);
        }
    }
    uint32_t m = max(mx & 0xFFFFu, mx >> 16) | (bad ? 0x80000000u : 0u);
    // block reduction (the non-finite flag rides in bit 31)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, m, o);
        m = max(m & 0x7FFFFFFFu, other & 0x7FFFFFFFu) | ((m | other) & 0x80000000u);
    }
    __shared__ uint32_t warp_max[kAmaxThreads / 32];
    __shared__ bool is_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) warp_max[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < kAmaxThreads / 32; ++w)
            b = max(b & 0x7FFFFFFFu, warp_max[w] & 0x7FFFFFFFu) | ((b | warp_max[w]) & 0x80000000u);
        partials[blockIdx.x] = b;
        const uint32_t ticket = atom_add_acq_rel_gpu(&ctrl->amax_ticket, 1u);   // releases the partial
        is_last = (ticket == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    // The last block to finish folds all partial maxima (visible after its
    // ticket's acquire and the barrier).
    uint32_t b = 0;
    for (int j = threadIdx.x; j < (int)gridDim.x; j += blockDim.x) {
        const uint32_t p = __ldcg(partials + j);
        b = max(b & 0x7FFFFFFFu, p & 0x7FFFFFFFu) | ((b | p) & 0x80000000u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, b, o);
        b = max(b & 0x7FFFFFFFu, other & 0x7FFFFFFFu) | ((b | other) & 0x80000000u);
    }
    __syncthreads();
    if (lane == 0) warp_max[warp] = b;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0;
        for (int w = 0; w < kAmaxThreads / 32; ++w)
            r = max(r & 0x7FFFFFFFu, warp_max[w] & 0x7FFFFFFFu) | ((r | warp_max[w]) & 0x80000000u);
        const float amax = __uint_as_float((r & 0x7FFFu) << 16);
        // tensor scale: amax / (q_max * E4M3_max) = amax / 2688, or 1 for an all-zero tensor
        *alpha_out = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
        if (r & 0x80000000u) post_error(ctrl, kErrNonFinite);
        ctrl->amax_ticket = 0;  // ready for the next pass on this workspace (visible at kernel end)
    }
}

cudaError_t launch_amax(const void* x, int64_t n, float* alpha_out, WsControl* ctrl, uint32_t* partials,
                        const DeviceInfo& di, cudaStream_t s)
{
    const int64_t n_vec = n / 8;
    int64_t blocks = (n_vec + kAmaxThreads * kAmaxUnroll - 1) / (kAmaxThreads * kAmaxUnroll);
    const int64_t cap = (int64_t)di.num_sms * MQ_AMAX_BLOCKS_PER_SM;
    if (blocks > cap) blocks = cap;
    if (blocks > kAmaxMaxBlocks) blocks = kAmaxMaxBlocks;
    if (blocks < 1) blocks = 1;
    return launch_pdl(amax_kernel, dim3((unsigned)blocks), dim3(kAmaxThreads), 0, s, static_cast<const uint4*>(x),
                      n_vec, alpha_out, ctrl, partials);
}

// ==========================================================================
// Block quantizer: BF16 [rows, K] -> NVFP4 codes + E4M3 block scales
// ==========================================================================
//
// One CTA tile = 128 rows x 256 columns = 4 scale atoms (2048 contiguous
// bytes of the scale layout); 8 warps, warp w owns rows 16w..16w+15.  Each
// thread owns one 16-element block per step: a half-warp covers one row's
// 256 columns (two 16-byte loads per thread, 512 contiguous bytes per
// half-warp), so the block amax needs no shuffles and the per-block work
// (two products and one conversion for the E4M3 scale, one table lookup for
// its reciprocal) is paid once per 16 elements.  Codes
// come from the conversion instruction (two per cvt) and leave as one
// 8-byte store per thread; scales are staged in shared memory and written
// as 16-byte stores.
//
// Tiles are visited in reverse order: when the amax pass has just streamed
// the tensor front to back, its tail is still in L2 and is consumed first.

#ifndef MQ_QUANT_UNROLL
#define MQ_QUANT_UNROLL 4
#endif
#ifndef MQ_QUANT_MIN_BLOCKS
#define MQ_QUANT_MIN_BLOCKS 4
#endif
constexpr int kQuantThreads = 256;
constexpr int64_t kQuantLeanTiles = 2048;   // tiles from which the lean quantize kernel is used
constexpr int kQuantStepUnroll = MQ_QUANT_UNROLL;   // steps (2 rows per warp each) with loads in flight

// Fills enc_tab[c] = fl(1 / fl(alpha * sigma_c)) for every E4M3 code c (0 when
// the product is 0) and returns the block-scale constants.  Every thread of
// the block calls it; it ends with __syncthreads().
__device__ __forceinline__ QuantConsts quant_setup(float alpha, float* enc_tab, float* dec_tab)
{
    const QuantConsts q = quant_consts(alpha);
    if (threadIdx.x < 128) {
        const float d = __fmul_rn(alpha, e4m3_to_float((uint32_t)threadIdx.x));
        enc_tab[threadIdx.x] = (d == 0.0f) ? 0.0f : __frcp_rn(d);
        dec_tab[threadIdx.x] = d;
    }
    __syncthreads();
    return q;
}

// Source row of output row r (gate/up interleave in 16-row groups when
// interleave_half > 0: output row 32c+t <- input row 16c+t for t < 16,
// I+16c+t-16 otherwise).
__device__ __forceinline__ int64_t quant_src_row(int64_t r, int64_t interleave_half)
{
    if (interleave_half <= 0) return r;
    const int64_t c = r >> 5, tt = r & 31;
    return (tt < 16) ? (16 * c + tt) : (interleave_half + 16 * c + (tt - 16));
}

// The work split of one 128-row x 256-column tile: warp w owns rows 16w..16w+15,
// taken two per step (lanes 0-15 the even row, 16-31 the odd one); lane l
// owns the 16-element block l % 16 of the row.  The same split is used for the
// amax pass and the quantization pass, so both read the same lines.
__device__ __forceinline__ uint32_t amax_tile(const uint16_t* __restrict__ x, int64_t rows, int64_t K,
                                              int64_t interleave_half, int64_t rb, int64_t kc, int warp, int half,
                                              int blk, uint32_t mx)
{
    const int64_t col = kc * 256 + 16 * blk;
    if (col >= K) return mx;
#pragma unroll 1
    for (int s0 = 0; s0 < 8; s0 += kQuantStepUnroll) {
        uint4 v[kQuantStepUnroll][2];
#pragma unroll
        for (int u = 0; u < kQuantStepUnroll; ++u) {   // all loads of the group in flight together
            const int64_t r = rb * 128 + 16 * warp + 2 * (s0 + u) + half;
            v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows) {
                const uint4* p = reinterpret_cast<const uint4*>(x + quant_src_row(r, interleave_half) * K + col);
                v[u][0] = __ldg(p);
                v[u][1] = __ldg(p + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kQuantStepUnroll; ++u) {
            const uint4 a = v[u][0], b = v[u][1];
            mx = max_u16x2(mx, max_u16x2(max_u16x2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu),
                                         max_u16x2(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu)));
            mx = max_u16x2(mx, max_u16x2(max_u16x2(b.x & 0x7FFF7FFFu, b.y & 0x7FFF7FFFu),
                                         max_u16x2(b.z & 0x7FFF7FFFu, b.w & 0x7FFF7FFFu)));
        }
    }
    return mx;
}

// Same tile, finite values only; bad |= non-zero if a NaN/Inf was seen.
__device__ __noinline__ uint32_t amax_tile_finite(const uint16_t* __restrict__ x, int64_t rows, int64_t K,
                                                  int64_t interleave_half, int64_t rb, int64_t kc, int warp, int half,
                                                  int blk, uint32_t mx, uint32_t& bad)
{
    const int64_t col = kc * 256 + 16 * blk;
    if (col >= K) return mx;
    for (int st = 0; st < 8; ++st) {
        const int64_t r = rb * 128 + 16 * warp + 2 * st + half;
        if (r < rows) {
            const uint4* p = reinterpret_cast<const uint4*>(x + quant_src_row(r, interleave_half) * K + col);
            const uint4 a = __ldg(p), b = __ldg(p + 1);
            amax_accum(a.x, mx, bad);
            amax_accum(a.y, mx, bad);
            amax_accum(a.z, mx, bad);
            amax_accum(a.w, mx, bad);
            amax_accum(b.x, mx, bad);
            amax_accum(b.y, mx, bad);
            amax_accum(b.z, mx, bad);
            amax_accum(b.w, mx, bad);
        }
    }
    return mx;
}

// Squared error of one coded 16-element block in binary32, element order
// 0..15: y = fl(d * v) with v the signed E2M1 value of the code, r = fl(x - y),
// e = fl(e + fl(r * r)).  Codes: nibble j of c0 / c1 is element j / 8 + j.
__device__ __forceinline__ float block_sq_error(const float (&f0)[8], const float (&f1)[8], uint32_t c0, uint32_t c1,
                                                float d)
{
    // E2M1 magnitude index -> 2 x value {0, 1, 2, 3, 4, 6, 8, 12}, one nibble each
    constexpr uint32_t kTwiceValue = 0xC8643210u;
    float e = 0.0f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t c = h ? c1 : c0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t nib = (c >> (4 * j)) & 15u;
            const float mag = (float)((kTwiceValue >> (4 * (nib & 7u))) & 15u) * 0.5f;   // exact
            const float v = (nib & 8u) ? -mag : mag;
            const float y = __fmul_rn(d, v);
            const float r = __fsub_rn(h ? f1[j] : f0[j], y);
            e = __fadd_rn(e, __fmul_rn(r, r));
        }
    }
    return e;
}

// Eq. 3 / Eq. 2 for one tile; scales staged in shared memory and written as
// one contiguous 2 KiB run of the MMA scale layout.
// With `search`, each block also tries the E4M3 neighbours of its Eq. 3 scale
// code (c0 - 1, then c0 + 1) and keeps the first with the smallest squared
// error, so ties keep the Eq. 3 scale.
// With NORM the loaded x are first replaced by h = bf16(fl(fl(x * rstd_row) *
// gamma_k)) (RMSNorm; rstd from rmsnorm_amax_kernel), optionally written to
// h_out, and h is quantized.
struct NormArgs {
    const uint16_t* gamma;   // [K] BF16
    const float* rstd;       // [rows]
    uint16_t* h_out;         // optional [rows, K] BF16
};

__device__ __forceinline__ uint32_t norm_pair(uint32_t xw, uint32_t gw, float r)
{
    float t0, t1, lo, hi;
    fmul2_rn(bf16_lo(xw), bf16_hi(xw), r, t0, t1);             // fl(x * rstd)
    fmul2v_rn(t0, t1, bf16_lo(gw), bf16_hi(gw), lo, hi);       // fl(fl(x * rstd) * gamma)
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

template <bool SEARCH, bool NORM>
__device__ __forceinline__ void quant_tile(const uint16_t* __restrict__ x, int64_t rows, int64_t K,
                                           int64_t interleave_half, int64_t rb, int64_t kc, int64_t chunks,
                                           const QuantConsts& qc, const float* enc_tab, const float* dec_tab,
                                           uint8_t* sf_stage, uint8_t* __restrict__ codes,
                                           uint8_t* __restrict__ scales, int warp, int half, int blk,
                                           const NormArgs& na)
{
    const int64_t col = kc * 256 + 16 * blk;
    const bool col_ok = col < K;
#pragma unroll 1
    for (int s0 = 0; s0 < 8; s0 += kQuantStepUnroll) {
        uint4 v[kQuantStepUnroll][2];
#pragma unroll
        for (int u = 0; u < kQuantStepUnroll; ++u) {
            const int64_t r = rb * 128 + 16 * warp + 2 * (s0 + u) + half;
            v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
            if (r < rows && col_ok) {
                const uint4* p = reinterpret_cast<const uint4*>(x + quant_src_row(r, interleave_half) * K + col);
                v[u][0] = __ldcs(p);
                v[u][1] = __ldcs(p + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kQuantStepUnroll; ++u) {
            const int rl = 16 * warp + 2 * (s0 + u) + half;   // row within the 128-row block
            const int64_t r = rb * 128 + rl;
            uint32_t w[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                             v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
            if (NORM && r < rows && col_ok) {
                const float rs = __ldg(na.rstd + r);
                const uint4 g0 = __ldg(reinterpret_cast<const uint4*>(na.gamma + col));
                const uint4 g1 = __ldg(reinterpret_cast<const uint4*>(na.gamma + col) + 1);
                const uint32_t g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) w[j] = norm_pair(w[j], g[j], rs);
                if (na.h_out != nullptr) {
                    uint4* hp = reinterpret_cast<uint4*>(na.h_out + r * K + col);
                    hp[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    hp[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
            // Eq. 3: sigma_b = Pi_E4M3(amax_b / (alpha * q_max))
            const float amax = bf16x16_absmax(w);
            uint32_t sc = e4m3_block_scale(amax, qc.alpha_qmax, qc.inv_lo, qc.inv_hi);
            // Eq. 2: q_i = Pi_FP4(x_i / (alpha * sigma_b)), as x * fl(1/fl(alpha*sigma))
            const float enc = enc_tab[sc];
            float f0[8], f1[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                f0[2 * j] = bf16_lo(w[j]);
                f0[2 * j + 1] = bf16_hi(w[j]);
                f1[2 * j] = bf16_lo(w[4 + j]);
                f1[2 * j + 1] = bf16_hi(w[4 + j]);
            }
            uint32_t c0 = e2m1x8_encode(f0, enc);
            uint32_t c1 = e2m1x8_encode(f1, enc);
            if (SEARCH) {
                float best = block_sq_error(f0, f1, c0, c1, dec_tab[sc]);
                const uint32_t base = sc;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (t == 0 ? base < 1u : base > 0x7Du) continue;
                    const uint32_t cand = t == 0 ? base - 1u : base + 1u;
                    const float ec = enc_tab[cand];
                    const uint32_t q0 = e2m1x8_encode(f0, ec);
                    const uint32_t q1 = e2m1x8_encode(f1, ec);
                    const float err = block_sq_error(f0, f1, q0, q1, dec_tab[cand]);
                    if (err < best) {
                        best = err;
                        sc = cand;
                        c0 = q0;
                        c1 = q1;
                    }
                }
            }
            const bool ok = (r < rows) && col_ok;
            if (ok) *reinterpret_cast<uint2*>(codes + r * (K / 2) + col / 2) = make_uint2(c0, c1);
            sf_stage[(blk >> 2) * 512 + (rl & 31) * 16 + (rl >> 5) * 4 + (blk & 3)] = ok ? (uint8_t)sc : 0;
        }
    }
    __syncthreads();
    if (threadIdx.x < 128) {
        uint4* dst = reinterpret_cast<uint4*>(scales + (rb * chunks + kc) * 2048);
        dst[threadIdx.x] = reinterpret_cast<const uint4*>(sf_stage)[threadIdx.x];
    }
    __syncthreads();
}


// Lean variant of quant_tile for tiles inside the tensor on both axes (see the
// LEAN parameter of quantize_kernel for where it runs): the pass is bound by
// instruction issue, and this loop has no per-block bounds checks or zeroing,
// and the thread's 8 rows are 2 apart in the tile and, with the gate/up
// interleave too, 2 apart in the source (a warp's 16 rows map onto 16
// consecutive source rows), so its load, code and staging addresses advance
// by constant steps.  quant_block_store is one block's Eq. 3 / Eq. 2 (h formed
// first with NORM: rstd rs, gamma at gp), codes stored at cp, scale code at sp.
template <bool SEARCH, bool NORM>
__device__ __forceinline__ void quant_block_store(uint32_t (&w)[8], bool ok, float rs, const uint16_t* gp,
                                                  uint16_t* hp, uint2* cp, uint8_t* sp, const QuantConsts& qc,
                                                  const float* enc_tab, const float* dec_tab)
{
    if (NORM && ok) {
        const uint4 g0 = __ldg(reinterpret_cast<const uint4*>(gp));
        const uint4 g1 = __ldg(reinterpret_cast<const uint4*>(gp) + 1);
        const uint32_t g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = norm_pair(w[j], g[j], rs);
        if (hp != nullptr) {
            reinterpret_cast<uint4*>(hp)[0] = make_uint4(w[0], w[1], w[2], w[3]);
            reinterpret_cast<uint4*>(hp)[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
    const float amax = bf16x16_absmax(w);
    uint32_t sc = e4m3_block_scale(amax, qc.alpha_qmax, qc.inv_lo, qc.inv_hi);
    const float enc = enc_tab[sc];
    float f0[8], f1[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        f0[2 * j] = bf16_lo(w[j]);
        f0[2 * j + 1] = bf16_hi(w[j]);
        f1[2 * j] = bf16_lo(w[4 + j]);
        f1[2 * j + 1] = bf16_hi(w[4 + j]);
    }
    uint32_t c0 = e2m1x8_encode(f0, enc);
    uint32_t c1 = e2m1x8_encode(f1, enc);
    if (SEARCH) {
        float best = block_sq_error(f0, f1, c0, c1, dec_tab[sc]);
        const uint32_t base = sc;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (t == 0 ? base < 1u : base > 0x7Du) continue;
            const uint32_t cand = t == 0 ? base - 1u : base + 1u;
            const float ec = enc_tab[cand];
            const uint32_t q0 = e2m1x8_encode(f0, ec);
            const uint32_t q1 = e2m1x8_encode(f1, ec);
            const float err = block_sq_error(f0, f1, q0, q1, dec_tab[cand]);
            if (err < best) {
                best = err;
                sc = cand;
                c0 = q0;
                c1 = q1;
            }
        }
    }
    if (ok) *cp = make_uint2(c0, c1);
    *sp = ok ? (uint8_t)sc : (uint8_t)0;
}

template <bool SEARCH, bool NORM>
__device__ __forceinline__ void quant_tile_lean(const uint16_t* __restrict__ x, int64_t K, int64_t interleave_half,
                                                int64_t rb, int64_t kc, int64_t chunks, const QuantConsts& qc,
                                                const float* enc_tab, const float* dec_tab, uint8_t* sf_stage,
                                                uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int warp,
                                                int half, int blk, const NormArgs& na)
{
    const int64_t col = kc * 256 + 16 * blk;
    const uint16_t* gp = NORM ? na.gamma + col : nullptr;
    const int rl0 = 16 * warp + half;    // the thread's first row in the tile; then every second one
    const int64_t r0 = rb * 128 + rl0;
    const uint16_t* xp = x + quant_src_row(r0, interleave_half) * K + col;
    uint8_t* cp = codes + r0 * (K / 2) + col / 2;
    uint16_t* hp = (NORM && na.h_out != nullptr) ? na.h_out + r0 * K + col : nullptr;
    // staging byte of (row rl0 + 2 st, block blk): (rl % 32) * 16 + (rl / 32) * 4 in the atom of
    // blk / 4, byte blk % 4, so 32 bytes on per step
    uint8_t* sp0 = sf_stage + (blk >> 2) * 512 + (rl0 & 31) * 16 + (rl0 >> 5) * 4 + (blk & 3);
#pragma unroll 1
    for (int s0 = 0; s0 < 8; s0 += kQuantStepUnroll) {
        uint4 v[kQuantStepUnroll][2];
#pragma unroll
        for (int u = 0; u < kQuantStepUnroll; ++u) {
            const uint4* p = reinterpret_cast<const uint4*>(xp + (int64_t)(2 * (s0 + u)) * K);
            v[u][0] = __ldcs(p);
            v[u][1] = __ldcs(p + 1);
        }
#pragma unroll
        for (int u = 0; u < kQuantStepUnroll; ++u) {
            const int st = s0 + u;
            uint32_t w[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w, v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
            const float rs = NORM ? __ldg(na.rstd + r0 + 2 * st) : 0.0f;
            quant_block_store<SEARCH, NORM>(w, true, rs, gp, hp != nullptr ? hp + (int64_t)(2 * st) * K : nullptr,
                                            reinterpret_cast<uint2*>(cp + (int64_t)st * K), sp0 + 32 * st, qc, enc_tab,
                                            dec_tab);
        }
    }
    __syncthreads();
    if (threadIdx.x < 128) {
        uint4* dst = reinterpret_cast<uint4*>(scales + (rb * chunks + kc) * 2048);
        dst[threadIdx.x] = reinterpret_cast<const uint4*>(sf_stage)[threadIdx.x];
    }
    __syncthreads();
}


__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Quantization of X [rows, K] in one launch.  Tiles of 128 rows x 256
// columns are dealt to the blocks round robin.
//   * alpha_static != nullptr: Eq. 2 / Eq. 3 with that tensor scale.
//   * otherwise (launched cooperatively, every block resident): the blocks
//     first take the |x| maximum of their tiles; the last block to finish
//     folds the per-block maxima into alpha = amax / (q_max * 448) (1 for an
//     all-zero tensor), stores it at alpha_out and publishes it with a
//     release store of a new epoch number, which the other blocks wait for
//     (bounded; a wait that runs out posts kErrTimeout and the block stops).
//     The quantization pass then walks the tiles in the opposite order, so
//     the lines read last by the amax pass, still in L2, are read first.
// LEAN: 0 the regular tile loop; 1 the lean tile loop for tiles inside the
// tensor and the regular one for its edge tiles, three blocks per SM (the two
// loops together need more than 64 registers); 2 the lean loop alone, for
// tensors whose sizes are multiples of 128 x 256, at four blocks per SM (three
// with NORM).
template <bool SEARCH, bool NORM, bool CLUSTER = false, int LEAN = 0>
__global__ void __launch_bounds__(kQuantThreads, (LEAN == 1 || NORM) ? MQ_QUANT_MIN_BLOCKS - 1 : MQ_QUANT_MIN_BLOCKS)
    quantize_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K, const float* __restrict__ alpha_static,
                    float* __restrict__ alpha_out, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                    int64_t interleave_half, WsControl* ctrl, uint32_t* __restrict__ partials, NormArgs na)
{
    __shared__ __align__(16) uint8_t sf_stage[2048];
    __shared__ float enc_tab[128];
    __shared__ float dec_tab[128];   // fl(alpha * sigma) for every E4M3 code sigma
    __shared__ uint32_t s_red[kQuantThreads / 32];
    __shared__ uint32_t s_epoch, s_last, s_ok;
    __shared__ uint32_t s_slot[CLUSTER ? 16 : 1];   // cluster hand-off: one maximum per CTA
    __shared__ float s_alpha;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4;
    const int blk = lane & 15;
    const int64_t chunks = (K + 255) / 256;
    const int64_t tiles = ((rows + 127) / 128) * chunks;
    // X, the tensor scale and the outputs may be touched by the previous kernel
    // of the stream; a consumer launched with programmatic serialization (the
    // uniform-NVFP4 decode, the GEMM) may start now and waits for this grid
    // before it reads what this kernel writes
    grid_dep_wait();
    grid_dep_launch_dependents();

    float alpha;
    if (alpha_static != nullptr) {
        alpha = *alpha_static;
    } else if (CLUSTER) {
        // The whole grid is one thread-block cluster: each CTA's maximum goes
        // straight into a slot of every CTA's shared memory and two cluster
        // barriers replace the global ticket, fold and spin.
        const int cluster = (int)gridDim.x;
        const uint32_t rank = cluster_ctarank();
        cluster_barrier();   // every CTA runs before its shared memory is written remotely
        uint32_t mx = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x)
            mx = amax_tile(x, rows, K, interleave_half, t / chunks, t % chunks, warp, half, blk, mx);
        uint32_t m = max(mx & 0xFFFFu, mx >> 16);
        if (m >= 0x7F80u) {
            uint32_t bad = 0;
            mx = 0;
            for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x)
                mx = amax_tile_finite(x, rows, K, interleave_half, t / chunks, t % chunks, warp, half, blk, mx, bad);
            m = max(mx & 0xFFFFu, mx >> 16) | (bad ? 0x80000000u : 0u);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fold_max_flag(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) s_red[warp] = m;
        __syncthreads();
        if (threadIdx.x < cluster) {
            uint32_t b = 0;
            for (int w = 0; w < kQuantThreads / 32; ++w) b = fold_max_flag(b, s_red[w]);
            st_cluster_u32(map_to_cta(smem_u32(&s_slot[rank]), (uint32_t)threadIdx.x), b);
        }
        cluster_barrier();   // release / acquire: every CTA's slot is written
        uint32_t r = 0;
        for (int q = 0; q < cluster; ++q) r = fold_max_flag(r, s_slot[q]);
        const float amax = __uint_as_float((r & 0x7FFFu) << 16);
        alpha = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
        if (rank == 0 && threadIdx.x == 0) {
            *alpha_out = alpha;
            if (r & 0x80000000u) post_error(ctrl, kErrNonFinite);
        }
    } else {
        uint32_t* epoch = &ctrl->epoch;
        // the epoch before this pass (a relaxed read: it cannot see this pass's
        // publication, which follows every block's ticket, and it does not hold
        // back the loads below)
        if (threadIdx.x == 0) s_epoch = ld_relaxed_gpu_u32(epoch);
        // ---- pass 1: |x| maximum of this block's tiles
        uint32_t mx = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x)
            mx = amax_tile(x, rows, K, interleave_half, t / chunks, t % chunks, warp, half, blk, mx);
        uint32_t m = max(mx & 0xFFFFu, mx >> 16);
        if (m >= 0x7F80u) {
            // a NaN/Inf in this thread's share: its finite maximum, and the flag
            uint32_t bad = 0;
            mx = 0;
            for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x)
                mx = amax_tile_finite(x, rows, K, interleave_half, t / chunks, t % chunks, warp, half, blk, mx, bad);
            m = max(mx & 0xFFFFu, mx >> 16) | (bad ? 0x80000000u : 0u);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fold_max_flag(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) s_red[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t b = 0;
            for (int w = 0; w < kQuantThreads / 32; ++w) b = fold_max_flag(b, s_red[w]);
            partials[blockIdx.x] = b;
            const uint32_t ticket = atom_add_acq_rel_gpu(&ctrl->amax_ticket, 1u);   // releases the partial
            s_last = (ticket == gridDim.x - 1);
        }
        __syncthreads();
        if (s_last) {
            // every block's maximum is in `partials` (visible after the ticket's
            // acquire and the barrier): fold them, publish alpha
            uint32_t b = 0;
            for (int j = threadIdx.x; j < (int)gridDim.x; j += blockDim.x) b = fold_max_flag(b, __ldcg(partials + j));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) b = fold_max_flag(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
            __syncthreads();
            if (lane == 0) s_red[warp] = b;
            __syncthreads();
            if (threadIdx.x == 0) {
                uint32_t r = 0;
                for (int w = 0; w < kQuantThreads / 32; ++w) r = fold_max_flag(r, s_red[w]);
                const float amax = __uint_as_float((r & 0x7FFFu) << 16);
                *alpha_out = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
                if (r & 0x80000000u) post_error(ctrl, kErrNonFinite);
                ctrl->amax_ticket = 0;   // ready for the next pass on this workspace
                st_release_u32(epoch, s_epoch + 1u);   // orders alpha and the reset before it
            }
        }
        // ---- every block: wait for the published alpha
        if (threadIdx.x == 0) {
            bool ok = ld_acquire_u32(epoch) != s_epoch;
            if (!ok) {
                const uint64_t t0 = globaltimer_ns();
                while (!(ok = (ld_acquire_u32(epoch) != s_epoch))) {
                    if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
                    __nanosleep(64);
                }
            }
            s_ok = ok;
            s_alpha = ok ? __ldcg(alpha_out) : 0.0f;
            if (!ok) post_error(ctrl, kErrTimeout);
        }
        __syncthreads();
        if (!s_ok) return;
        alpha = s_alpha;
    }
    const QuantConsts qc = quant_setup(alpha, enc_tab, dec_tab);
    // ---- pass 2: quantize, tiles in reverse order of pass 1
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t tile = tiles - 1 - t;
        const int64_t rb = tile / chunks, kc = tile % chunks;
        if (LEAN == 2 || (LEAN == 1 && (rb + 1) * 128 <= rows && (kc + 1) * 256 <= K))
            quant_tile_lean<SEARCH, NORM>(x, K, interleave_half, rb, kc, chunks, qc, enc_tab, dec_tab, sf_stage, codes,
                                          scales, warp, half, blk, na);
        else
            quant_tile<SEARCH, NORM>(x, rows, K, interleave_half, rb, kc, chunks, qc, enc_tab, dec_tab, sf_stage,
                                     codes, scales, warp, half, blk, na);
    }
}

// Resident blocks per SM of quantize_kernel<SEARCH, NORM, false, LEAN> (cached per device).
template <bool SEARCH, bool NORM, int LEAN = 0>
int quantize_blocks_per_sm(const DeviceInfo& di)
{
    static std::mutex mu;
    static int per_sm[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (di.device >= 0 && di.device < 64 && per_sm[di.device] > 0) return per_sm[di.device];
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_kernel<SEARCH, NORM, false, LEAN>, kQuantThreads,
                                                      0) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        occ = 0;
    }
    if (di.device >= 0 && di.device < 64 && occ > 0) per_sm[di.device] = occ;
    return occ;
}

// Whether `kern` can run as one cluster of `cl` CTAs of kQuantThreads (cached
// per device, kernel and size; sizes above 8 are non-portable and opted into).
template <bool SEARCH>
bool quantize_cluster_fits(int cl, const DeviceInfo& di)
{
    static std::mutex mu;
    static std::map<std::pair<int, int>, bool> cache;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(di.device, cl);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    auto kern = quantize_kernel<SEARCH, false, true>;
    bool ok = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    if (ok) {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)cl, 1, 1);
        cfg.blockDim = dim3(kQuantThreads, 1, 1);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cl;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        ok = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters >= 1;
    }
    (void)cudaGetLastError();
    cache[key] = ok;
    return ok;
}

cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, const float* alpha_static, float* alpha_out,
                            uint8_t* codes, uint8_t* scales, int64_t interleave_half, WsControl* ctrl,
                            uint32_t* partials, const DeviceInfo& di, cudaStream_t s, bool scale_search)
{
    const int64_t tiles = ((rows + 127) / 128) * ((K + 255) / 256);
    const int occ = scale_search ? quantize_blocks_per_sm<true, false>(di) : quantize_blocks_per_sm<false, false>(di);
    const int64_t resident = (int64_t)di.num_sms * std::max(1, occ);
    // Small tensors (at most one tile per SM): one launch takes the amax,
    // hands alpha to every block and quantizes; the two-kernel path would pay
    // a second launch and its ramp for a few microseconds of work.  Up to 16
    // tiles the grid is one thread-block cluster whose CTAs exchange their
    // maxima through distributed shared memory; otherwise a cooperative launch
    // hands alpha over through global memory.  Larger tensors: the amax kernel
    // (full occupancy) and then the quantization kernel with that alpha.
    const bool single = (alpha_static == nullptr) && tiles <= di.num_sms && occ > 0;
    const int cl = (single && tiles <= 16 &&
                    (scale_search ? quantize_cluster_fits<true>((int)tiles, di)
                                  : quantize_cluster_fits<false>((int)tiles, di)))
                       ? (int)tiles
                       : 0;
    const float* alpha_in = alpha_static;
    if (alpha_static == nullptr && !single) {
        cudaError_t e = launch_amax(x, rows * K, alpha_out, ctrl, partials, di, s);
        if (e != cudaSuccess) return e;
        alpha_in = alpha_out;
    }
    // The lean tile loop skips the per-block bounds checks of tiles inside the
    // tensor.  From kQuantLeanTiles tiles (several waves) at three blocks per SM
    // with the regular loop for edge tiles (8192 x 12288: 84.8 -> 75 us for amax
    // + quantization); below that, for sizes that are multiples of 128 x 256,
    // alone at four blocks per SM (8192 x 4096: 35.6 -> 33.9 us).
    const bool aligned = rows % 128 == 0 && K % 256 == 0;
    const int lean = (scale_search || single) ? 0 : tiles >= kQuantLeanTiles ? 1 : aligned ? 2 : 0;
    const int64_t res =
        lean == 1   ? (int64_t)di.num_sms * std::max(1, quantize_blocks_per_sm<false, false, 1>(di))
        : lean == 2 ? (int64_t)di.num_sms * std::max(1, quantize_blocks_per_sm<false, false, 2>(di))
                    : resident;
    int64_t blocks = std::min(tiles, res);
    if (blocks > kAmaxMaxBlocks) blocks = kAmaxMaxBlocks;
    if (blocks < 1) blocks = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(kQuantThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    cfg.attrs = attr;
    if (cl > 0) {   // one cluster (the grid is `tiles` CTAs); may overlap its predecessor's tail
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cl;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 2;
    } else if (single) {   // blocks wait on one another only in the single-launch amax
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.numAttrs = 1;
    } else {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 1;
    }
    auto kern = cl > 0 ? (scale_search ? quantize_kernel<true, false, true> : quantize_kernel<false, false, true>)
                : lean == 1 ? quantize_kernel<false, false, false, 1>
                : lean == 2 ? quantize_kernel<false, false, false, 2>
                       : (scale_search ? quantize_kernel<true, false> : quantize_kernel<false, false>);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<const uint16_t*>(x), rows, K, alpha_in, alpha_out,
                                       codes, scales, interleave_half, ctrl, partials, NormArgs{});
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ==========================================================================
// RMSNorm fused with the quantization of its output
// ==========================================================================
//
// Pass 1 (this kernel): one warp per row computes ms = fl32(sum x^2 / K) with
// the sum in binary64, rstd = fl32(1 / sqrt(ms + eps)) (binary64, one
// rounding), stores rstd and takes the |h| maximum of the row's
// h = bf16(fl(fl(x * rstd) * gamma)); the last block folds the per-block
// maxima into alpha_h = amax/2688 (1 if 0; NaN/Inf excluded and reported).
// Pass 2 is quantize_kernel with NORM (launch_norm_quantize), which forms h again on load.
constexpr int kNormThreads = 256;
constexpr int64_t kNormGammaSmem = 8192;   // gamma elements staged in shared memory (16 KiB)

// End of an RMSNorm first pass: folds the threads' |h| maxima (BF16
// magnitudes, two per word in mx) and non-finite flags into one word per
// block (bit 31 = flag), publishes it in partials[block], and the block that
// takes the last ticket folds every block's word into
// alpha_h = amax / 2688 (1 if the maximum is 0) and posts kErrNonFinite if
// any block saw a NaN/Inf.  Every thread of the block calls it.
template <int WARPS>
__device__ __forceinline__ void norm_alpha_publish(uint32_t mx, uint32_t bad, float* __restrict__ alpha_out,
                                                   WsControl* ctrl, uint32_t* __restrict__ partials)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t m = max(mx & 0xFFFFu, mx >> 16) | (bad ? 0x80000000u : 0u);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fold_max_flag(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ uint32_t s_red[WARPS];
    __shared__ bool is_last;
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < WARPS; ++w) b = fold_max_flag(b, s_red[w]);
        partials[blockIdx.x] = b;
        is_last = (atom_add_acq_rel_gpu(&ctrl->amax_ticket, 1u) == gridDim.x - 1);   // releases the partial
    }
    __syncthreads();
    if (!is_last) return;
    // the last block folds every block's maximum, all threads at once
    uint32_t b = 0;
    for (int j = threadIdx.x; j < (int)gridDim.x; j += WARPS * 32) b = fold_max_flag(b, __ldcg(partials + j));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) b = fold_max_flag(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
    __syncthreads();
    if (lane == 0) s_red[warp] = b;
    __syncthreads();
    if (threadIdx.x == 0) {
        b = 0;
        for (int w = 0; w < WARPS; ++w) b = fold_max_flag(b, s_red[w]);
        const float amax = __uint_as_float((b & 0x7FFFu) << 16);
        *alpha_out = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
        if (b & 0x80000000u) post_error(ctrl, kErrNonFinite);
        ctrl->amax_ticket = 0;   // visible at kernel end
    }
}

__global__ void __launch_bounds__(kNormThreads) rmsnorm_amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                                    int64_t K, const uint16_t* __restrict__ gamma,
                                                                    float eps, float* __restrict__ rstd,
                                                                    float* __restrict__ alpha_out, WsControl* ctrl,
                                                                    uint32_t* __restrict__ partials)
{
    grid_dep_wait();   // X may be the previous kernel's output
    grid_dep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t wstride = (int64_t)gridDim.x * (kNormThreads / 32);
    uint32_t mx = 0, bad = 0;
    // A row is read in chunks of kNormChunk 16-byte vectors per lane, all in
    // flight at once; a row of at most one chunk (K <= 4096) stays in
    // registers for the |h| pass, longer rows are read again (from L2).
    constexpr int kNormChunk = 16;
    const int64_t nv = K / 8;
    const int64_t chunk = 32 * kNormChunk;
    // gamma, read by every row, staged once per block in shared memory when it
    // fits (K <= kNormGammaSmem elements)
    extern __shared__ uint4 s_gamma[];
    const bool g_smem = K <= kNormGammaSmem;
    if (g_smem)
        for (int64_t i = threadIdx.x; i < nv; i += kNormThreads) s_gamma[i] = __ldg(reinterpret_cast<const uint4*>(gamma) + i);
    __syncthreads();
    const uint4* gr = g_smem ? s_gamma : reinterpret_cast<const uint4*>(gamma);
    // Each warp takes rows r, r + wstride, ...; while it works on one row, the
    // next one is prefetched into L2 with one bulk prefetch.
    for (int64_t r = (int64_t)blockIdx.x * (kNormThreads / 32) + warp; r < rows; r += wstride) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + r * K);
        if (lane == 0 && r + wstride < rows)
            bulk_prefetch_l2(x + (r + wstride) * K, (uint32_t)std::min<int64_t>(K * 2, (int64_t)1 << 20));
        uint4 v[kNormChunk];
        // sum of squares in binary64: x widened exactly, x * x exact (16
        // significant bits, every BF16 value incl. subnormals and |x| >= 2^64)
        // and added with one rounding by the fused multiply-add, as in the
        // definition; four running sums per lane, then a butterfly over the
        // warp: the definition's sum up to the order of the additions, which
        // moves ms only when the sum lies within ~2^-40 relative of an FP32
        // rounding boundary.
        double s[4] = {0.0, 0.0, 0.0, 0.0};   // four independent chains
        for (int64_t c0 = 0; c0 < nv; c0 += chunk) {
#pragma unroll
            for (int u = 0; u < kNormChunk; ++u) {
                const int64_t i = c0 + lane + 32 * u;
                v[u] = (i < nv) ? __ldg(xr + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kNormChunk; ++u) {
                const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const double a = (double)bf16_lo(w[j]), b = (double)bf16_hi(w[j]);
                    s[(j & 1) * 2] = __fma_rn(a, a, s[(j & 1) * 2]);
                    s[(j & 1) * 2 + 1] = __fma_rn(b, b, s[(j & 1) * 2 + 1]);
                }
            }
        }
        double ss = __dadd_rn(__dadd_rn(s[0], s[1]), __dadd_rn(s[2], s[3]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
        const float ms = __double2float_rn(__ddiv_rn(ss, (double)K));
        const float rs = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn((double)ms, (double)eps))));
        if (lane == 0) rstd[r] = rs;
        // |h| maximum of the row over all values (two instructions per pair);
        // a NaN or Inf among them (magnitude bits 0x7F80 and above, rare) sends
        // the row through the finite-only fold, which also raises the flag
        uint32_t mrow = 0;
        for (int64_t c0 = 0; c0 < nv; c0 += chunk) {
            if (nv > chunk) {   // the chunk is no longer in registers
#pragma unroll
                for (int u = 0; u < kNormChunk; ++u) {
                    const int64_t i = c0 + lane + 32 * u;
                    v[u] = (i < nv) ? __ldg(xr + i) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < kNormChunk; ++u) {
                const int64_t i = c0 + lane + 32 * u;
                if (i < nv) {
                    const uint4 g = g_smem ? gr[i] : __ldg(gr + i);
                    mrow = max_u16x2(mrow, norm_pair(v[u].x, g.x, rs) & 0x7FFF7FFFu);
                    mrow = max_u16x2(mrow, norm_pair(v[u].y, g.y, rs) & 0x7FFF7FFFu);
                    mrow = max_u16x2(mrow, norm_pair(v[u].z, g.z, rs) & 0x7FFF7FFFu);
                    mrow = max_u16x2(mrow, norm_pair(v[u].w, g.w, rs) & 0x7FFF7FFFu);
                }
            }
        }
        if (__any_sync(0xFFFFFFFFu, max(mrow & 0xFFFFu, mrow >> 16) >= 0x7F80u)) {
            mrow = 0;
            for (int64_t i = lane; i < nv; i += 32) {
                const uint4 xv = __ldg(xr + i);
                const uint4 g = g_smem ? gr[i] : __ldg(gr + i);
                amax_accum(norm_pair(xv.x, g.x, rs), mrow, bad);
                amax_accum(norm_pair(xv.y, g.y, rs), mrow, bad);
                amax_accum(norm_pair(xv.z, g.z, rs), mrow, bad);
                amax_accum(norm_pair(xv.w, g.w, rs), mrow, bad);
            }
        }
        mx = max_u16x2(mx, mrow);
    }
    norm_alpha_publish<kNormThreads / 32>(mx, bad, alpha_out, ctrl, partials);
}

// Pass 1 with two warps per row, for rows of at most kNormPairMaxK elements:
// warp 2p + g of the block takes half g of each of its rows (16-byte vectors
// [g nh, (g + 1) nh), nh = K / 16), so the grid holds twice as many rows in
// flight as with one warp per row, with half the registers per warp.  The
// two warps add their binary64 partial sums in a fixed order (half 0 +
// half 1) through shared memory (double-buffered by row parity, one named
// barrier per row), so both derive the same rstd; each then takes the |h|
// maximum of its half.  Arithmetic otherwise as rmsnorm_amax_kernel.
constexpr int64_t kNormPairMaxK = 4096;
constexpr int kNormPairChunk = 8;   // 16-byte vectors per lane: half a row of 4096
static_assert(kNormThreads == 256, "four warp pairs per block: named barriers 1-4");
#ifndef MQ_NORM_PAIR_MIN_BLOCKS
#define MQ_NORM_PAIR_MIN_BLOCKS 3
#endif

__global__ void __launch_bounds__(kNormThreads, MQ_NORM_PAIR_MIN_BLOCKS) rmsnorm_amax_pair_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t K, const uint16_t* __restrict__ gamma, float eps,
    float* __restrict__ rstd, float* __restrict__ alpha_out, WsControl* ctrl, uint32_t* __restrict__ partials)
{
    grid_dep_wait();   // X may be the previous kernel's output
    grid_dep_launch_dependents();
    constexpr int kPairs = kNormThreads / 64;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = warp & 1, pr = warp >> 1;
    const int64_t pstride = (int64_t)gridDim.x * kPairs;
    const int64_t nv = K / 8, nh = nv / 2;
    extern __shared__ uint4 s_gamma[];
    __shared__ double s_part[2][kNormThreads / 32];
    for (int64_t i = threadIdx.x; i < nv; i += kNormThreads) s_gamma[i] = __ldg(reinterpret_cast<const uint4*>(gamma) + i);
    __syncthreads();
    const uint4* gh = s_gamma + g * nh;
    uint32_t mx = 0, bad = 0;
    int par = 0;
    for (int64_t r = (int64_t)blockIdx.x * kPairs + pr; r < rows; r += pstride, par ^= 1) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + r * K) + g * nh;
        if (lane == 0 && r + pstride < rows)
            bulk_prefetch_l2(reinterpret_cast<const uint4*>(x + (r + pstride) * K) + g * nh, (uint32_t)K);
        uint4 v[kNormPairChunk];
#pragma unroll
        for (int u = 0; u < kNormPairChunk; ++u) {
            const int64_t i = lane + 32 * u;
            v[u] = (i < nh) ? __ldg(xr + i) : make_uint4(0u, 0u, 0u, 0u);
        }
        // binary64 sum of the half's exact squares (four chains, then the warp)
        double s[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int u = 0; u < kNormPairChunk; ++u) {
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const double a = (double)bf16_lo(w[j]), b = (double)bf16_hi(w[j]);
                s[(j & 1) * 2] = __fma_rn(a, a, s[(j & 1) * 2]);
                s[(j & 1) * 2 + 1] = __fma_rn(b, b, s[(j & 1) * 2 + 1]);
            }
        }
        double sp = __dadd_rn(__dadd_rn(s[0], s[1]), __dadd_rn(s[2], s[3]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sp = __dadd_rn(sp, __shfl_xor_sync(0xFFFFFFFFu, sp, o));
        if (lane == 0) s_part[par][warp] = sp;
        // the pair's barrier (ids 1-4; literal ids keep the block's barrier count at five)
        switch (pr) {
            case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
            case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
            case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
            default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
        }
        const double ss = __dadd_rn(s_part[par][2 * pr], s_part[par][2 * pr + 1]);
        const float ms = __double2float_rn(__ddiv_rn(ss, (double)K));
        const float rs = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn((double)ms, (double)eps))));
        if (g == 0 && lane == 0) rstd[r] = rs;
        // |h| maximum of the half (two running maxima); NaN/Inf halves take the finite-only fold
        uint32_t m2[2] = {0u, 0u};
#pragma unroll
        for (int u = 0; u < kNormPairChunk; ++u) {
            const int64_t i = lane + 32 * u;
            if (i < nh) {
                const uint4 gv = gh[i];
                m2[0] = max_u16x2(m2[0], norm_pair(v[u].x, gv.x, rs) & 0x7FFF7FFFu);
                m2[1] = max_u16x2(m2[1], norm_pair(v[u].y, gv.y, rs) & 0x7FFF7FFFu);
                m2[0] = max_u16x2(m2[0], norm_pair(v[u].z, gv.z, rs) & 0x7FFF7FFFu);
                m2[1] = max_u16x2(m2[1], norm_pair(v[u].w, gv.w, rs) & 0x7FFF7FFFu);
            }
        }
        uint32_t mrow = max_u16x2(m2[0], m2[1]);
        if (__any_sync(0xFFFFFFFFu, max(mrow & 0xFFFFu, mrow >> 16) >= 0x7F80u)) {
            mrow = 0;
            for (int64_t i = lane; i < nh; i += 32) {
                const uint4 xv = __ldg(xr + i), gv = gh[i];
                amax_accum(norm_pair(xv.x, gv.x, rs), mrow, bad);
                amax_accum(norm_pair(xv.y, gv.y, rs), mrow, bad);
                amax_accum(norm_pair(xv.z, gv.z, rs), mrow, bad);
                amax_accum(norm_pair(xv.w, gv.w, rs), mrow, bad);
            }
        }
        mx = max_u16x2(mx, mrow);
    }
    norm_alpha_publish<kNormThreads / 32>(mx, bad, alpha_out, ctrl, partials);
}

// Pass 2: quantize_kernel with NORM forms h again on load and encodes it
// with the alpha_h of pass 1.
static cudaError_t launch_norm_quantize(const void* x, int64_t rows, int64_t K, const void* gamma, float* rstd,
                                        uint8_t* codes, uint8_t* scales, float* alpha_out, void* h_out,
                                        WsControl* ctrl, uint32_t* partials, const DeviceInfo& di, cudaStream_t s)
{
    const int64_t tiles = ((rows + 127) / 128) * ((K + 255) / 256);
    // sizes that are multiples of 128 x 256: the lean tile loop alone (three
    // blocks per SM, as every NORM instantiation; 8192 x 4096: 54.5 -> 51.6 us
    // for the fused pair)
    const bool aligned = rows % 128 == 0 && K % 256 == 0;
    const int occ = aligned ? quantize_blocks_per_sm<false, true, 2>(di) : quantize_blocks_per_sm<false, true>(di);
    int64_t qb = std::min(tiles, (int64_t)di.num_sms * std::max(1, occ));
    qb = std::max<int64_t>(qb, 1);
    NormArgs na{static_cast<const uint16_t*>(gamma), rstd, static_cast<uint16_t*>(h_out)};
    return launch_pdl(aligned ? quantize_kernel<false, true, false, 2> : quantize_kernel<false, true>, dim3((unsigned)qb),
                      dim3(kQuantThreads), 0, s,
                      static_cast<const uint16_t*>(x), rows, K, static_cast<const float*>(alpha_out), alpha_out,
                      codes, scales, (int64_t)0, ctrl, partials, na);
}

cudaError_t launch_rmsnorm_quantize(const void* x, int64_t rows, int64_t K, const void* gamma, float eps,
                                    float* rstd, uint8_t* codes, uint8_t* scales, float* alpha_out, void* h_out,
                                    WsControl* ctrl, uint32_t* partials, const DeviceInfo& di, cudaStream_t s)
{
    if (K <= kNormPairMaxK) {
        // two warps per row; one wave of resident blocks
        const size_t smem = (size_t)K * 2;
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rmsnorm_amax_pair_kernel, kNormThreads, smem) !=
            cudaSuccess) {
            (void)cudaGetLastError();
            per_sm = 1;
        }
        constexpr int kPairs = kNormThreads / 64;
        int64_t blocks = (rows + kPairs - 1) / kPairs;
        blocks = std::min<int64_t>(blocks, (int64_t)di.num_sms * std::max(1, per_sm));
        blocks = std::min<int64_t>(blocks, kAmaxMaxBlocks);
        blocks = std::max<int64_t>(blocks, 1);
        cudaError_t e = launch_pdl(rmsnorm_amax_pair_kernel, dim3((unsigned)blocks), dim3(kNormThreads), smem, s,
                                   static_cast<const uint16_t*>(x), rows, K, static_cast<const uint16_t*>(gamma), eps,
                                   rstd, alpha_out, ctrl, partials);
        if (e != cudaSuccess) return e;
        return launch_norm_quantize(x, rows, K, gamma, rstd, codes, scales, alpha_out, h_out, ctrl, partials, di, s);
    }
    // one wave of resident blocks; every warp then walks several rows
    const size_t gsmem = (K <= kNormGammaSmem) ? (size_t)K * 2 : 0;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rmsnorm_amax_kernel, kNormThreads, gsmem) != cudaSuccess) {
        (void)cudaGetLastError();
        per_sm = 1;
    }
    int64_t blocks = (rows + kNormThreads / 32 - 1) / (kNormThreads / 32);
    blocks = std::min<int64_t>(blocks, (int64_t)di.num_sms * std::max(1, per_sm));
    blocks = std::min<int64_t>(blocks, kAmaxMaxBlocks);
    blocks = std::max<int64_t>(blocks, 1);
    cudaError_t e = launch_pdl(rmsnorm_amax_kernel, dim3((unsigned)blocks), dim3(kNormThreads), gsmem, s,
                               static_cast<const uint16_t*>(x), rows, K, static_cast<const uint16_t*>(gamma), eps,
                               rstd, alpha_out, ctrl, partials);
    if (e != cudaSuccess) return e;
    return launch_norm_quantize(x, rows, K, gamma, rstd, codes, scales, alpha_out, h_out, ctrl, partials, di, s);
}

__global__ void selftest_e2m1_kernel(unsigned long long* counts)
{
    const uint32_t total = 0x41000000u + 1u;
    unsigned long long bad_pos = 0, bad_neg = 0;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
        const float m = __uint_as_float(i);
        const float n = -m;
        const uint32_t hw_p = e2m1x8_cvt(m, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & 15u;
        const uint32_t hw_n = e2m1x8_cvt(n, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & 15u;
        bad_pos += (hw_p != e2m1_code(m, 1.0f));
        bad_neg += (hw_n != e2m1_code(n, 1.0f));
    }
    if (bad_pos) atomicAdd(&counts[0], bad_pos);
    if (bad_neg) atomicAdd(&counts[1], bad_neg);
}

cudaError_t launch_selftest_e2m1(unsigned long long* counts, const DeviceInfo& di, cudaStream_t s)
{
    selftest_e2m1_kernel<<<di.num_sms * 8, 256, 0, s>>>(counts);
    return cudaGetLastError();
}

// Failure-detection self-test: one warp waits, with the pipelines' own
// warp-voted bounded wait, for a phase of an mbarrier that nothing ever
// arrives on; when the wait gives up after timeout_ns the kernel posts
// kErrTimeout to the workspace control block and returns normally, so the
// context stays usable.  waited_ns receives the wall time spent waiting.
__global__ void selftest_timeout_kernel(WsControl* ctrl, uint64_t timeout_ns, unsigned long long* waited_ns)
{
    __shared__ uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    const uint64_t t0 = globaltimer_ns();
    const bool ok = warp_wait(&bar, 0, &abort_flag, timeout_ns);
    if (threadIdx.x == 0) {
        if (!ok) post_error(ctrl, kErrTimeout);
        if (waited_ns != nullptr) *waited_ns = globaltimer_ns() - t0;
    }
}

cudaError_t launch_selftest_timeout(WsControl* ctrl, uint64_t timeout_ns, unsigned long long* waited_ns,
                                    cudaStream_t s)
{
    selftest_timeout_kernel<<<1, 32, 0, s>>>(ctrl, timeout_ns, waited_ns);
    return cudaGetLastError();
}

// ==========================================================================
// Scale layout -> plain row-major [rows, K/16] (test and inspection helper)
// ==========================================================================

__global__ void unswizzle_kernel(const uint8_t* __restrict__ scales, int64_t rows, int64_t nb,
                                 int64_t atoms_per_rowblk, uint8_t* __restrict__ out)
{
    const int64_t total = rows * nb;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / nb, b = i % nb;
        out[i] = scales[sf_offset(r, b, atoms_per_rowblk)];
    }
}

cudaError_t launch_unswizzle(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* out, cudaStream_t s)
{
    const int64_t total = rows * (K / 16);
    int64_t blocks = (total + 255) / 256;
    if (blocks > 65535) blocks = 65535;
    if (blocks < 1) blocks = 1;
    unswizzle_kernel<<<(unsigned)blocks, 256, 0, s>>>(scales, rows, K / 16, sf_atoms_per_rowblk(K), out);
    return cudaGetLastError();
}

}  // namespace mq
