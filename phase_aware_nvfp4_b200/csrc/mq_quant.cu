// mq_quant.cu -- NVFP4 quantization on sm_100a: tensor amax (the tensor-level
// scale) and the block quantizer, after "Mix-Quant: Quantized Prefilling,
// Precise Decoding for Agentic LLMs", section 3.3, Eq. 2 and Eq. 3.
//
// Both kernels are HBM-bound streams: 128-bit coalesced loads, a handful of
// FP32 operations per element, no shared-memory staging of the input.
#include "mq_device.cuh"

namespace mq {

// ==========================================================================
// Tensor amax -> alpha = amax / (q_max * 448)
// ==========================================================================

#ifndef MQ_AMAX_UNROLL
#define MQ_AMAX_UNROLL 4
#endif
#ifndef MQ_AMAX_BLOCKS_PER_SM
#define MQ_AMAX_BLOCKS_PER_SM 4
#endif
constexpr int kAmaxThreads = 512;
constexpr int kAmaxUnroll = MQ_AMAX_UNROLL;

// Per-halfword |bf16| maximum over the finite values of a 32-bit word pair,
// plus a flag word that is non-zero if a NaN/Inf was seen.
__device__ __forceinline__ void amax_accum(uint32_t w, uint32_t& mx, uint32_t& bad)
{
    const uint32_t mag = w & 0x7FFF7FFFu;
    const uint32_t nonfin = __vcmpgeu2(mag, 0x7F807F80u);  // 0xFFFF per NaN/Inf halfword
    bad |= nonfin;
    mx = max_u16x2(mx, mag & ~nonfin);
}

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
        __threadfence();
        const uint32_t ticket = atomicAdd(&ctrl->amax_ticket, 1u);
        is_last = (ticket == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    // The last block to finish folds all partial maxima.
    __threadfence();
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
        ctrl->amax_ticket = 0;  // ready for the next pass on this workspace
        __threadfence();
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
    amax_kernel<<<(unsigned)blocks, kAmaxThreads, 0, s>>>(static_cast<const uint4*>(x), n_vec, alpha_out, ctrl,
                                                         partials);
    return cudaGetLastError();
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
constexpr int kQuantStepUnroll = MQ_QUANT_UNROLL;   // steps (2 rows per warp each) with loads in flight

__global__ void __launch_bounds__(kQuantThreads, MQ_QUANT_MIN_BLOCKS) quantize_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                                 int64_t K, const float* __restrict__ alpha_ptr,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint8_t* __restrict__ scales,
                                                                 int64_t interleave_half)
{
    __shared__ __align__(16) uint8_t sf_stage[2048];
    __shared__ float enc_tab[128];   // fl(1 / fl(alpha * sigma)) for every E4M3 code sigma
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4;   // which of the two rows of a step
    const int blk = lane & 15;    // 16-element block within the 256-column chunk
    const float alpha = *alpha_ptr;
    const float alpha_qmax = __fmul_rn(alpha, 6.0f);
    // 1/alpha_qmax bracketed by the floats next to fl(1/alpha_qmax) (see
    // e4m3_block_scale).  When that reciprocal is not a normal finite float
    // the bracket [0, inf] sends every block to the exact division.
    const float inv_near = __frcp_rn(alpha_qmax);
    const bool inv_normal = inv_near >= 1.17549435e-38f && inv_near < 3.0e38f;
    const float inv_lo = inv_normal ? __uint_as_float(__float_as_uint(inv_near) - 1u) : 0.0f;
    const float inv_hi = inv_normal ? __uint_as_float(__float_as_uint(inv_near) + 1u) : __int_as_float(0x7F800000);
    if (threadIdx.x < 128) {
        const float d = __fmul_rn(alpha, e4m3_to_float((uint32_t)threadIdx.x));
        enc_tab[threadIdx.x] = (d == 0.0f) ? 0.0f : __frcp_rn(d);
    }
    __syncthreads();
    const int64_t chunks = (K + 255) / 256;              // 256-column chunks per row block
    const int64_t tiles = ((rows + 127) / 128) * chunks;

    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int64_t tile = tiles - 1 - t;
        const int64_t rb = tile / chunks, kc = tile % chunks;
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
                    int64_t src = r;
                    if (interleave_half > 0) {
                        const int64_t c = r >> 5, tt = r & 31;
                        src = (tt < 16) ? (16 * c + tt) : (interleave_half + 16 * c + (tt - 16));
                    }
                    const uint4* p = reinterpret_cast<const uint4*>(x + src * K + col);
                    v[u][0] = __ldcs(p);
                    v[u][1] = __ldcs(p + 1);
                }
            }
#pragma unroll
            for (int u = 0; u < kQuantStepUnroll; ++u) {
                const int rl = 16 * warp + 2 * (s0 + u) + half;   // row within the 128-row block
                const int64_t r = rb * 128 + rl;
                const uint32_t w[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                                       v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
                // Eq. 3: sigma_b = Pi_E4M3(amax_b / (alpha * q_max))
                const float amax = bf16x16_absmax(w);
                const uint32_t sc = e4m3_block_scale(amax, alpha_qmax, inv_lo, inv_hi);
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
                const uint32_t c0 = e2m1x8_encode(f0, enc);
                const uint32_t c1 = e2m1x8_encode(f1, enc);
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
}

cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, const float* alpha, uint8_t* codes,
                            uint8_t* scales, int64_t interleave_half, const DeviceInfo& di, cudaStream_t s)
{
    const int64_t tiles = ((rows + 127) / 128) * ((K + 255) / 256);
    int64_t blocks = (int64_t)di.num_sms * (MQ_QUANT_MIN_BLOCKS > 4 ? MQ_QUANT_MIN_BLOCKS : 4);
    if (blocks > tiles) blocks = tiles;
    if (blocks < 1) blocks = 1;
    quantize_kernel<<<(unsigned)blocks, kQuantThreads, 0, s>>>(static_cast<const uint16_t*>(x), rows, K, alpha,
                                                               codes, scales, interleave_half);
    return cudaGetLastError();
}

// ==========================================================================
// Self-test of the E2M1 conversion instruction against the definition
// ==========================================================================
//
// For every FP32 bit pattern p in [0, 0x41000000] (0 .. 8.0) and its
// negative, compare the conversion instruction with the comparison-chain
// rounding of the definition (nearest E2M1 magnitude, ties to even, clip at
// 6, sign kept).  Counts mismatches into counts[0] (positive) / counts[1].

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
