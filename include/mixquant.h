/*
 * mixquant.h -- C ABI of libmixquant, the B200 (sm_100a) NVFP4 prefill linear
 * layer with its BF16 decode counterpart.
 *
 * Method: "Mix-Quant: Quantized Prefilling, Precise Decoding for Agentic
 * LLMs", section 3.3.  The prefill phase runs every linear layer as an NVFP4
 * W4A4 GEMM: weights are quantized once, activations on the fly, with
 *   Eq. 2   q_i = Pi_FP4( x_i / (alpha_x sigma_b(i)) ),  xhat_i = alpha_x sigma_b(i) q_i
 *   Eq. 3   sigma_b = Pi_E4M3( max_{i in b} |x_i| / (alpha_x q_max) ),  q_max = 6
 * over blocks b of g = 16 consecutive elements along the GEMM K dimension.
 * The decode phase keeps the BF16 weights ("Prefill-Decode Disaggregation
 * Deployment", same section).  Readings of the steps the paper leaves open:
 *   alpha  = amax(|X|) / (6 * 448) in FP32 (1 for an all-zero tensor);
 *   Pi_E4M3, Pi_FP4: round to nearest, ties to even, saturating (448, 6);
 *   the quotient of Eq. 2 is |x| * fl(1 / fl(alpha * sigma)); the sign of x
 *   is kept on a zero code.
 *
 * Conventions for every call
 *   - All pointers are DEVICE pointers owned by the caller, except where a
 *     parameter says "host".  The library allocates no memory.
 *   - Calls are asynchronous on `stream`.  Argument errors are returned
 *     synchronously before anything is launched.  Errors found on the device
 *     (a NaN/Inf in a tensor being quantized, a pipeline wait that timed out)
 *     are posted to the control block of the workspace `ws` and returned by
 *     mq_async_status().
 *   - BF16 tensors are row-major with a 16-byte aligned base.
 *   - Shapes: K (the reduction dimension) is a multiple of 64; N is a
 *     multiple of 16 (128 for the fused MLP epilogue); M >= 1; M, N and K
 *     are at most 2^30 (MQ_ERR_SHAPE beyond).
 *
 * NVFP4 tensor storage (mq_nvfp4), for a logical [rows, cols] matrix:
 *   codes   rows x cols/2 bytes, row-major; element k of a row is in byte
 *           k/2, even k in the low nibble; E2M1 code = sign bit 3 + index of
 *           the magnitude in {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *   scales  E4M3 block scales in the tcgen05 block-scaled MMA layout: for
 *           each 128-row block and each 64-column chunk, a 512-byte atom in
 *           which (row r, block kb) sits at (r%32)*16 + ((r%128)/32)*4 + kb%4;
 *           atoms are ordered K-fastest, ceil(cols/256)*4 atoms per row
 *           block; padding rows/atoms hold 0.  Size: mq_nvfp4_sizes().
 *           mq_unswizzle_scales() converts to plain row-major [rows, cols/16].
 *   alpha   one FP32 tensor scale (device).
 */
#ifndef MIXQUANT_H
#define MIXQUANT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MQ_API __attribute__((visibility("default")))
#else
#define MQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mq_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum mq_status {
    MQ_OK = 0,
    MQ_ERR_INVALID_ARG = 1, /* null pointer where one is required, bad enum */
    MQ_ERR_SHAPE = 2,       /* K % 64, N % 16 (128 with the MLP epilogue), M range */
    MQ_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
    MQ_ERR_WORKSPACE = 4,   /* workspace missing or smaller than mq_workspace_bytes() */
    MQ_ERR_NONFINITE = 5,   /* (async) NaN or Inf in a tensor that was quantized */
    MQ_ERR_TIMEOUT = 6,     /* (async) a device-side pipeline wait gave up */
    MQ_ERR_CUDA = 7,        /* a CUDA runtime/driver call failed */
    MQ_ERR_DEVICE = 8,      /* current device is not compute capability 10.0 (B200) */
    MQ_ERR_INDEX = 9        /* (async) a token position or cache slot out of range */
} mq_status;

typedef enum mq_epilogue {
    MQ_EPI_BF16 = 0,           /* Y = bf16(alpha_x alpha_w X W^T) */
    MQ_EPI_SILU_MUL_NVFP4 = 1, /* h = bf16(silu(gate) * up), stored as NVFP4 with a static alpha_h */
    MQ_EPI_SILU_MUL_BF16 = 2   /* h = bf16(silu(gate) * up), stored as BF16 (the unfused MLP path) */
} mq_epilogue;

/* An NVFP4 tensor: views of caller-owned device buffers (layout above). */
typedef struct mq_nvfp4 {
    uint8_t* codes;
    uint8_t* scales;
    float* alpha;
    int64_t rows;
    int64_t cols;
} mq_nvfp4;

/* Fixed part of every workspace: control block (error bits, counters) and
 * the amax partial maxima.  A workspace must be zero-filled once before its
 * first use; afterwards the library keeps it consistent.  Use one workspace
 * per stream (concurrent calls must not share one). */
#define MQ_WS_CONTROL_BYTES 16384

/* Human-readable name of a status code (static string). */
MQ_API const char* mq_status_string(mq_status s);

/* Library version as "major.minor.patch" (static string). */
MQ_API const char* mq_version(void);

/* Byte sizes of the codes and scales buffers of an NVFP4 [rows, cols] tensor
 * (cols a multiple of 64).  Host-only; writes through the two host pointers. */
MQ_API mq_status mq_nvfp4_sizes(int64_t rows, int64_t cols, size_t* codes_bytes, size_t* scales_bytes);

/* Workspace bytes for mq_prefill_linear / mq_quantize_activation on an
 * activation of M x K: the control block plus room for the NVFP4 copy of
 * the activation.  mq_workspace_bytes(0, 0) == MQ_WS_CONTROL_BYTES is enough
 * for calls that quantize nothing in the workspace. */
MQ_API size_t mq_workspace_bytes(int64_t M, int64_t K);

/*
 * Offline weight quantization (section 3.3: the same NVFP4 format is applied
 * to the weights, so the prefill GEMM is W4A4).  W: BF16 [N, K].  Computes
 * the tensor scale alpha_w = amax/(6*448), then Eq. 3 block scales and
 * Eq. 2 codes into `out` (out->rows == N, out->cols == K).
 * gate_up_interleave != 0 declares W as [2I, K] = [W_gate; W_up] (I = N/2,
 * I % 64 == 0) and stores the rows interleaved in groups of 16
 * (out row 32c+t = gate row 16c+t for t < 16, up row 16c+t-16 otherwise), the
 * B-operand order the MQ_EPI_SILU_MUL_NVFP4 epilogue expects.
 * ws: >= MQ_WS_CONTROL_BYTES.
 */
MQ_API mq_status mq_quantize_weight(const void* W_bf16, int64_t N, int64_t K, int gate_up_interleave,
                             const mq_nvfp4* out, void* ws, size_t ws_bytes, mq_stream_t stream);

/*
 * On-the-fly activation quantization (Eq. 2, Eq. 3).  X: BF16 [M, K].
 * alpha_static: device FP32 tensor scale to use, or NULL to compute the
 * dynamic alpha = amax(|X|)/(6*448) into out->alpha (one extra read of X).
 * ws: >= MQ_WS_CONTROL_BYTES.
 */
MQ_API mq_status mq_quantize_activation(const void* X_bf16, int64_t M, int64_t K, const float* alpha_static,
                                 const mq_nvfp4* out, void* ws, size_t ws_bytes, mq_stream_t stream);

/*
 * The NVFP4 prefill linear layer: quantize X (unless X_q is given), then the
 * block-scaled FP4 x FP4 GEMM with FP32 accumulation,
 *   acc[m, n] = sum_k (sigma q)_X[m, k] (sigma q)_W[n, k],
 * and the epilogue:
 *   MQ_EPI_BF16            Y[m, n] = bf16(acc * alpha_x * alpha_w), Y BF16 [M, N];
 *   MQ_EPI_SILU_MUL_NVFP4  W is an interleaved gate/up weight (N = 2I); with
 *                          g, u = acc * alpha_x * alpha_w of the paired gate/up
 *                          columns, h = bf16(silu(g) * u) is quantized (Eq. 2,
 *                          Eq. 3) with the static device scale *alpha_h into
 *                          H_out ([M, I]; H_out->alpha is not written).
 *                          h_debug (optional, BF16 [M, I]) also receives h.
 *   MQ_EPI_SILU_MUL_BF16   the same h, written as BF16 to Y ([M, I], 16-byte
 *                          aligned) instead of being quantized.  Passing this h
 *                          to a second mq_prefill_linear (X_bf16 = h) quantizes
 *                          it with its dynamic tensor scale amax|h|/2688: the
 *                          unfused MLP, whose alpha_h is exact for every batch
 *                          but which writes and reads h in BF16, against the
 *                          fused epilogue's static alpha_h (a scale the caller
 *                          calibrated beforehand; blocks above it clip, Eq. 2).
 * Exactly one of X_bf16 / X_q is non-NULL.  With X_bf16, the activation is
 * quantized into the workspace (ws_bytes >= mq_workspace_bytes(M, K)) with
 * alpha_x = *alpha_static, or the dynamic amax scale when alpha_static is NULL.
 * With X_q (already NVFP4, e.g. the H_out of a previous call), ws_bytes >=
 * MQ_WS_CONTROL_BYTES.
 */
MQ_API mq_status mq_prefill_linear(const void* X_bf16, const mq_nvfp4* X_q, int64_t M, const mq_nvfp4* W,
                            mq_epilogue epi, const float* alpha_static, const float* alpha_h, void* Y,
                            const mq_nvfp4* H_out, void* h_debug, void* ws, size_t ws_bytes, mq_stream_t stream);

/* Workspace bytes for mq_decode_linear and mq_decode_linear_nvfp4 on M
 * tokens and an [N, K] weight: what mq_workspace_bytes(M, K) covers (its
 * control block also holds one counter per 128 weight rows, for N up to
 * 253952) and, for M <= 16, room for the FP32 partial sums of the K
 * dimension split across up to 8 CTAs per 128 weight rows (8 * ceil(N/128) *
 * M * 512 bytes).  With it, the decode splits K across independent CTAs that
 * add their partials in a fixed order, so the weight stream covers every SM;
 * a smaller workspace (at least MQ_WS_CONTROL_BYTES, or mq_workspace_bytes(M,
 * K) for the NVFP4 decode) still works, with the K split limited to thread-
 * block clusters.  Zero-filled once, like every workspace. */
MQ_API size_t mq_decode_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * The precise decode path (section 3.3: decoding stays on the original BF16
 * weights): Y[M, N] = bf16(sum_k X[m, k] W[n, k]) with FP32 accumulation, on
 * the tensor cores (a single token: FP32 fused multiply-adds on the CUDA
 * cores).  X BF16 [M, K] with 1 <= M <= 256, W BF16 [N, K], Y BF16 [M, N].
 * ws: >= MQ_WS_CONTROL_BYTES; mq_decode_workspace_bytes(M, N, K) for the
 * fastest launch shape.
 */
MQ_API mq_status mq_decode_linear(const void* X_bf16, int64_t M, const void* W_bf16, int64_t N, int64_t K, void* Y_bf16,
                           void* ws, size_t ws_bytes, mq_stream_t stream);

/*
 * mq_prefill_linear_noalloc -- the same NVFP4 prefill linear layer (dynamic
 * or static activation scale, BF16 epilogue) for callers that cannot
 * allocate device memory and so cannot pass a workspace: for example a
 * plugin of an inference engine that owns all device memory and may not
 * allocate when it is enqueued, or a latency-critical serving loop that must
 * not call cudaMalloc (it can synchronize the whole device).  The paper has
 * no counterpart of this call; it is a deployment convenience.
 *
 * The scratch this call needs (control block + the NVFP4 copy of X) lives in
 * a static device array of MQ_NOALLOC_SCRATCH_BYTES that every GPU loading
 * the library holds until the process exits.  Arguments are those of
 * mq_prefill_linear with X_bf16 given and epi = MQ_EPI_BF16; inputs and
 * outputs are still caller-owned device buffers.
 *   - M x K activations whose NVFP4 copy does not fit the array are rejected
 *     with MQ_ERR_WORKSPACE (the limit admits e.g. M = 8192 with K = 12288).
 *   - The first call on a device sets the array up: it looks up the array's
 *     device address on that device (cudaGetSymbolAddress, which can load
 *     the library's kernels).  Make that first call before any stream
 *     capture.  A set-up that failed is not remembered: the next call
 *     tries again.
 *   - All calls share the one array, which keeps what the last call left
 *     in it.  Calls that overlap on the GPU (other streams, other host
 *     threads) race and give wrong results: serialize them.  Each call
 *     first clears, on its own stream, the one counter that must start at
 *     zero, so calls made after such an overlap are not affected by it.
 *   - Device-side errors (NaN/Inf in X, a pipeline timeout) are not reported
 *     by this call; mq_prefill_linear with a workspace reports them.
 * It calls no cudaMalloc, cudaFree or allocating library routine.
 */
#define MQ_NOALLOC_SCRATCH_BYTES (64u << 20)
MQ_API mq_status mq_prefill_linear_noalloc(const void* X_bf16, int64_t M, const mq_nvfp4* W,
                                           const float* alpha_static, void* Y_bf16, mq_stream_t stream);

/* Flags of mq_quantize. */
#define MQ_QUANT_GATE_UP_INTERLEAVE 1u  /* rows = [gate; up], interleaved in 16-row groups (as mq_quantize_weight) */
#define MQ_QUANT_SCALE_SEARCH 2u        /* per-block scale search (below) */

/* General quantization entry: BF16 [rows, K] -> NVFP4 `out` (Eq. 2, Eq. 3),
 * tensor scale dynamic (amax/2688, 1 for an all-zero tensor) unless
 * alpha_static is given (then copied to out->alpha).
 * MQ_QUANT_SCALE_SEARCH: the paper mentions "scale optimization" once without
 * defining it; read here as an opt-in per-block search: besides the Eq. 3
 * scale code c0, its E4M3 neighbours c0 - 1 and c0 + 1 are tried (each with
 * its Eq. 2 codes) and the one with the smallest squared error
 * sum_i (x_i - fl(fl(alpha*sigma) * v_i))^2, accumulated in binary32 in
 * element order, is kept; ties keep c0.  Costs about three times the
 * quantization arithmetic; meant for the offline weights.
 * MQ_QUANT_GATE_UP_INTERLEAVE needs rows % 128 == 0.  Other flag bits:
 * MQ_ERR_INVALID_ARG.  Shapes, alignment, workspace and errors as
 * mq_quantize_weight. */
MQ_API mq_status mq_quantize(const void* X_bf16, int64_t rows, int64_t K, const float* alpha_static, unsigned flags,
                             const mq_nvfp4* out, void* ws, size_t ws_bytes, mq_stream_t stream);

/* K/V projection of the prefill with its outputs in the decode precision
 * ("Prefill-Decode Disaggregation Deployment": the prefill writes the KV cache
 * in the precision the high-precision decode engine expects): one NVFP4 GEMM
 * against W_kv = [K-projection rows; V-projection rows], 2 * n_kv_heads * 128
 * rows of head dimension 128, whose epilogue
 *   - scales the FP32 sums by fl(alpha_x * alpha_w),
 *   - applies rotary position embedding to the K heads (rotate-half form:
 *     pairs i, i + 64 with c = cos_sin[pos][i], s = cos_sin[pos][64 + i]:
 *     k'_i = fl(fl(k_i c) - fl(k_{i+64} s)), k'_{i+64} = fl(fl(k_{i+64} c) +
 *     fl(k_i s)), binary32),
 *   - rounds to BF16 and writes token m's heads to k_cache[slots[m]][h][:] and
 *     v_cache[slots[m]][h][:] ([num_slots, n_kv_heads, 128] BF16 each).
 * positions: int32 [M] (4-byte aligned), slots: int64 [M] (8-byte aligned),
 * cos_sin: FP32 [max_pos, 128] (cos of the 64 frequencies, then sin; 16-byte
 * aligned), caches 16-byte aligned.  X as in mq_prefill_linear (BF16 quantized
 * on the fly with a dynamic alpha, or an NVFP4 X_q).  A position outside
 * [0, max_pos) or a slot outside [0, num_slots) skips that token and posts
 * MQ_ERR_INDEX (read with mq_async_status).  Slots must be distinct.
 * The method has no fused form of this; RoPE is the Qwen3 attention's. */
MQ_API mq_status mq_prefill_kv_rope(const void* X_bf16, const mq_nvfp4* X_q, int64_t M, const mq_nvfp4* W_kv,
                                    int64_t n_kv_heads, const int32_t* positions, const float* cos_sin,
                                    int64_t max_pos, const int64_t* slots, void* k_cache, void* v_cache,
                                    int64_t num_slots, void* ws, size_t ws_bytes, mq_stream_t stream);

/* RMSNorm fused with the quantization of its output: the NVFP4 copy of
 *   h[m][k] = bf16( fl32( fl32(x[m][k] * rstd_m) * gamma[k] ) ),
 *   ms_m = fl32( sum_k x^2 (binary64) / K ), rstd_m = fl32( 1/sqrt(ms_m + eps) ),
 *   (the kernel adds the exact squares of the BF16 values in binary64 in its
 *   own order, which gives the same ms for every BF16 input except when the
 *   sum lies within ~2^-40 relative of an FP32 rounding boundary),
 * with a dynamic tensor scale over h (alpha_h = amax|h| / 2688, 1 if 0) and
 * Eq. 2 / Eq. 3 as mq_quantize_activation -- the same codes and scales as an
 * unfused RMSNorm writing BF16 h followed by mq_quantize_activation(h), with
 * h never written to memory (two reads of X instead of a write and three
 * reads of h).  This puts the activation quantization inside the producer of
 * the prefill linear's input (the pages give no fused design; RMSNorm is the
 * pre-projection norm of the Qwen3 layers they evaluate).
 * X [M, K] BF16, gamma [K] BF16, both 16-byte aligned; eps finite >= 0;
 * K % 64 == 0.  h_debug: optional BF16 [M, K] output of h (testing).
 * Workspace: mq_workspace_bytes(M, K) (it also holds the M per-row factors).
 * Errors as mq_quantize_activation (NaN/Inf in h -> MQ_ERR_NONFINITE). */
MQ_API mq_status mq_rmsnorm_quantize(const void* X_bf16, int64_t M, int64_t K, const void* gamma_bf16, float eps,
                                     const mq_nvfp4* out, void* h_debug, void* ws, size_t ws_bytes,
                                     mq_stream_t stream);

/* Uniform-NVFP4 decode (the decode side of the paper's "uniform NVFP4"
 * comparison, Section 4, whose decode also runs in NVFP4):
 * Y[M,N] = bf16(fl(alpha_x*alpha_w) * sum_k (sigma_x q_x)(sigma_w q_w)), FP32
 * accumulation, with X [M, K] BF16 quantized on the fly (Eq. 2 / Eq. 3, dynamic
 * alpha_x unless alpha_static is given) into the workspace, and W the NVFP4
 * weight from mq_quantize_weight (not gate/up interleaved).  The same weight
 * bytes as the prefill path; 0.5625 instead of 2 bytes per weight element
 * streamed per token batch.  M in [1, 128]; K % 64 == 0; N % 16 == 0; X and
 * Y 16-byte aligned.  Workspace: mq_workspace_bytes(M, K), zero-filled once;
 * mq_decode_workspace_bytes(M, N, K) for the fastest launch shape.
 * Errors as mq_prefill_linear. */
MQ_API mq_status mq_decode_linear_nvfp4(const void* X_bf16, int64_t M, const mq_nvfp4* W, const float* alpha_static,
                                        void* Y_bf16, void* ws, size_t ws_bytes, mq_stream_t stream);

/* Copy the block scales of `t` to plain row-major [rows, cols/16] bytes. */
MQ_API mq_status mq_unswizzle_scales(const mq_nvfp4* t, uint8_t* rowmajor_out, mq_stream_t stream);

/* Self-test of the device E2M1 rounding used by the quantizers: for every
 * FP32 value v in [0, 8] and -v, compares the sm_100 conversion instruction
 * (cvt.rn.satfinite.e2m1x2.f32) with the definition of Pi_FP4 in Eq. 2
 * (nearest E2M1 magnitude, ties to even, clipped at 6, sign kept) and ADDS the
 * numbers of mismatches to mismatch_counts[0] (positive v) and [1] (negative
 * v), two device uint64 the caller zero-fills.  Both must stay 0. */
MQ_API mq_status mq_selftest_e2m1(unsigned long long* mismatch_counts, mq_stream_t stream);

/* Self-test of the failure path: one warp waits, with the same bounded
 * mbarrier wait every pipeline stage uses, for a phase that nothing ever
 * completes.  After timeout_ns (1 .. 2e9) the wait gives up, MQ_ERR_TIMEOUT is
 * posted to workspace `ws` (read it with mq_async_status) and the kernel
 * returns normally: no fault, the context stays usable.  If waited_ns is not
 * NULL (8-byte aligned device pointer) it receives the nanoseconds waited.
 * Returns MQ_ERR_INVALID_ARG for a timeout out of range.  The method has no
 * counterpart: it checks this library's own error reporting. */
MQ_API mq_status mq_selftest_timeout(void* ws, size_t ws_bytes, uint64_t timeout_ns, unsigned long long* waited_ns,
                                     mq_stream_t stream);

/* Synchronize `stream`, then read and clear the asynchronous error bits of
 * workspace `ws`: MQ_OK, MQ_ERR_NONFINITE, MQ_ERR_TIMEOUT, MQ_ERR_INDEX (or MQ_ERR_CUDA if
 * the synchronization itself failed). */
MQ_API mq_status mq_async_status(void* ws, mq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MIXQUANT_H */
