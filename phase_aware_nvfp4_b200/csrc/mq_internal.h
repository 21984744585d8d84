// mq_internal.h -- declarations shared by the CUDA sources of libmixquant
// (not part of the public ABI; the public header is include/mixquant.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mq {

// Bounded waits: a device-side wait on an mbarrier gives up after this much
// wall time, posts kErrTimeout and unwinds.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

// Asynchronous error bits posted by kernels into the workspace control block.
constexpr uint32_t kErrNonFinite = 1u;  // NaN / Inf in a tensor being quantized
constexpr uint32_t kErrTimeout = 2u;    // a pipeline wait gave up
constexpr uint32_t kErrIndex = 4u;      // a position or cache slot out of range (KV epilogue)

// Control block at the start of every workspace (zero-filled by the caller
// once, before first use; kernels keep the counters consistent afterwards).
struct WsControl {
    uint32_t error_bits;   // OR of kErr* posted since the last status query
    uint32_t amax_ticket;  // blocks of the running amax pass that have finished
    uint32_t epoch;        // bumped when a single-launch amax pass publishes its alpha
    uint32_t reserved[5];
    float alpha;           // tensor scale of the activation quantized in-workspace
    uint32_t pad[55];
};
static_assert(sizeof(WsControl) == 256, "control block is 256 bytes");

constexpr int kAmaxMaxBlocks = 2048;          // partial maxima slots
constexpr size_t kWsPartialsOffset = 256;     // uint32 partials follow the control block
constexpr size_t kWsControlBytes = 16384;     // control + partials, rounded up
constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// NVFP4 storage geometry (see include/mixquant.h for the layout).
inline int64_t sf_atoms_per_rowblk(int64_t cols) { return ((cols + 255) / 256) * 4; }
inline int64_t sf_rowblks(int64_t rows) { return (rows + 127) / 128; }
inline size_t nvfp4_codes_bytes(int64_t rows, int64_t cols) { return (size_t)rows * (size_t)(cols / 2); }
inline size_t nvfp4_scales_bytes(int64_t rows, int64_t cols)
{
    return (size_t)sf_rowblks(rows) * (size_t)sf_atoms_per_rowblk(cols) * 512u;
}

struct DeviceInfo {
    int device;
    int num_sms;
    int cc_major, cc_minor;
    size_t max_smem_optin;
    size_t smem_per_sm;           // shared memory of one SM
    size_t smem_reserved_per_cta; // shared memory the runtime reserves per resident CTA
};
// Cached per device; returns cudaSuccess or the error of the attribute query.
cudaError_t device_info(DeviceInfo* out);

// ----- launchers (stream-ordered, no host synchronisation) -----

// amax of n BF16 values (n % 8 == 0, 16-byte aligned) -> *alpha_out = amax/2688
// (1 if amax == 0); kErrNonFinite posted on NaN/Inf.
cudaError_t launch_amax(const void* x, int64_t n, float* alpha_out, WsControl* ctrl, uint32_t* partials,
                        const DeviceInfo& di, cudaStream_t s);

// NVFP4 quantization of X [rows, K] (ld = K).  With alpha_static the tensor
// scale is *alpha_static; otherwise alpha = amax/2688 (1 if amax == 0) is
// computed first and stored at *alpha_out (kErrNonFinite on NaN/Inf): by the
// amax kernel, or, for tensors of at most one tile per SM, inside one
// cooperative launch of the quantization kernel.  interleave_half > 0
// interleaves gate/up rows in 16-row groups (output row 32c+t <- input row
// 16c+t for t<16, I+16c+t-16 else).
// scale_search: per block, also try the E4M3 neighbours of the Eq. 3 scale
// and keep the smallest binary32 squared error (ties keep the Eq. 3 scale).
cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, const float* alpha_static, float* alpha_out,
                            uint8_t* codes, uint8_t* scales, int64_t interleave_half, WsControl* ctrl,
                            uint32_t* partials, const DeviceInfo& di, cudaStream_t s, bool scale_search = false);

// RMSNorm of X [rows, K] (gamma [K], eps) fused with the NVFP4 quantization of
// its BF16 output h: rstd per row to `rstd`, alpha_h to *alpha_out, codes and
// scales of h; h itself to h_out when not null.
cudaError_t launch_rmsnorm_quantize(const void* x, int64_t rows, int64_t K, const void* gamma, float eps,
                                    float* rstd, uint8_t* codes, uint8_t* scales, float* alpha_out, void* h_out,
                                    WsControl* ctrl, uint32_t* partials, const DeviceInfo& di, cudaStream_t s);

// Sweep of the E2M1 conversion instruction against the definition; adds
// mismatch counts for positive / negative inputs into counts[0] / counts[1].
cudaError_t launch_selftest_e2m1(unsigned long long* counts, const DeviceInfo& di, cudaStream_t s);
// A bounded mbarrier wait that runs out (nothing arrives): posts kErrTimeout.
cudaError_t launch_selftest_timeout(WsControl* ctrl, uint64_t timeout_ns, unsigned long long* waited_ns,
                                    cudaStream_t s);

cudaError_t launch_unswizzle(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* out, cudaStream_t s);

// Block-scaled NVFP4 GEMM: Y[M,N] = alpha_a*alpha_b * A[M,K] B[N,K]^T.
struct GemmArgs {
    const uint8_t* a_codes;
    const uint8_t* a_scales;
    const float* a_alpha;
    const uint8_t* b_codes;
    const uint8_t* b_scales;
    const float* b_alpha;
    int64_t M, N, K;
    int epilogue;          // 0: BF16 Y; 1: SiLU-mul + NVFP4 requantize; 2: RoPE + KV-cache write
    void* y;               // epilogue 0: BF16 [M, N]
    uint8_t* h_codes;      // epilogue 1: [M, N/4] bytes (h has N/2 columns)
    uint8_t* h_scales;     // epilogue 1: scale layout for [M, N/2]
    const float* h_alpha;  // epilogue 1: static tensor scale of h
    uint16_t* h_debug;     // epilogue 1, optional: BF16 h [M, N/2]
    // epilogue 2: N = 2 * n_heads * 128 columns = K heads then V heads
    const int32_t* positions;   // [M]
    const float* cos_sin;       // [max_pos, 128]: cos of the 64 frequencies, then sin
    int64_t max_pos;
    const int64_t* slots;       // [M] cache slot of each token
    uint16_t* k_cache;          // [num_slots, n_heads, 128] BF16
    uint16_t* v_cache;
    int64_t num_slots;
    int n_heads;
    WsControl* ctrl;
};
cudaError_t launch_gemm_nvfp4(const GemmArgs& a, const DeviceInfo& di, cudaStream_t s);

// Workspace of the decode kernels' split-K reduction across independent CTAs:
// per 128-row weight tile a counter (zero when idle) and up to `part_bytes` of
// FP32 partial tiles.  part == nullptr: the K split uses clusters instead.
struct DecodeSplitWs {
    float* part;
    uint32_t* tile_ctr;
    size_t part_bytes;
};

// BF16 decode linear: Y[M,N] = X[M,K] W[N,K]^T, FP32 accumulation.
cudaError_t launch_decode_bf16(const void* x, int64_t M, const void* w, int64_t N, int64_t K, void* y,
                               WsControl* ctrl, const DecodeSplitWs& sw, const DeviceInfo& di, cudaStream_t s);

// Uniform-NVFP4 decode: Y[M,N] = bf16(fl(alpha_w*alpha_x) * sum_k dequant)
// with X [M <= 128, K] and W [N, K] both NVFP4 (codes, MMA-layout scales).
cudaError_t launch_decode_nvfp4(const uint8_t* x_codes, const uint8_t* x_scales, const float* alpha_x, int64_t M,
                                const uint8_t* w_codes, const uint8_t* w_scales, const float* alpha_w, int64_t N,
                                int64_t K, void* y, WsControl* ctrl, const DecodeSplitWs& sw, const DeviceInfo& di,
                                cudaStream_t s);

// Uniform-NVFP4 decode with the token quantization inside the kernel: X BF16
// [M <= 128, K] is quantized (Eq. 2 / Eq. 3; dynamic alpha_x unless
// alpha_static) by every CTA for its own K slice, straight into shared
// memory.  Returns cudaErrorNotSupported (nothing launched) when no launch
// shape fits the token slice in shared memory.
cudaError_t launch_decode_nvfp4_fused(const void* x, int64_t M, const float* alpha_static, const uint8_t* w_codes,
                                      const uint8_t* w_scales, const float* alpha_w, int64_t N, int64_t K, void* y,
                                      WsControl* ctrl, const DecodeSplitWs& sw, const DeviceInfo& di, cudaStream_t s);

// cuTensorMapEncodeTiled obtained from the driver at run time.
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);
// 3-D tiled map without swizzle: extents d0 (innermost) .. d2, byte strides of
// dimensions 1 and 2, box b0 x b1 x b2.
bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2);

}  // namespace mq
