// mq_api.cu -- the extern "C" entry points of libmixquant (include/mixquant.h):
// argument validation, workspace layout, tensor-map creation and the
// stream-ordered launch sequence of each call.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "mq_abi_checks.h"

namespace mq {

// ---------------------------------------------------------------- device info

cudaError_t device_info(DeviceInfo* out)
{
    static std::mutex mu;
    static DeviceInfo cache[64];
    static bool valid[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!valid[dev]) {
        DeviceInfo d{};
        d.device = dev;
        int v = 0;
        if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        d.num_sms = v;
        if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
        d.cc_major = v;
        if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
        d.cc_minor = v;
        if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
        d.max_smem_optin = (size_t)v;
        if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess) return e;
        d.smem_per_sm = (size_t)v;
        if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
        d.smem_reserved_per_cta = (size_t)v;
        cache[dev] = d;
        valid[dev] = true;
    }
    *out = cache[dev];
    return cudaSuccess;
}

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    std::memset(map, 0, sizeof(*map));
    CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    std::memset(map, 0, sizeof(*map));
    CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- workspace

namespace {

struct Ws {
    WsControl* ctrl;
    uint32_t* partials;
    uint8_t* xq_codes;
    uint8_t* xq_scales;
};

size_t ws_bytes_for(int64_t M, int64_t K)
{
    if (M <= 0 || K <= 0) return kWsControlBytes;
    return kWsControlBytes + align_up(nvfp4_codes_bytes(M, K), kWsAlign) + align_up(nvfp4_scales_bytes(M, K), kWsAlign);
}

Ws carve(void* ws, int64_t M, int64_t K)
{
    uint8_t* b = static_cast<uint8_t*>(ws);
    Ws w{};
    w.ctrl = reinterpret_cast<WsControl*>(b);
    w.partials = reinterpret_cast<uint32_t*>(b + kWsPartialsOffset);
    if (M > 0 && K > 0) {
        w.xq_codes = b + kWsControlBytes;
        w.xq_scales = w.xq_codes + align_up(nvfp4_codes_bytes(M, K), kWsAlign);
    }
    return w;
}

// Decode workspace: the per-tile counters of the split-K reduction across
// independent CTAs sit in the control block, behind the amax partials, at an
// offset that does not depend on the shapes (so one workspace serves calls of
// any shape: every counter is zero between calls); the FP32 partial tiles
// follow what mq_workspace_bytes(M, K) covers (control block and the tokens'
// NVFP4 copy), up to kDecodeMaxSplit CTAs per tile, M rows of 128 each.
constexpr int64_t kDecodeMaxSplit = 8;
constexpr size_t kDecodeCtrOffset = kWsPartialsOffset + (size_t)kAmaxMaxBlocks * 4u;
constexpr int64_t kDecodeMaxTiles = (int64_t)((kWsControlBytes - kDecodeCtrOffset) / 4u);
static_assert(kDecodeCtrOffset < kWsControlBytes, "decode counters inside the control block");

constexpr int64_t kDecodeMaxGpartTokens = 16;   // the decode kernels split K this way up to 16 tokens

size_t decode_ws_bytes(int64_t M, int64_t N, int64_t K)
{
    const int64_t n_tiles = (N + 127) / 128;
    if (M > kDecodeMaxGpartTokens || n_tiles > kDecodeMaxTiles) return ws_bytes_for(M, K);
    return align_up(ws_bytes_for(M, K), 256) + (size_t)kDecodeMaxSplit * (size_t)n_tiles * (size_t)M * 128u * 4u;
}

DecodeSplitWs decode_split_ws(void* ws, size_t ws_bytes, int64_t M, int64_t N, int64_t K)
{
    const int64_t n_tiles = (N + 127) / 128;
    const size_t part_off = align_up(ws_bytes_for(M, K), 256);
    const size_t two_splits = 2u * (size_t)n_tiles * (size_t)M * 128u * 4u;
    if (n_tiles > kDecodeMaxTiles || ws_bytes < part_off + two_splits)
        return DecodeSplitWs{nullptr, nullptr, 0};   // the K split stays inside clusters
    uint8_t* b = static_cast<uint8_t*>(ws);
    return DecodeSplitWs{reinterpret_cast<float*>(b + part_off), reinterpret_cast<uint32_t*>(b + kDecodeCtrOffset),
                         ws_bytes - part_off};
}

mq_status check_ws(void* ws, size_t ws_bytes, size_t need)
{
    if (ws == nullptr || ws_bytes < need) return MQ_ERR_WORKSPACE;
    if (!aligned16(ws)) return MQ_ERR_ALIGNMENT;
    return MQ_OK;
}

// Tensor amax (unless a static alpha is given) and quantization.  Returns the device
// pointer of the tensor scale used in *alpha_used.  With a static alpha and
// copy_static, the value is also copied to alpha_out.
mq_status quantize_into(const void* x, int64_t rows, int64_t K, const float* alpha_static, uint8_t* codes,
                        uint8_t* scales, float* alpha_out, bool copy_static, int64_t interleave_half,
                        const Ws& w, const DeviceInfo& di, cudaStream_t s, const float** alpha_used,
                        bool scale_search = false)
{
    if (alpha_static != nullptr && copy_static && alpha_out != alpha_static) {
        if (cudaMemcpyAsync(alpha_out, alpha_static, sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return MQ_ERR_CUDA;
    }
    if (alpha_used != nullptr) *alpha_used = (alpha_static != nullptr) ? alpha_static : alpha_out;
    return cuda_status(launch_quantize(x, rows, K, alpha_static, alpha_out, codes, scales, interleave_half, w.ctrl,
                                       w.partials, di, s, scale_search));
}

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" {

const char* mq_status_string(mq_status s)
{
    switch (s) {
        case MQ_OK: return "MQ_OK";
        case MQ_ERR_INVALID_ARG: return "MQ_ERR_INVALID_ARG";
        case MQ_ERR_SHAPE: return "MQ_ERR_SHAPE";
        case MQ_ERR_ALIGNMENT: return "MQ_ERR_ALIGNMENT";
        case MQ_ERR_WORKSPACE: return "MQ_ERR_WORKSPACE";
        case MQ_ERR_NONFINITE: return "MQ_ERR_NONFINITE";
        case MQ_ERR_TIMEOUT: return "MQ_ERR_TIMEOUT";
        case MQ_ERR_CUDA: return "MQ_ERR_CUDA";
        case MQ_ERR_DEVICE: return "MQ_ERR_DEVICE";
        case MQ_ERR_INDEX: return "MQ_ERR_INDEX";
    }
    return "MQ_ERR_UNKNOWN";
}

const char* mq_version(void) { return "0.1.0"; }

mq_status mq_nvfp4_sizes(int64_t rows, int64_t cols, size_t* codes_bytes, size_t* scales_bytes)
{
    if (codes_bytes == nullptr || scales_bytes == nullptr) return MQ_ERR_INVALID_ARG;
    if (rows < 1 || cols < 64 || cols % 64 != 0) return MQ_ERR_SHAPE;
    *codes_bytes = nvfp4_codes_bytes(rows, cols);
    *scales_bytes = nvfp4_scales_bytes(rows, cols);
    return MQ_OK;
}

size_t mq_workspace_bytes(int64_t M, int64_t K) { return ws_bytes_for(M, K); }

size_t mq_decode_workspace_bytes(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 1 || K < 1) return kWsControlBytes;
    return decode_ws_bytes(M, N, K);
}

mq_status mq_quantize_weight(const void* W_bf16, int64_t N, int64_t K, int gate_up_interleave, const mq_nvfp4* out,
                             void* ws, size_t ws_bytes, mq_stream_t stream)
{
    if (W_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if (N < 1 || K < 64 || K % 64 != 0 || N > kMaxDim || K > kMaxDim) return MQ_ERR_SHAPE;
    if (gate_up_interleave && (N % 128 != 0)) return MQ_ERR_SHAPE;
    if (!aligned16(W_bf16)) return MQ_ERR_ALIGNMENT;
    mq_status st = check_nvfp4(out, N, K);
    if (st != MQ_OK) return st;
    if ((st = check_ws(ws, ws_bytes, kWsControlBytes)) != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    const Ws w = carve(ws, 0, 0);
    return quantize_into(W_bf16, N, K, nullptr, out->codes, out->scales, out->alpha, false,
                         gate_up_interleave ? N / 2 : 0, w, di, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

mq_status mq_quantize_activation(const void* X_bf16, int64_t M, int64_t K, const float* alpha_static,
                                 const mq_nvfp4* out, void* ws, size_t ws_bytes, mq_stream_t stream)
{
    if (X_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if (M < 1 || K < 64 || K % 64 != 0 || M > kMaxDim || K > kMaxDim) return MQ_ERR_SHAPE;
    if (!aligned16(X_bf16)) return MQ_ERR_ALIGNMENT;
    mq_status st = check_nvfp4(out, M, K);
    if (st != MQ_OK) return st;
    if ((st = check_ws(ws, ws_bytes, kWsControlBytes)) != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    const Ws w = carve(ws, 0, 0);
    return quantize_into(X_bf16, M, K, alpha_static, out->codes, out->scales, out->alpha, true, 0, w, di,
                         reinterpret_cast<cudaStream_t>(stream), nullptr);
}

mq_status mq_quantize(const void* X_bf16, int64_t rows, int64_t K, const float* alpha_static, unsigned flags,
                      const mq_nvfp4* out, void* ws, size_t ws_bytes, mq_stream_t stream)
{
    if (X_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if ((flags & ~(unsigned)(MQ_QUANT_GATE_UP_INTERLEAVE | MQ_QUANT_SCALE_SEARCH)) != 0) return MQ_ERR_INVALID_ARG;
    if (rows < 1 || K < 64 || K % 64 != 0 || rows > kMaxDim || K > kMaxDim) return MQ_ERR_SHAPE;
    const bool interleave = (flags & MQ_QUANT_GATE_UP_INTERLEAVE) != 0;
    if (interleave && rows % 128 != 0) return MQ_ERR_SHAPE;
    if (!aligned16(X_bf16)) return MQ_ERR_ALIGNMENT;
    mq_status st = check_nvfp4(out, rows, K);
    if (st != MQ_OK) return st;
    if ((st = check_ws(ws, ws_bytes, kWsControlBytes)) != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    const Ws w = carve(ws, 0, 0);
    return quantize_into(X_bf16, rows, K, alpha_static, out->codes, out->scales, out->alpha, true,
                         interleave ? rows / 2 : 0, w, di, reinterpret_cast<cudaStream_t>(stream), nullptr,
                         (flags & MQ_QUANT_SCALE_SEARCH) != 0);
}

mq_status mq_prefill_kv_rope(const void* X_bf16, const mq_nvfp4* X_q, int64_t M, const mq_nvfp4* W_kv,
                             int64_t n_kv_heads, const int32_t* positions, const float* cos_sin, int64_t max_pos,
                             const int64_t* slots, void* k_cache, void* v_cache, int64_t num_slots, void* ws,
                             size_t ws_bytes, mq_stream_t stream)
{
    if ((X_bf16 == nullptr) == (X_q == nullptr)) return MQ_ERR_INVALID_ARG;
    if (W_kv == nullptr || W_kv->codes == nullptr || W_kv->scales == nullptr || W_kv->alpha == nullptr)
        return MQ_ERR_INVALID_ARG;
    if (positions == nullptr || cos_sin == nullptr || slots == nullptr || k_cache == nullptr || v_cache == nullptr)
        return MQ_ERR_INVALID_ARG;
    const int64_t N = W_kv->rows, K = W_kv->cols;
    if (n_kv_heads < 1 || n_kv_heads > 4096 || N != 2 * n_kv_heads * 128) return MQ_ERR_SHAPE;
    if (M < 1 || M > kMaxDim || K < 64 || K % 64 != 0 || K > kMaxDim) return MQ_ERR_SHAPE;
    if (max_pos < 1 || num_slots < 1) return MQ_ERR_SHAPE;
    if (!aligned16(cos_sin) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(positions) & 3u) || (reinterpret_cast<uintptr_t>(slots) & 7u))
        return MQ_ERR_ALIGNMENT;
    mq_status st = check_nvfp4(W_kv, N, K);
    if (st != MQ_OK) return st;
    const bool quantize_x = X_bf16 != nullptr;
    if (quantize_x) {
        if (!aligned16(X_bf16)) return MQ_ERR_ALIGNMENT;
    } else if ((st = check_nvfp4(X_q, M, K)) != MQ_OK) {
        return st;
    }
    if ((st = check_ws(ws, ws_bytes, quantize_x ? ws_bytes_for(M, K) : kWsControlBytes)) != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Ws w = carve(ws, quantize_x ? M : 0, quantize_x ? K : 0);
    GemmArgs g{};
    if (quantize_x) {
        const float* ax = nullptr;
        st = quantize_into(X_bf16, M, K, nullptr, w.xq_codes, w.xq_scales, &w.ctrl->alpha, false, 0, w, di, s, &ax);
        if (st != MQ_OK) return st;
        g.a_codes = w.xq_codes;
        g.a_scales = w.xq_scales;
        g.a_alpha = ax;
    } else {
        g.a_codes = X_q->codes;
        g.a_scales = X_q->scales;
        g.a_alpha = X_q->alpha;
    }
    g.b_codes = W_kv->codes;
    g.b_scales = W_kv->scales;
    g.b_alpha = W_kv->alpha;
    g.M = M;
    g.N = N;
    g.K = K;
    g.epilogue = 2;
    g.positions = positions;
    g.cos_sin = cos_sin;
    g.max_pos = max_pos;
    g.slots = slots;
    g.k_cache = static_cast<uint16_t*>(k_cache);
    g.v_cache = static_cast<uint16_t*>(v_cache);
    g.num_slots = num_slots;
    g.n_heads = (int)n_kv_heads;
    g.ctrl = w.ctrl;
    return cuda_status(launch_gemm_nvfp4(g, di, s));
}

mq_status mq_rmsnorm_quantize(const void* X_bf16, int64_t M, int64_t K, const void* gamma_bf16, float eps,
                              const mq_nvfp4* out, void* h_debug, void* ws, size_t ws_bytes, mq_stream_t stream)
{
    if (X_bf16 == nullptr || gamma_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return MQ_ERR_INVALID_ARG;
    if (M < 1 || M > kMaxDim || K < 64 || K % 64 != 0 || K > kMaxDim) return MQ_ERR_SHAPE;
    if (!aligned16(X_bf16) || !aligned16(gamma_bf16) || (h_debug != nullptr && !aligned16(h_debug)))
        return MQ_ERR_ALIGNMENT;
    mq_status st = check_nvfp4(out, M, K);
    if (st != MQ_OK) return st;
    if ((st = check_ws(ws, ws_bytes, ws_bytes_for(M, K))) != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    const Ws w = carve(ws, M, K);
    float* rstd = reinterpret_cast<float*>(w.xq_codes);   // M floats; the NVFP4 scratch is not used here
    return cuda_status(launch_rmsnorm_quantize(X_bf16, M, K, gamma_bf16, eps, rstd, out->codes, out->scales,
                                               out->alpha, h_debug, w.ctrl, w.partials, di,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

mq_status mq_prefill_linear(const void* X_bf16, const mq_nvfp4* X_q, int64_t M, const mq_nvfp4* W, mq_epilogue epi,
                            const float* alpha_static, const float* alpha_h, void* Y, const mq_nvfp4* H_out,
                            void* h_debug, void* ws, size_t ws_bytes, mq_stream_t stream)
{
    if ((X_bf16 == nullptr) == (X_q == nullptr)) return MQ_ERR_INVALID_ARG;
    if (W == nullptr || W->codes == nullptr || W->scales == nullptr || W->alpha == nullptr) return MQ_ERR_INVALID_ARG;
    if (epi != MQ_EPI_BF16 && epi != MQ_EPI_SILU_MUL_NVFP4 && epi != MQ_EPI_SILU_MUL_BF16) return MQ_ERR_INVALID_ARG;
    const int64_t N = W->rows, K = W->cols;
    mq_status st = check_linear_shape(M, N, K);
    if (st != MQ_OK) return st;
    if ((st = check_nvfp4(W, N, K)) != MQ_OK) return st;
    if (epi == MQ_EPI_BF16 || epi == MQ_EPI_SILU_MUL_BF16) {
        if (Y == nullptr) return MQ_ERR_INVALID_ARG;
        if (epi == MQ_EPI_SILU_MUL_BF16 && N % 128 != 0) return MQ_ERR_SHAPE;
        if (!aligned16(Y)) return MQ_ERR_ALIGNMENT;
    } else {
        if (alpha_h == nullptr) return MQ_ERR_INVALID_ARG;
        if (N % 128 != 0) return MQ_ERR_SHAPE;
        if (H_out == nullptr || H_out->codes == nullptr || H_out->scales == nullptr) return MQ_ERR_INVALID_ARG;
        if (H_out->rows != M || H_out->cols != N / 2) return MQ_ERR_SHAPE;
        if (!aligned16(H_out->codes) || !aligned16(H_out->scales)) return MQ_ERR_ALIGNMENT;
        if (h_debug != nullptr && !aligned16(h_debug)) return MQ_ERR_ALIGNMENT;
    }
    const bool quantize_x = X_bf16 != nullptr;
    if (quantize_x) {
        if (!aligned16(X_bf16)) return MQ_ERR_ALIGNMENT;
    } else if ((st = check_nvfp4(X_q, M, K)) != MQ_OK) {
        return st;
    }
    if ((st = check_ws(ws, ws_bytes, quantize_x ? ws_bytes_for(M, K) : kWsControlBytes)) != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    const Ws w = carve(ws, quantize_x ? M : 0, quantize_x ? K : 0);
    GemmArgs g{};
    if (quantize_x) {
        const float* ax = nullptr;
        st = quantize_into(X_bf16, M, K, alpha_static, w.xq_codes, w.xq_scales, &w.ctrl->alpha, false, 0, w, di, s,
                           &ax);
        if (st != MQ_OK) return st;
        g.a_codes = w.xq_codes;
        g.a_scales = w.xq_scales;
        g.a_alpha = ax;
    } else {
        g.a_codes = X_q->codes;
        g.a_scales = X_q->scales;
        g.a_alpha = X_q->alpha;
    }
    g.b_codes = W->codes;
    g.b_scales = W->scales;
    g.b_alpha = W->alpha;
    g.M = M;
    g.N = N;
    g.K = K;
    // kernel epilogues: 0 BF16 Y, 1 SiLU-mul -> NVFP4 h, 2 RoPE + KV cache, 3 SiLU-mul -> BF16 h
    g.epilogue = (epi == MQ_EPI_SILU_MUL_BF16) ? 3 : (int)epi;
    g.y = Y;
    if (epi == MQ_EPI_SILU_MUL_NVFP4) {
        g.h_codes = H_out->codes;
        g.h_scales = H_out->scales;
        g.h_alpha = alpha_h;
        g.h_debug = static_cast<uint16_t*>(h_debug);
    }
    g.ctrl = w.ctrl;
    return cuda_status(launch_gemm_nvfp4(g, di, s));
}

mq_status mq_decode_linear(const void* X_bf16, int64_t M, const void* W_bf16, int64_t N, int64_t K, void* Y_bf16,
                           void* ws, size_t ws_bytes, mq_stream_t stream)
{
    if (X_bf16 == nullptr || W_bf16 == nullptr || Y_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if (M < 1 || M > 256 || N < 16 || N % 16 != 0 || K < 64 || K % 64 != 0) return MQ_ERR_SHAPE;
    if (N > kMaxDim || K > kMaxDim) return MQ_ERR_SHAPE;
    if (!aligned16(X_bf16) || !aligned16(W_bf16) || !aligned16(Y_bf16)) return MQ_ERR_ALIGNMENT;
    mq_status st = check_ws(ws, ws_bytes, kWsControlBytes);
    if (st != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    const Ws w = carve(ws, 0, 0);
    const DecodeSplitWs sw = decode_split_ws(ws, ws_bytes, M, N, K);
    return cuda_status(
        launch_decode_bf16(X_bf16, M, W_bf16, N, K, Y_bf16, w.ctrl, sw, di, reinterpret_cast<cudaStream_t>(stream)));
}

mq_status mq_decode_linear_nvfp4(const void* X_bf16, int64_t M, const mq_nvfp4* W, const float* alpha_static,
                                 void* Y_bf16, void* ws, size_t ws_bytes, mq_stream_t stream)
{
    if (X_bf16 == nullptr || Y_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if (W == nullptr || W->codes == nullptr || W->scales == nullptr || W->alpha == nullptr) return MQ_ERR_INVALID_ARG;
    const int64_t N = W->rows, K = W->cols;
    if (M < 1 || M > 128 || N < 16 || N % 16 != 0 || K < 64 || K % 64 != 0) return MQ_ERR_SHAPE;
    if (N > kMaxDim || K > kMaxDim) return MQ_ERR_SHAPE;
    mq_status st = check_nvfp4(W, N, K);
    if (st != MQ_OK) return st;
    if (!aligned16(X_bf16) || !aligned16(Y_bf16)) return MQ_ERR_ALIGNMENT;
    if ((st = check_ws(ws, ws_bytes, ws_bytes_for(M, K))) != MQ_OK) return st;
    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Ws w = carve(ws, M, K);
    const DecodeSplitWs sw = decode_split_ws(ws, ws_bytes, M, N, K);
    // One kernel that quantizes the tokens itself; when its token slice does not
    // fit in shared memory, the quantization kernel and then the decode GEMM.
    const cudaError_t fe = launch_decode_nvfp4_fused(X_bf16, M, alpha_static, W->codes, W->scales, W->alpha, N, K,
                                                     Y_bf16, w.ctrl, sw, di, s);
    if (fe != cudaErrorNotSupported) return cuda_status(fe);
    const float* ax = nullptr;
    st = quantize_into(X_bf16, M, K, alpha_static, w.xq_codes, w.xq_scales, &w.ctrl->alpha, false, 0, w, di, s, &ax);
    if (st != MQ_OK) return st;
    return cuda_status(launch_decode_nvfp4(w.xq_codes, w.xq_scales, ax, M, W->codes, W->scales, W->alpha, N, K, Y_bf16,
                                           w.ctrl, sw, di, s));
}

mq_status mq_unswizzle_scales(const mq_nvfp4* t, uint8_t* rowmajor_out, mq_stream_t stream)
{
    if (t == nullptr || t->scales == nullptr || rowmajor_out == nullptr) return MQ_ERR_INVALID_ARG;
    if (t->rows < 1 || t->cols < 64 || t->cols % 64 != 0) return MQ_ERR_SHAPE;
    DeviceInfo di;
    mq_status st = check_device(&di);
    if (st != MQ_OK) return st;
    return cuda_status(launch_unswizzle(t->scales, t->rows, t->cols, rowmajor_out,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

mq_status mq_selftest_e2m1(unsigned long long* mismatch_counts, mq_stream_t stream)
{
    if (mismatch_counts == nullptr) return MQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mismatch_counts) & 7u) != 0) return MQ_ERR_ALIGNMENT;
    DeviceInfo di;
    mq_status st = check_device(&di);
    if (st != MQ_OK) return st;
    return cuda_status(launch_selftest_e2m1(mismatch_counts, di, reinterpret_cast<cudaStream_t>(stream)));
}

mq_status mq_selftest_timeout(void* ws, size_t ws_bytes, uint64_t timeout_ns, unsigned long long* waited_ns,
                              mq_stream_t stream)
{
    if (timeout_ns == 0 || timeout_ns > kWaitTimeoutNs) return MQ_ERR_INVALID_ARG;
    if (waited_ns != nullptr && (reinterpret_cast<uintptr_t>(waited_ns) & 7u) != 0) return MQ_ERR_ALIGNMENT;
    mq_status st = check_ws(ws, ws_bytes, kWsControlBytes);
    if (st != MQ_OK) return st;
    DeviceInfo di;
    st = check_device(&di);
    if (st != MQ_OK) return st;
    return cuda_status(launch_selftest_timeout(static_cast<WsControl*>(ws), timeout_ns, waited_ns,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

mq_status mq_async_status(void* ws, mq_stream_t stream)
{
    if (ws == nullptr) return MQ_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    WsControl* ctrl = static_cast<WsControl*>(ws);
    uint32_t bits = 0;
    if (cudaMemcpyAsync(&bits, &ctrl->error_bits, sizeof(bits), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MQ_ERR_CUDA;
    if (bits != 0) {
        if (cudaMemsetAsync(&ctrl->error_bits, 0, sizeof(uint32_t), s) != cudaSuccess) return MQ_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return MQ_ERR_CUDA;
    }
    if (bits & kErrTimeout) return MQ_ERR_TIMEOUT;
    if (bits & kErrIndex) return MQ_ERR_INDEX;
    if (bits & kErrNonFinite) return MQ_ERR_NONFINITE;
    return MQ_OK;
}

}  // extern "C"
