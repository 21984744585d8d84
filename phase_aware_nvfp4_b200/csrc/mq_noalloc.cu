// mq_noalloc.cu -- mq_prefill_linear_noalloc: the NVFP4 prefill linear layer
// for callers that cannot allocate device memory.
//
// Some callers have no way to give the library a workspace: a plugin inside
// an inference engine that owns every byte of device memory and forbids
// allocations at enqueue time, or a latency-critical serving loop where a
// cudaMalloc (which can synchronize the device) is not acceptable.  This
// entry point runs the same kernels as mq_prefill_linear, but its scratch
// memory (the control block of the amax pass and the NVFP4 copy of the
// activation) lives in one file-scope __device__ array that the CUDA module
// loader reserves when the library is loaded.  Each GPU that loads the
// library holds this array until the process exits.
#include <mutex>

#include "mq_abi_checks.h"

namespace mq {
namespace {

// The scratch array.  In host code its name is only a host-side stand-in for
// the symbol, not a device address; the device address is obtained below
// with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MQ_NOALLOC_SCRATCH_BYTES];

// Device address of the array, per device ordinal (device_info() refuses
// ordinals >= 64).  Only a successful lookup is kept, so a first call that
// failed (for example one made during stream capture) is retried by the next.
std::mutex g_mu;
uint8_t* g_ptr[64] = {};

// Once per device, with that device current: look up the device address of
// the scratch array.  Nothing in the array needs initialising here: every
// call resets the one counter that must start at zero on its own stream.
cudaError_t scratch_for_device(int dev, uint8_t** out)
{
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_ptr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_ptr[dev] = static_cast<uint8_t*>(p);
    }
    *out = g_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" MQ_API mq_status mq_prefill_linear_noalloc(const void* X_bf16, int64_t M, const mq_nvfp4* W,
                                                      const float* alpha_static, void* Y_bf16, mq_stream_t stream)
{
    // The same argument checks as mq_prefill_linear with X_bf16 and MQ_EPI_BF16.
    if (X_bf16 == nullptr || Y_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if (W == nullptr || W->codes == nullptr || W->scales == nullptr || W->alpha == nullptr) return MQ_ERR_INVALID_ARG;
    const int64_t N = W->rows, K = W->cols;
    mq_status st = check_linear_shape(M, N, K);
    if (st != MQ_OK) return st;
    if ((st = check_nvfp4(W, N, K)) != MQ_OK) return st;
    if (!aligned16(X_bf16) || !aligned16(Y_bf16)) return MQ_ERR_ALIGNMENT;
    // The activation's NVFP4 copy plus the control block must fit the static array.
    const size_t codes_b = align_up(nvfp4_codes_bytes(M, K), kWsAlign);
    const size_t need = kWsControlBytes + codes_b + align_up(nvfp4_scales_bytes(M, K), kWsAlign);
    if (need > (size_t)MQ_NOALLOC_SCRATCH_BYTES) return MQ_ERR_WORKSPACE;

    DeviceInfo di;
    if ((st = check_device(&di)) != MQ_OK) return st;
    uint8_t* base = nullptr;
    if (scratch_for_device(di.device, &base) != cudaSuccess) return MQ_ERR_CUDA;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    WsControl* ctrl = reinterpret_cast<WsControl*>(base);
    uint32_t* partials = reinterpret_cast<uint32_t*>(base + kWsPartialsOffset);
    uint8_t* xq_codes = base + kWsControlBytes;
    uint8_t* xq_scales = xq_codes + codes_b;

    // The amax pass counts finished blocks in the control block and its last
    // block resets the counter; calls that overlapped on the GPU can leave it
    // wrong, so each call starts from zero (stream-ordered, no allocation).
    if (cudaMemsetAsync(&ctrl->amax_ticket, 0, sizeof(uint32_t), s) != cudaSuccess) return MQ_ERR_CUDA;
    const float* alpha_x = (alpha_static != nullptr) ? alpha_static : &ctrl->alpha;
    if (launch_quantize(X_bf16, M, K, alpha_static, &ctrl->alpha, xq_codes, xq_scales, 0, ctrl, partials, di, s) !=
        cudaSuccess)
        return MQ_ERR_CUDA;

    GemmArgs g{};
    g.a_codes = xq_codes;
    g.a_scales = xq_scales;
    g.a_alpha = alpha_x;
    g.b_codes = W->codes;
    g.b_scales = W->scales;
    g.b_alpha = W->alpha;
    g.M = M;
    g.N = N;
    g.K = K;
    g.epilogue = 0;
    g.y = Y_bf16;
    g.ctrl = ctrl;
    return cuda_status(launch_gemm_nvfp4(g, di, s));
}
