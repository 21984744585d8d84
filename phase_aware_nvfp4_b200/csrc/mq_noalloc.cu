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

#include "../../include/mixquant.h"
#include "mq_internal.h"

namespace mq {
namespace {

// The scratch array.  In host code its name is only a host-side stand-in for
// the symbol, not a device address; the device address is obtained below
// with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MQ_NOALLOC_SCRATCH_BYTES];

struct ScratchState {
    std::once_flag once;
    cudaError_t setup_error = cudaSuccess;
    uint8_t* ptr = nullptr;
};

ScratchState g_state[64];

// Once per device, with that device current: look up the device address of
// the scratch array and zero its control block (error bits and the amax
// pass's block counter must start at zero; the kernels keep the counter
// consistent afterwards).
uint8_t* scratch_for_device(int dev, cudaError_t* err)
{
    ScratchState& st = g_state[dev];
    std::call_once(st.once, [&st] {
        void* p = nullptr;
        st.setup_error = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (st.setup_error != cudaSuccess) return;
        st.setup_error = cudaMemset(p, 0, kWsControlBytes);
        if (st.setup_error != cudaSuccess) return;
        st.setup_error = cudaDeviceSynchronize();
        if (st.setup_error == cudaSuccess) st.ptr = static_cast<uint8_t*>(p);
    });
    *err = st.setup_error;
    return st.ptr;
}

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" MQ_API mq_status mq_prefill_linear_noalloc(const void* X_bf16, int64_t M, const mq_nvfp4* W,
                                                      const float* alpha_static, void* Y_bf16, mq_stream_t stream)
{
    if (X_bf16 == nullptr || Y_bf16 == nullptr) return MQ_ERR_INVALID_ARG;
    if (W == nullptr || W->codes == nullptr || W->scales == nullptr || W->alpha == nullptr) return MQ_ERR_INVALID_ARG;
    const int64_t N = W->rows, K = W->cols;
    if (M < 1 || M > (int64_t)1 << 30 || K < 64 || K % 64 != 0 || N < 16 || N % 16 != 0 || N > (int64_t)1 << 30)
        return MQ_ERR_SHAPE;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(X_bf16) || !a16(Y_bf16) || !a16(W->codes) || !a16(W->scales)) return MQ_ERR_ALIGNMENT;
    // The activation's NVFP4 copy plus the control block must fit the static array.
    const size_t codes_b = align_up(nvfp4_codes_bytes(M, K), kWsAlign);
    const size_t need = kWsControlBytes + codes_b + align_up(nvfp4_scales_bytes(M, K), kWsAlign);
    if (need > (size_t)MQ_NOALLOC_SCRATCH_BYTES) return MQ_ERR_WORKSPACE;

    DeviceInfo di;
    if (device_info(&di) != cudaSuccess) return MQ_ERR_CUDA;
    if (di.cc_major != 10 || di.cc_minor != 0) return MQ_ERR_DEVICE;
    cudaError_t e = cudaSuccess;
    uint8_t* base = scratch_for_device(di.device, &e);
    if (base == nullptr || e != cudaSuccess) return MQ_ERR_CUDA;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    WsControl* ctrl = reinterpret_cast<WsControl*>(base);
    uint32_t* partials = reinterpret_cast<uint32_t*>(base + kWsPartialsOffset);
    uint8_t* xq_codes = base + kWsControlBytes;
    uint8_t* xq_scales = xq_codes + codes_b;

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
    return launch_gemm_nvfp4(g, di, s) == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}
