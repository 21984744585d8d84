// mq_abi_checks.h -- argument checks shared by the extern "C" entry points
// (mq_api.cu, mq_noalloc.cu), so that every entry point that takes the same
// kind of argument accepts and refuses exactly the same values.
#pragma once

#include <cstdint>

#include "../../include/mixquant.h"
#include "mq_internal.h"

namespace mq {

// Largest M, N or K any call accepts: keeps every byte offset and element count
// far inside 64 bits and every tensor-map coordinate inside 32 bits.
constexpr int64_t kMaxDim = (int64_t)1 << 30;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline mq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MQ_OK : MQ_ERR_CUDA; }

// The current device must be a B200 (compute capability 10.0).
inline mq_status check_device(DeviceInfo* di)
{
    if (device_info(di) != cudaSuccess) return MQ_ERR_CUDA;
    if (di->cc_major != 10 || di->cc_minor != 0) return MQ_ERR_DEVICE;
    return MQ_OK;
}

// An NVFP4 tensor view of the expected logical shape: non-null buffers,
// 16-byte aligned codes and scales, 4-byte aligned tensor scale.
inline mq_status check_nvfp4(const mq_nvfp4* t, int64_t rows, int64_t cols)
{
    if (t == nullptr || t->codes == nullptr || t->scales == nullptr || t->alpha == nullptr)
        return MQ_ERR_INVALID_ARG;
    if (t->rows != rows || t->cols != cols) return MQ_ERR_SHAPE;
    if (!aligned16(t->codes) || !aligned16(t->scales) || (reinterpret_cast<uintptr_t>(t->alpha) & 3u))
        return MQ_ERR_ALIGNMENT;
    return MQ_OK;
}

// Shapes of the prefill linear layer: activation [M, K], weight [N, K].
inline mq_status check_linear_shape(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || M > kMaxDim || K < 64 || K % 64 != 0 || N < 16 || N % 16 != 0) return MQ_ERR_SHAPE;
    if (N > kMaxDim || K > kMaxDim) return MQ_ERR_SHAPE;
    return MQ_OK;
}

}  // namespace mq
