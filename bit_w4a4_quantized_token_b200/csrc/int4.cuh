// int4.cuh -- GEMM of the INT4 W4A4 variant (group 64, bf16 scales).
// Placeholder: the int4 GEMM kernel is not built yet.
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {

inline cudaError_t int4_prepare_device() { return cudaSuccess; }

inline svdq_status int4_gemm(const void*, const void*, int64_t, const void*, const void*, int64_t, int64_t,
                             const void*, const void*, int, const void*, void*, cudaStream_t) {
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace svdq
