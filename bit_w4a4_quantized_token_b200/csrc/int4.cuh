// int4.cuh -- INT4 W4A4 variant of the SVDQ layer (group 64, bf16 scales).
// Placeholder entry points: the int4 kernels are not built yet.
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {

inline cudaError_t int4_prepare_device() { return cudaSuccess; }

inline svdq_status int4_quantize_rows(const void*, const float*, int64_t, int64_t, void*, void*, cudaStream_t) {
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
}
inline svdq_status int4_quantize_act(const void*, int64_t, int64_t, const float*, const void*, int, void*, void*,
                                     void*, cudaStream_t) {
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
}
inline svdq_status int4_gemm(const void*, const void*, int64_t, const void*, const void*, int64_t, int64_t,
                             const void*, const void*, int, const void*, void*, cudaStream_t) {
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace svdq
