// qkv_norm_rope.cuh -- per-head RMSNorm and rotary embedding of the Q and K
// columns of a fused to_qkv projection (sm_100a).
//
// The attention-input fusion of the original Nunchaku engine (the tutorial
// page's "structural rewrite" passage: one to_qkv projection, then norm_q /
// norm_k per head and apply_rotary_emb, as one fused operator; the Diffusers
// docs page "Nunchaku Lite", section "Fused kernels", "QKV+norm+RoPE").  For a
// row y of the projection, N = 3 H D columns (Q, K, V, head-major), each head
// of Q and of K becomes
//     v' = v / sqrt(mean(v^2) + eps) * w            (w: D weights, one set for Q, one for K)
//     out[2i] = v'[2i] cos_i - v'[2i+1] sin_i,  out[2i+1] = v'[2i+1] cos_i + v'[2i] sin_i
// with the token's rotary table (cos_i, sin_i), i < D/2; V passes through.
//
// Two forms:
//  * the GEMM epilogue (gemm_nvfp4_pair.cuh) applies it to the fp32
//    accumulator before the single bf16 rounding (D = 128: one head per
//    epilogue warp's 128 columns);
//  * qkv_norm_rope_kernel applies it to a bf16 y already in memory (the unfused
//    path: projection, then this kernel), one warp per (row, head).
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {

// One warp per (row, Q or K head) of a bf16 [M, 3 H D] tensor, D == 128:
// lane l owns columns 4l .. 4l + 3 (rotary pairs 2l and 2l + 1).
__global__ void __launch_bounds__(256)
    qkv_norm_rope_kernel(const __nv_bfloat16* __restrict__ y_in, __nv_bfloat16* __restrict__ y_out, int64_t M,
                         int H, const __nv_bfloat16* __restrict__ wq, const __nv_bfloat16* __restrict__ wk, float eps,
                         const float* __restrict__ cosv, const float* __restrict__ sinv) {
    constexpr int D = 128;
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = (int)(threadIdx.x & 31u);
    const int64_t per_row = 2 * (int64_t)H;
    if (wid >= M * per_row) return;
    const int64_t m = wid / per_row;
    const int hh = (int)(wid - m * per_row);          // 0..H-1: Q heads, H..2H-1: K heads
    const __nv_bfloat16* w = hh < H ? wq : wk;
    const int64_t N = 3 * (int64_t)H * D;
    const int64_t off = m * N + (int64_t)hh * D + 4 * lane;
    const uint2 raw = *reinterpret_cast<const uint2*>(y_in + off);
    float v[4] = {bf16lo_to_f32(raw.x), bf16hi_to_f32(raw.x), bf16lo_to_f32(raw.y), bf16hi_to_f32(raw.y)};
    float ss = v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss * (1.0f / D) + eps);
    const uint2 wr = __ldg(reinterpret_cast<const uint2*>(w + 4 * lane));
    const float wv[4] = {bf16lo_to_f32(wr.x), bf16hi_to_f32(wr.x), bf16lo_to_f32(wr.y), bf16hi_to_f32(wr.y)};
    const float2 c = __ldg(reinterpret_cast<const float2*>(cosv + m * (D / 2) + 2 * lane));
    const float2 s = __ldg(reinterpret_cast<const float2*>(sinv + m * (D / 2) + 2 * lane));
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = v[i] * r * wv[i];
    const float o0 = v[0] * c.x - v[1] * s.x, o1 = v[1] * c.x + v[0] * s.x;
    const float o2 = v[2] * c.y - v[3] * s.y, o3 = v[3] * c.y + v[2] * s.y;
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(o0, o1), p1 = __floats2bfloat162_rn(o2, o3);
    *reinterpret_cast<uint2*>(y_out + off) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1));
}

// V columns of the unfused path when writing out of place: a plain copy.
__global__ void __launch_bounds__(256) copy_v_kernel(const __nv_bfloat16* __restrict__ y_in,
                                                     __nv_bfloat16* __restrict__ y_out, int64_t M, int H) {
    constexpr int D = 128;
    const int64_t hd = (int64_t)H * D;                 // V columns per row
    const int64_t n8 = M * hd / 8;                     // 16-byte pieces
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = (i * 8) / hd, c = (i * 8) - m * hd;
        const int64_t off = m * 3 * hd + 2 * hd + c;
        *reinterpret_cast<uint4*>(y_out + off) = *reinterpret_cast<const uint4*>(y_in + off);
    }
}

}  // namespace svdq
