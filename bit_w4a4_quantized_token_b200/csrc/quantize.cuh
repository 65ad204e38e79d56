// quantize.cuh -- the quantizers of the SVDQ W4A4 layer (sm_100a).
//
//  * the NVFP4 tensor-scale pre-pass (amax, then S = amax / 2688),
//  * the weight packer (R -> 4-bit codes + group scales; 1/lambda folded into
//    L_down as an fp32 value carried by a bf16 hi/lo pair, L_up transposed),
//  * the activation quantizer fused with the rank-r down-projection
//    (x/lambda -> codes + scales, and (x/lambda) . L_down on the tensor cores
//    from the same shared-memory tile), for nvfp4 and int4.
//
// Group rule (Diffusers docs "Nunchaku Lite", "Supported quantization types":
// nvfp4, group 16): for a group of 16 smoothed values v with a = max|v|,
//   e   = E4M3(a / (6 S))          one UE4M3 scale per group, nearest-even
//   dec = e * S
//   q_i = E2M1(v_i * (1 / dec))    nearest-even, saturating at 6
// with every product, quotient and reciprocal a single IEEE fp32 operation
// rounded to nearest (no FMA contraction), and inv = 0 when dec == 0.
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {

// Byte offset of the scale of (row r, group g) in the tensor-core scale layout
// (512-byte blocks of 128 rows x 4 groups; kg4 = K / 64 blocks per 128 rows).
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t g, int64_t kg4) {
    return ((r >> 7) * kg4 + (g >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (g & 3);
}

// One group of 16: returns the scale byte, writes the 16 codes as two words.
__device__ __forceinline__ uint32_t quant_group16(const float (&v)[16], float S, float six_s, uint32_t& lo,
                                                  uint32_t& hi) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t eb = cvt_e4m3(__fdiv_rn(amax, six_s));
    const float dec = __fmul_rn(e4m3_to_f32(eb), S);
    const float inv = (dec == 0.0f) ? 0.0f : __frcp_rn(dec);
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[i], inv);
    lo = cvt_e2m1x8(q);
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(v[8 + i], inv);
    hi = cvt_e2m1x8(q);
    return eb;
}

// Splits v into hi = bf16(v) and lo = bf16(v - hi): hi + lo carries v to
// about 2^-17 relative, so two bf16 MMAs reproduce an fp32 operand.
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
    hi = __float2bfloat16_rn(v);
    lo = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
}

// int4 group of 64 (Diffusers docs "Nunchaku Lite", "Supported quantization
// types": int4, group 64): s = bf16(a / 7), q = clamp(rint(v * (1/s)), -8, 7).
// Returns the bf16 scale bits; codes as eight words of two's-complement nibbles.
__device__ __forceinline__ uint32_t quant_group64_int4(const float (&v)[64], uint32_t (&cw)[8]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
    const float sf = __bfloat162float(sb);
    const float inv = (sf == 0.0f) ? 0.0f : __frcp_rn(sf);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int q = __float2int_rn(__fmul_rn(v[8 * w + i], inv));
            q = max(-8, min(7, q));
            word |= ((uint32_t)q & 15u) << (4 * i);
        }
        cw[w] = word;
    }
    return (uint32_t)__bfloat16_as_ushort(sb);
}

// ---------------------------------------------------------------- pre-pass
// amax over v = x (inv_lambda == nullptr) or v = fl32(x * inv_lambda[k]);
// the result's bits are atomically max-ed into *out (non-negative floats
// order like their bit patterns).  *out must be zeroed first.
__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                   const float* __restrict__ inv_lambda, int64_t rows, int64_t K,
                                                   unsigned int* out) {
    const int64_t nvec = rows * K / 8;   // 16-byte vectors of 8 values, grid-stride
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t kv = K / 8;            // vectors per row (K % 64 == 0)
    const int64_t dk = stride % kv;      // how far the column advances per stride
    int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t col = v % kv;                // the vector's column position, kept without a division per step
    float m = 0.0f;
    // |v_i| of 8 values starting at column 8 c, with v = x / lambda when given
    auto fold = [&](const uint4 w, int64_t c) {
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        float4 l0 = make_float4(1.0f, 1.0f, 1.0f, 1.0f), l1 = l0;
        if (inv_lambda) {
            l0 = __ldg(reinterpret_cast<const float4*>(inv_lambda) + 2 * c);
            l1 = __ldg(reinterpret_cast<const float4*>(inv_lambda) + 2 * c + 1);
        }
        const float il[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float a0 = bf16lo_to_f32(ws[q]), a1 = bf16hi_to_f32(ws[q]);
            if (inv_lambda) {
                a0 = __fmul_rn(a0, il[2 * q]);
                a1 = __fmul_rn(a1, il[2 * q + 1]);
            }
            m = fmaxf(m, fmaxf(fabsf(a0), fabsf(a1)));
        }
    };
    // two vectors in flight per thread
    for (; v + stride < nvec; v += 2 * stride) {
        int64_t col2 = col + dk;
        if (col2 >= kv) col2 -= kv;
        const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(x) + v);
        const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(x) + v + stride);
        fold(w0, col);
        fold(w1, col2);
        col = col2 + dk;
        if (col >= kv) col -= kv;
    }
    if (v < nvec) fold(__ldg(reinterpret_cast<const uint4*>(x) + v), col);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
        atomicMax(out, __float_as_uint(m));
    }
}

// S = fl32(amax / 2688) in place; an all-zero tensor gets S = 1.
__global__ void finalize_tensor_scale_kernel(float* s) {
    const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(s));
    float S = __fdiv_rn(amax, 2688.0f);
    if (!(S > 0.0f)) S = 1.0f;
    *s = S;
}

// -------------------------------------------------------- weight packing
// One thread per (row, group of 16) over rows_pad rows; rows >= `rows` only
// write zero scale bytes (the padding of the scale layout).
__global__ void __launch_bounds__(256) quantize_rows_nvfp4_kernel(const __nv_bfloat16* __restrict__ R, int64_t rows,
                                                                  int64_t rows_pad, int64_t K,
                                                                  const float* __restrict__ S_ptr,
                                                                  uint8_t* __restrict__ codes,
                                                                  uint8_t* __restrict__ scales) {
    const int64_t kg = K / 16;
    const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (gid >= rows_pad * kg) return;
    const int64_t r = gid / kg, g = gid % kg;
    uint32_t eb = 0;
    if (r < rows) {
        const float S = *S_ptr;
        const float six_s = __fmul_rn(6.0f, S);
        const uint4* src = reinterpret_cast<const uint4*>(R + r * K + g * 16);
        const uint4 w0 = __ldg(src), w1 = __ldg(src + 1);
        const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        float v[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            v[2 * q] = bf16lo_to_f32(ws[q]);
            v[2 * q + 1] = bf16hi_to_f32(ws[q]);
        }
        uint32_t lo, hi;
        eb = quant_group16(v, S, six_s, lo, hi);
        *reinterpret_cast<uint2*>(codes + r * (K / 2) + g * 8) = make_uint2(lo, hi);
    }
    scales[sf_offset(r, g, K / 64)] = (uint8_t)eb;
}

// int4 weight packing: one thread per (row, group of 64) over rows_pad rows;
// the bf16 scales are group-major (scales[g * rows_pad + r]).
__global__ void __launch_bounds__(256) quantize_rows_int4_kernel(const __nv_bfloat16* __restrict__ R, int64_t rows,
                                                                 int64_t rows_pad, int64_t K,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint16_t* __restrict__ scales) {
    const int64_t kg = K / 64;
    const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (gid >= rows_pad * kg) return;
    const int64_t r = gid % rows_pad, g = gid / rows_pad;   // consecutive threads: consecutive rows
    uint32_t sb = 0;
    if (r < rows) {
        const uint4* src = reinterpret_cast<const uint4*>(R + r * K + g * 64);
        float v[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 w = __ldg(src + c);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                v[8 * c + 2 * p] = bf16lo_to_f32(ws[p]);
                v[8 * c + 2 * p + 1] = bf16hi_to_f32(ws[p]);
            }
        }
        uint32_t cw[8];
        sb = quant_group64_int4(v, cw);
        uint4* dst = reinterpret_cast<uint4*>(codes + r * (K / 2) + g * 32);
        dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    }
    scales[g * rows_pad + r] = (uint16_t)sb;
}

// inv_lambda = 1/lambda; with v = fl32(L_down[k, j] / lambda[k]):
// L_down_t[0, j, k] = bf16(v) and L_down_t[1, j, k] = bf16(v - bf16(v));
// L_up_t[n, j] = L_up[j, n].
__global__ void __launch_bounds__(256) fold_lowrank_kernel(const float* __restrict__ lambda,
                                                           const __nv_bfloat16* __restrict__ L_down,
                                                           const __nv_bfloat16* __restrict__ L_up, int64_t K,
                                                           int64_t N, int rank, float* __restrict__ inv_lambda,
                                                           __nv_bfloat16* __restrict__ L_down_t,
                                                           __nv_bfloat16* __restrict__ L_up_t) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t t0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    for (int64_t k = t0; k < K; k += stride) inv_lambda[k] = __frcp_rn(lambda[k]);
    for (int64_t i = t0; i < K * rank; i += stride) {  // i = j * K + k (coalesced stores)
        const int64_t j = i / K, k = i % K;
        const float v = __fdiv_rn(__bfloat162float(L_down[k * rank + j]), lambda[k]);
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        L_down_t[i] = hi;
        L_down_t[K * rank + i] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
    }
    for (int64_t i = t0; i < N * rank; i += stride) {  // i = n * rank + j
        const int64_t n = i / rank, j = i % rank;
        L_up_t[i] = L_up[j * N + n];
    }
}

}  // namespace svdq
