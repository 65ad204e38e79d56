// gelu_mlp.cuh -- pieces of the fused GELU MLP (sm_100a): the DiT feed-forward
// block fc1 -> GELU -> fc2 with both linears SVDQ W4A4 nvfp4 layers, fused the
// way the "fused GELU kernel" of the Diffusers docs page "Nunchaku Lite"
// (section "Fused kernels", the GELU-MLP row) fuses it: fc1's GEMM epilogue
// applies GELU and performs fc2's activation step itself -- the nvfp4 codes
// and scales of h / lambda2 and the partial sums of fc2's rank-r
// down-projection h (L_down2 / lambda2) -- so the [M, N1] intermediate never
// goes to HBM.  The epilogue code lives in gemm_nvfp4_pair.cuh; this header
// holds what it shares with the stand-alone kernels of the unfused path:
//   * gelu_f32: the activation (exact erf form or the tanh form);
//   * gelu_bf16_kernel: the unfused activation pass, bf16 -> bf16;
//   * lowrank_finalize_kernel: turns the fp32 partial sums of the rank-r
//     down-projection into the hi/lo bf16 operand fc2's GEMM reads, and
//     zeroes the partial sums for the next call;
//   * the warp-level MMA and ldmatrix wrappers the epilogue uses for the
//     small [32 rows x 32 K] x [32 K x r] products of the down-projection.
#pragma once
#include "quantize.cuh"
#include "sm100_ptx.cuh"

namespace svdq {

// GELU in fp32.  approx = 0: x Phi(x) = 0.5 x erfc(-x / sqrt(2)) (erfc keeps
// the relative accuracy of the tail for negative x); approx = 1: the tanh
// form 0.5 x (1 + tanh(u)), u = sqrt(2/pi)(x + 0.044715 x^3), evaluated as
// x / (1 + e^(-2u)) for u >= 0 and x e^(2u) / (1 + e^(2u)) for u < 0: the
// same function without the cancellation of 1 + tanh(u) and without an
// exponential that overflows while the result is still a bf16 subnormal.
__device__ __forceinline__ float gelu_f32(float x, int approx) {
    if (approx == 0) return 0.5f * x * erfcf(-x * 0.70710678118654752f);
    const float u = 0.79788456080286536f * fmaf(0.044715f * x, x * x, x);
    const float e = expf(-2.0f * fabsf(u));   // in [0, 1]
    return u >= 0.0f ? x / (1.0f + e) : x * e / (1.0f + e);
}

// bf16 -> bf16 GELU as both the fused epilogue and the unfused pass compute
// it, so that the two hand fc2 the same h bit for bit.  The input has only
// 65536 values, and for most of them the result is a table entry:
//  * |x| in [2^-10, 16) (biased exponent 117 .. 130, both signs): a table of
//    bf16(gelu_f32(x)), 3584 entries (7 KB) built once per CTA;
//  * |x| < 2^-10: GELU(x) = x/2 + x^2/sqrt(2 pi) + O(x^4) (both forms), and
//    the x^2 term is below a quarter of a bf16 ulp of x/2, so the result is
//    bf16(x / 2) (computed in fp32: exact, then rounded to bf16);
//  * |x| >= 16: Phi(x) rounds to 1 (x > 0: the result is x) or x Phi(x)
//    underflows fp32 (x < 0: -0), for both forms, as gelu_f32 gives them.
constexpr int kGeluTabE0 = 117;                     // biased exponent of 2^-10
constexpr int kGeluTabNE = 14;                      // exponents 117 .. 130
constexpr int kGeluTabEntries = 2 * kGeluTabNE * 128;
constexpr int kGeluTabBytes = kGeluTabEntries * 2;

// Fills the table (threads tid, tid + nthreads, ...); the caller syncs.
__device__ __forceinline__ void gelu_table_fill(uint16_t* tab, int tid, int nthreads, int approx) {
    for (int i = tid; i < kGeluTabEntries; i += nthreads) {
        const uint32_t sign = (uint32_t)(i / (kGeluTabNE * 128));
        const uint32_t e = (uint32_t)kGeluTabE0 + (uint32_t)((i / 128) % kGeluTabNE);
        const uint32_t bits = (sign << 15) | (e << 7) | (uint32_t)(i & 127);
        tab[i] = __bfloat16_as_ushort(__float2bfloat16_rn(gelu_f32(__uint_as_float(bits << 16), approx)));
    }
}

// GELU of one bf16 (bits in the low 16 of b) -> bf16 bits.  The table holds
// the magnitudes 117 * 128 .. 131 * 128 - 1 (exponent and mantissa bits) of
// the positive values, then the same of the negative ones.
__device__ __forceinline__ uint32_t gelu_bf16_bits(uint32_t b, const uint16_t* tab) {
    constexpr uint32_t kSpan = (uint32_t)kGeluTabNE << 7;
    const uint32_t off = (b & 0x7FFFu) - ((uint32_t)kGeluTabE0 << 7);   // wraps below the table
    if (off < kSpan) return tab[off + ((b & 0x8000u) ? kSpan : 0u)];
    if (((b >> 7) & 0xFFu) < (uint32_t)kGeluTabE0)
        return __bfloat16_as_ushort(__float2bfloat16_rn(0.5f * __uint_as_float(b << 16)));
    return (b & 0x8000u) ? 0x8000u : b;
}

// The unfused activation pass: y[i] = bf16(GELU(x[i])) over n elements
// (eight per thread per step, grid-stride).
__global__ void __launch_bounds__(256) gelu_bf16_kernel(const __nv_bfloat16* __restrict__ x,
                                                        __nv_bfloat16* __restrict__ y, int64_t n, int approx) {
    __shared__ uint16_t tab[kGeluTabEntries];
    gelu_table_fill(tab, (int)threadIdx.x, (int)blockDim.x, approx);
    __syncthreads();
    const int64_t n8 = n / 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o[e] = gelu_bf16_bits(w[e] & 0xFFFFu, tab) | (gelu_bf16_bits(w[e] >> 16, tab) << 16);
        reinterpret_cast<uint4*>(y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (blockIdx.x == 0 && threadIdx.x < (unsigned)(n - 8 * n8)) {
        const int64_t i = 8 * n8 + threadIdx.x;
        y[i] = __ushort_as_bfloat16((uint16_t)gelu_bf16_bits(__bfloat16_as_ushort(x[i]), tab));
    }
}

// out[0][i] + out[1][i] = acc[i] / (S_x S_w) as a bf16 hi/lo pair (the form
// of the rank-r activations the GEMM reads), then acc[i] = 0.
__global__ void __launch_bounds__(256) lowrank_finalize_kernel(float* __restrict__ acc, int64_t count,
                                                               const float* __restrict__ x_scale,
                                                               const float* __restrict__ w_scale,
                                                               __nv_bfloat16* __restrict__ out) {
    griddep_wait();   // the partial sums come from the kernel ahead of this one
    const float inv_ss = __frcp_rn(__fmul_rn(*x_scale, *w_scale));
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
        __nv_bfloat16 hi, lo;
        split_bf16(__fmul_rn(acc[i], inv_ss), hi, lo);
        out[i] = hi;
        out[count + i] = lo;
        acc[i] = 0.0f;
    }
}

// Four 8x8 b16 matrices from shared memory (lane l gives the address of row
// l % 8 of matrix l / 8); d[i] is this lane's word of matrix i.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&d)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(addr));
}

// D[16x8] += A[16x16] B[16x8], bf16 operands, fp32 accumulators (warp-wide).
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

}  // namespace svdq
