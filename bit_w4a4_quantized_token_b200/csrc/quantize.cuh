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
    const int64_t nvec = rows * K / 8;
    float m = 0.0f;
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < nvec;
         v += (int64_t)gridDim.x * blockDim.x) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(x) + v);
        const int64_t k0 = (v * 8) % K;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float a0 = bf16lo_to_f32(ws[q]), a1 = bf16hi_to_f32(ws[q]);
            if (inv_lambda) {
                a0 = __fmul_rn(a0, __ldg(inv_lambda + k0 + 2 * q));
                a1 = __fmul_rn(a1, __ldg(inv_lambda + k0 + 2 * q + 1));
            }
            m = fmaxf(m, fmaxf(fabsf(a0), fabsf(a1)));
        }
    }
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

// ------------------------------------------------- activation quantizer
namespace qa {
constexpr int kRows = 128;              // rows per CTA (= TMEM lanes)
constexpr int kCols = 64;               // columns per pipeline stage (128 B of bf16)
constexpr int kXBytes = kRows * kCols * 2;
constexpr int kThreads = 192;           // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 quantize
constexpr int kMaxStages = 8;
}  // namespace qa

struct QuantActArgs {
    const float* inv_lambda;   // [K]
    const float* x_scale;      // S_x (nvfp4)
    const float* w_scale;      // S_w (nvfp4 with rank > 0)
    uint8_t* x_codes;          // [M, K/2]
    uint8_t* x_scales;         // nvfp4: scale-factor layout; int4: bf16 [K/64, rows_pad]
    __nv_bfloat16* lowrank;    // [2, M, rank]: hi and lo bf16 parts
    int M, K, rank;
    int rows_pad;              // M rounded up to 128
    int chunks;                // K / 64
    int cluster;               // CTAs of one cluster split K for one 128-row block
    int stages;
    uint32_t stage_bytes;      // 16 KB x tile + two L_down_t tiles (hi, lo: rank x 128 B each)
    uint32_t tmem_cols;
};


__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_smem_addr, uint32_t cta_rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_smem_addr), "r"(cta_rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

enum : uint32_t { kSiteQaEmpty = 1, kSiteQaFullMma = 2, kSiteQaFullWork = 3, kSiteQaAcc = 4, kSiteQaDrain = 5 };

constexpr int kPrecNvfp4 = 0, kPrecInt4 = 1;

// Grid (cluster, ceil(M/128)); cluster dims (cluster, 1, 1).  CTA `q` of a
// cluster handles chunks [q*T/c, (q+1)*T/c) of the T = K/64 column chunks of
// its 128-row block; the clusters' partial rank-r sums are reduced through
// distributed shared memory in a fixed order (deterministic).  The rank-r
// down-projection runs on the tensor cores: x (bf16, exact) times the hi and
// lo bf16 parts of L_down / lambda, fp32 accumulate in TMEM.
template <int PREC>
__global__ void __launch_bounds__(qa::kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_ld,
                        QuantActArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nst = a.stages;
    float* invl = reinterpret_cast<float*>(smem + (size_t)nst * a.stage_bytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(invl + qa::kMaxStages * qa::kCols);
    uint64_t* empty = full + qa::kMaxStages;
    uint64_t* accb = empty + qa::kMaxStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accb + 1);
    __shared__ int s_issued, s_failed;

    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t crank = (a.cluster > 1) ? cluster_ctarank() : 0u;
    const int m0 = blockIdx.y * qa::kRows;
    const int c_lo = (int)((int64_t)a.chunks * crank / a.cluster);
    const int c_hi = (int)((int64_t)a.chunks * (crank + 1) / a.cluster);
    const int n_it = c_hi - c_lo;
    const bool has_lr = a.rank > 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4u + (has_lr ? 1u : 0u));
        }
        mbar_init(accb, 1);
        s_issued = 0;
        s_failed = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_x);
        if (has_lr) prefetch_tensormap(&tm_ld);
    }
    if (warp == 1 && has_lr) {
        tmem_alloc(tmem_slot, a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = has_lr ? *tmem_slot : 0u;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            const uint32_t ld_tile = (uint32_t)a.rank * 128u;
            const uint32_t bytes = qa::kXBytes + (has_lr ? 2u * ld_tile : 0u) + qa::kCols * 4u;
            int it = 0;
            for (; it < n_it; ++it) {
                const int s = it % nst;
                const uint32_t ph = (uint32_t)(it / nst) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, kSiteQaEmpty)) {
                    s_failed = 1;
                    break;
                }
                const int kc = c_lo + it;
                uint8_t* st = smem + (size_t)s * a.stage_bytes;
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(st, &tm_x, &full[s], kc * qa::kCols, m0);
                if (has_lr) {
                    tma_load_3d(st + qa::kXBytes, &tm_ld, &full[s], kc * qa::kCols, 0, 0);
                    tma_load_3d(st + qa::kXBytes + ld_tile, &tm_ld, &full[s], kc * qa::kCols, 0, 1);
                }
                bulk_load(invl + s * qa::kCols, a.inv_lambda + (int64_t)kc * qa::kCols, qa::kCols * 4, &full[s]);
            }
            s_issued = it;
        }
    } else if (warp == 1) {
        // --------------------------------------------------- rank-r MMA issuer
        if (has_lr && lane == 0) {
            const uint32_t idesc = idesc_bf16_f32((uint32_t)a.rank);
            bool ok = true;
            for (int it = 0; it < n_it; ++it) {
                const int s = it % nst;
                const uint32_t ph = (uint32_t)(it / nst) & 1u;
                if (!mbar_wait(&full[s], ph, kSiteQaFullMma)) {
                    ok = false;
                    s_failed = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t xa = smem_u32(smem + (size_t)s * a.stage_bytes);
                const uint32_t lb = xa + qa::kXBytes;
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16(tmem, desc_sw128(xa + 32u * j),
                                 desc_sw128(lb + (uint32_t)part * (uint32_t)a.rank * 128u + 32u * j), idesc,
                                 (it > 0 || part > 0 || j > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(accb);
        }
    } else {
        // --------------------------------------------------------- quantizers
        const uint32_t q = warp & 3u;
        const int row = (int)(32u * q + lane);
        const int64_t grow = (int64_t)m0 + row;
        float S = 1.0f, six_s = 6.0f;
        if (PREC == kPrecNvfp4) {
            S = *a.x_scale;
            six_s = __fmul_rn(6.0f, S);
        }
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int s = it % nst;
            const uint32_t ph = (uint32_t)(it / nst) & 1u;
            if (!mbar_wait(&full[s], ph, kSiteQaFullWork)) {
                ok = false;
                s_failed = 1;
                break;
            }
            const uint8_t* xr = smem + (size_t)s * a.stage_bytes + row * 128;
            uint4 raw[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) raw[c] = *reinterpret_cast<const uint4*>(xr + ((c ^ (row & 7)) << 4));
            float v[64];
            const float4* ilp = reinterpret_cast<const float4*>(invl + s * qa::kCols);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 l0 = ilp[2 * c], l1 = ilp[2 * c + 1];
                const uint32_t ws[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
                v[8 * c + 0] = __fmul_rn(bf16lo_to_f32(ws[0]), l0.x);
                v[8 * c + 1] = __fmul_rn(bf16hi_to_f32(ws[0]), l0.y);
                v[8 * c + 2] = __fmul_rn(bf16lo_to_f32(ws[1]), l0.z);
                v[8 * c + 3] = __fmul_rn(bf16hi_to_f32(ws[1]), l0.w);
                v[8 * c + 4] = __fmul_rn(bf16lo_to_f32(ws[2]), l1.x);
                v[8 * c + 5] = __fmul_rn(bf16hi_to_f32(ws[2]), l1.y);
                v[8 * c + 6] = __fmul_rn(bf16lo_to_f32(ws[3]), l1.z);
                v[8 * c + 7] = __fmul_rn(bf16hi_to_f32(ws[3]), l1.w);
            }
            const int kc = c_lo + it;
            uint32_t cw[8];
            if (PREC == kPrecNvfp4) {
                uint32_t scw = 0;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float vg[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) vg[i] = v[16 * g + i];
                    scw |= quant_group16(vg, S, six_s, cw[2 * g], cw[2 * g + 1]) << (8 * g);
                }
                *reinterpret_cast<uint32_t*>(a.x_scales + sf_offset(grow, (int64_t)kc * 4, a.chunks)) = scw;
            } else {
                const uint32_t sb = quant_group64_int4(v, cw);
                reinterpret_cast<uint16_t*>(a.x_scales)[(int64_t)kc * a.rows_pad + grow] = (uint16_t)sb;
            }
            if (grow < a.M) {
                uint4* dst = reinterpret_cast<uint4*>(a.x_codes + grow * (int64_t)(a.K / 2) + (int64_t)kc * 32);
                dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
            }
            // release the stage only after its data has been consumed
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (has_lr) {
            // partial rank-r sums of this CTA -> shared memory (reusing the stages)
            if (ok && !mbar_wait(accb, 0, kSiteQaAcc)) {
                ok = false;
                s_failed = 1;
            }
            tc_fence_after();
            named_bar_sync(1, 128);   // every quantizer warp is done with the stage buffers
            float* red = reinterpret_cast<float*>(smem);
            const int rs = a.rank + 1;  // padded row stride: conflict-free stores
            for (int c0 = 0; c0 < a.rank; c0 += 16) {
                uint32_t r16[16];
                tmem_ld_32x32b_x16(tmem + ((32u * q) << 16) + (uint32_t)c0, r16);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) red[row * rs + c0 + i] = ok ? __uint_as_float(r16[i]) : 0.0f;
            }
        }
    }

    __syncthreads();
    if (has_lr) {
        if (a.cluster > 1) cluster_sync_all();
        if (warp >= 2) {
            // reduce this CTA's slice of rows over the cluster, in rank order
            const float ss = (PREC == kPrecNvfp4) ? __fmul_rn(*a.x_scale, *a.w_scale) : 1.0f;
            const int64_t plane = (int64_t)a.M * a.rank;
            const float* red = reinterpret_cast<const float*>(smem);
            const int rs = a.rank + 1;
            const int rows_per = qa::kRows / a.cluster;
            const int r0 = (int)crank * rows_per;
            const int total = rows_per * a.rank;
            for (int e = (int)threadIdx.x - 64; e < total; e += 128) {
                const int rr = r0 + e / a.rank, j = e % a.rank;
                const uint32_t la = smem_u32(red + rr * rs + j);
                float sum = 0.0f;
                if (a.cluster > 1) {
                    for (int p = 0; p < a.cluster; ++p) sum += ld_cluster_f32(la, (uint32_t)p);
                } else {
                    sum = red[rr * rs + j];
                }
                const int64_t gm = (int64_t)m0 + rr;
                if (gm < a.M) {
                    __nv_bfloat16 hi, lo;
                    split_bf16(PREC == kPrecNvfp4 ? __fdiv_rn(sum, ss) : sum, hi, lo);
                    a.lowrank[gm * a.rank + j] = hi;
                    a.lowrank[plane + gm * a.rank + j] = lo;
                }
            }
        }
        if (a.cluster > 1) cluster_sync_all();
    }
    // on a timeout, let the copies already issued land before the CTA exits
    if (s_failed && warp == 0 && lane == 0) {
        const int issued = s_issued;
        for (int it = (issued > nst ? issued - nst : 0); it < issued; ++it)
            mbar_wait(&full[it % nst], (uint32_t)(it / nst) & 1u, kSiteQaDrain);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && has_lr) {
        tc_fence_after();
        tmem_dealloc(tmem, a.tmem_cols);
    }
}

}  // namespace svdq
