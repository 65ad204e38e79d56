// quantize_act.cuh -- activation quantizer of the SVDQ W4A4 layer, fused with
// the rank-r down-projection (sm_100a).
//
// One CTA owns a 128-row block of x and a contiguous range of 64-column
// chunks.  Three producer warps (0, 2, 3; chunks taken in turn, since one
// issuing thread cannot stream fast enough) load each chunk -- a 128 x 64
// bf16 tile, 128-byte swizzled -- and the matching hi/lo tiles of
// L_down / lambda into a ring of shared-memory stages with TMA; 1/lambda for
// the CTA's columns is loaded once.  Sixteen quantizer warps (4..19) turn the
// tile into 4-bit codes and group scales (one thread per row and group of 16
// columns).  Warp 1 issues tcgen05.mma on the same tile: x (bf16, exact)
// times the hi and lo parts of L_down / lambda, fp32 in TMEM.
// When K is split over several CTAs, each writes its fp32 partial of the
// rank-r product to a workspace and the last CTA of the row block (found with
// a counter it resets afterwards) adds the partials in split order, so the
// result does not depend on timing.
#pragma once
#include "quantize.cuh"
#include "sm100_ptx.cuh"

namespace svdq {
namespace qa {
constexpr int kRows = 128;              // rows per CTA (= TMEM lanes of the MMA)
constexpr int kCols = 64;               // columns per stage (128 B of bf16)
constexpr int kXBytes = kRows * kCols * 2;
constexpr int kWorkerWarps = 16;
constexpr int kWorker0 = 4;             // first quantizer warp (a multiple of 4: TMEM lane quadrants)
constexpr int kProducers = 3;           // warps 0, 2, 3
constexpr int kThreads = 32 * (kWorker0 + kWorkerWarps);   // warp 1: MMA + TMEM
constexpr int kMaxStages = 8;
constexpr int kMaxSplits = 16;
constexpr int kSplitTarget = 148;       // CTAs wanted for one wave (SMs of a B200)
}  // namespace qa

constexpr int kPrecNvfp4 = 0, kPrecInt4 = 1;

struct QuantActArgs {
    const float* inv_lambda;   // [K]
    const float* x_scale;      // S_x (nvfp4)
    const float* w_scale;      // S_w (nvfp4 with rank > 0)
    uint8_t* x_codes;          // [M, K/2]
    uint8_t* x_scales;         // nvfp4: scale-factor layout; int4: bf16 [K/64, rows_pad]
    __nv_bfloat16* lowrank;    // [2, M, rank]: hi and lo bf16 planes
    float* partials;           // [row_blocks, splits, 128, rank] fp32 (splits > 1)
    unsigned int* counters;    // [row_blocks] (splits > 1); zero between calls
    int M, K, rank;
    int rows_pad;              // M rounded up to 128
    int chunks;                // K / 64
    int splits;                // CTAs sharing one 128-row block
    int stages;
    int max_chunks;            // ceil(chunks / splits): 1/lambda values kept in shared memory / 64
    uint32_t stage_bytes;      // x tile + hi and lo L_down_t tiles (rank x 128 B each)
    uint32_t tmem_cols;
};

enum : uint32_t { kSiteQaEmpty = 1, kSiteQaFullMma = 2, kSiteQaFullWork = 3, kSiteQaAcc = 4, kSiteQaDrain = 5 };

// Writes `n` rank-r values of one row: L' = v / ss as a bf16 hi/lo pair
// (`dst` points at column 0 of the chunk in the hi plane).
__device__ __forceinline__ void store_lowrank_row(__nv_bfloat16* dst, int64_t plane, int64_t grow, int rank,
                                                  const float* v, int n, float ss, bool scaled) {
    for (int j = 0; j < n; j += 2) {
        __nv_bfloat16 h0, l0, h1, l1;
        split_bf16(scaled ? __fdiv_rn(v[j], ss) : v[j], h0, l0);
        split_bf16(scaled ? __fdiv_rn(v[j + 1], ss) : v[j + 1], h1, l1);
        *reinterpret_cast<__nv_bfloat162*>(dst + grow * rank + j) = __halves2bfloat162(h0, h1);
        *reinterpret_cast<__nv_bfloat162*>(dst + plane + grow * rank + j) = __halves2bfloat162(l0, l1);
    }
}

// Grid (splits, ceil(M/128)).  CTA (s, b) handles rows [128b, 128b+128) and
// chunks [s*T/splits, (s+1)*T/splits) of the T = K/64 column chunks.
template <int PREC>
__global__ void __launch_bounds__(qa::kThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_ld,
                        QuantActArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nst = a.stages;
    float* invl = reinterpret_cast<float*>(smem + (size_t)nst * a.stage_bytes);   // [max_chunks * 64]
    float* inv_tab = invl + a.max_chunks * qa::kCols;                              // [128] 1/(e*S)
    uint64_t* full = reinterpret_cast<uint64_t*>(inv_tab + 128);
    uint64_t* empty = full + qa::kMaxStages;
    uint64_t* accb = empty + qa::kMaxStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accb + 1);
    __shared__ int s_failed, s_last;
    __shared__ int s_issued[qa::kMaxStages];   // loads issued into each stage (phases started)

    const uint32_t warp = warp_id(), lane = lane_id();
    const int split = blockIdx.x, rb = blockIdx.y;
    const int m0 = rb * qa::kRows;
    const int c_lo = (int)((int64_t)a.chunks * split / a.splits);
    const int c_hi = (int)((int64_t)a.chunks * (split + 1) / a.splits);
    const int n_it = c_hi - c_lo;
    const bool has_lr = a.rank > 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], qa::kWorkerWarps + (has_lr ? 1u : 0u));   // quantizer warps + MMA commit
        }
        mbar_init(accb, 1);
        for (int s = 0; s < qa::kMaxStages; ++s) s_issued[s] = 0;
        s_failed = 0;
        s_last = 0;
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
    if (warp >= (uint32_t)qa::kWorker0) {
        const int t = (int)threadIdx.x - 32 * qa::kWorker0;
        // 1/lambda for this CTA's columns, once
        const float4* src = reinterpret_cast<const float4*>(a.inv_lambda + (int64_t)c_lo * qa::kCols);
        for (int i = t; i < n_it * (qa::kCols / 4); i += 32 * qa::kWorkerWarps)
            reinterpret_cast<float4*>(invl)[i] = __ldg(src + i);
        if (PREC == kPrecNvfp4 && t < 128) {
            // reciprocals of the 128 possible decoded group scales e * S
            const float dec = __fmul_rn(e4m3_to_f32((uint32_t)t), *a.x_scale);
            inv_tab[t] = (dec == 0.0f) ? 0.0f : __frcp_rn(dec);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = has_lr ? *tmem_slot : 0u;

    if (warp == 0 || warp == 2 || warp == 3) {
        // ---------------------------------------------------------- producers
        if (lane == 0) {
            const int pid = warp == 0 ? 0 : (int)warp - 1;     // 0, 1, 2
            const uint32_t bytes = qa::kXBytes + (has_lr ? 2u * (uint32_t)a.rank * 128u : 0u);
            int it = pid;
            for (; it < n_it; it += qa::kProducers) {
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
                if (has_lr) tma_load_3d(st + qa::kXBytes, &tm_ld, &full[s], kc * qa::kCols, 0, 0);   // hi and lo
                // a stage is refilled only after its previous load was consumed: no concurrent updates
                reinterpret_cast<volatile int*>(s_issued)[s] += 1;
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- rank-r MMA issuer
        if (has_lr && lane == 0) {
            // B = the hi and lo tiles stacked (2r rows): one MMA per k-step when
            // 2r <= 256, with hi and lo accumulated in separate column ranges
            const bool fused = 2 * a.rank <= 256;
            const uint32_t idesc = idesc_bf16_f32((uint32_t)(fused ? 2 * a.rank : a.rank));
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
                if (fused) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16(tmem, desc_sw128(xa + 32u * j), desc_sw128(lb + 32u * j), idesc,
                                 (it > 0 || j > 0) ? 1u : 0u);
                } else {
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16(tmem + (uint32_t)part * (uint32_t)a.rank, desc_sw128(xa + 32u * j),
                                     desc_sw128(lb + (uint32_t)part * (uint32_t)a.rank * 128u + 32u * j), idesc,
                                     (it > 0 || j > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(accb);
        }
    } else if (warp >= (uint32_t)qa::kWorker0) {
        // --------------------------------------------------------- quantizers
        const int t = (int)threadIdx.x - 32 * qa::kWorker0;
        const int row = t >> 2, g = t & 3;            // 4 lanes per row: one group of 16 columns each
        const int64_t grow = (int64_t)m0 + row;
        float S = 1.0f, six_s = 6.0f;
        if (PREC == kPrecNvfp4) {
            S = *a.x_scale;
            six_s = __fmul_rn(6.0f, S);
        }
        for (int it = 0; it < n_it; ++it) {
            const int s = it % nst;
            const uint32_t ph = (uint32_t)(it / nst) & 1u;
            if (!mbar_wait(&full[s], ph, kSiteQaFullWork)) {
                s_failed = 1;
                break;
            }
            const uint8_t* xr = smem + (size_t)s * a.stage_bytes + row * 128;
            const uint4 r0 = *reinterpret_cast<const uint4*>(xr + (((2 * g) ^ (row & 7)) << 4));
            const uint4 r1 = *reinterpret_cast<const uint4*>(xr + (((2 * g + 1) ^ (row & 7)) << 4));
            const float4* il = reinterpret_cast<const float4*>(invl + it * qa::kCols + 16 * g);
            const float4 l0 = il[0], l1 = il[1], l2 = il[2], l3 = il[3];
            float v[16];
            fmul2_rn(bf16lo_to_f32(r0.x), bf16hi_to_f32(r0.x), l0.x, l0.y, v[0], v[1]);
            fmul2_rn(bf16lo_to_f32(r0.y), bf16hi_to_f32(r0.y), l0.z, l0.w, v[2], v[3]);
            fmul2_rn(bf16lo_to_f32(r0.z), bf16hi_to_f32(r0.z), l1.x, l1.y, v[4], v[5]);
            fmul2_rn(bf16lo_to_f32(r0.w), bf16hi_to_f32(r0.w), l1.z, l1.w, v[6], v[7]);
            fmul2_rn(bf16lo_to_f32(r1.x), bf16hi_to_f32(r1.x), l2.x, l2.y, v[8], v[9]);
            fmul2_rn(bf16lo_to_f32(r1.y), bf16hi_to_f32(r1.y), l2.z, l2.w, v[10], v[11]);
            fmul2_rn(bf16lo_to_f32(r1.z), bf16hi_to_f32(r1.z), l3.x, l3.y, v[12], v[13]);
            fmul2_rn(bf16lo_to_f32(r1.w), bf16hi_to_f32(r1.w), l3.z, l3.w, v[14], v[15]);
            const int kc = c_lo + it;
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
            uint32_t c0, c1;
            if (PREC == kPrecNvfp4) {
                const uint32_t eb = cvt_e4m3(__fdiv_rn(amax, six_s));
                const float inv = inv_tab[eb];
                float q[8];
#pragma unroll
                for (int i = 0; i < 8; i += 2) fmul2_rn(v[i], v[i + 1], inv, inv, q[i], q[i + 1]);
                c0 = cvt_e2m1x8(q);
#pragma unroll
                for (int i = 0; i < 8; i += 2) fmul2_rn(v[8 + i], v[9 + i], inv, inv, q[i], q[i + 1]);
                c1 = cvt_e2m1x8(q);
                // the four scale bytes of this row's chunk are adjacent: gather them in lane g == 0
                const uint32_t b1 = __shfl_down_sync(0xffffffffu, eb, 1);
                const uint32_t b2 = __shfl_down_sync(0xffffffffu, eb, 2);
                const uint32_t b3 = __shfl_down_sync(0xffffffffu, eb, 3);
                if (g == 0)
                    *reinterpret_cast<uint32_t*>(a.x_scales + sf_offset(grow, (int64_t)kc * 4, a.chunks)) =
                        eb | (b1 << 8) | (b2 << 16) | (b3 << 24);
            } else {
                // one int4 group of 64 = the four lanes of this row
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
                const float sf = __bfloat162float(sb);
                const float inv = (sf == 0.0f) ? 0.0f : __frcp_rn(sf);
                uint32_t w[2] = {0u, 0u};
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    int qi = __float2int_rn(__fmul_rn(v[i], inv));
                    qi = max(-8, min(7, qi));
                    w[i >> 3] |= ((uint32_t)qi & 15u) << (4 * (i & 7));
                }
                c0 = w[0];
                c1 = w[1];
                if (g == 0)
                    reinterpret_cast<uint16_t*>(a.x_scales)[(int64_t)kc * a.rows_pad + grow] = __bfloat16_as_ushort(sb);
            }
            if (grow < a.M)
                *reinterpret_cast<uint2*>(a.x_codes + grow * (int64_t)(a.K / 2) + (int64_t)kc * 32 + g * 8) =
                    make_uint2(c0, c1);
            // release the stage only after its data has been consumed
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }

    // ------------------------------------------------- rank-r result of the CTA
    if (has_lr && warp >= (uint32_t)qa::kWorker0 && warp < (uint32_t)qa::kWorker0 + 4) {
        // four warps cover the four TMEM lane quadrants: one thread per row,
        // 16 columns at a time
        const uint32_t q = warp & 3u;
        const int row = (int)(32u * q + lane);
        const int64_t grow = (int64_t)m0 + row;
        const bool ok = mbar_wait(accb, 0, kSiteQaAcc);
        if (!ok) s_failed = 1;
        tc_fence_after();
        const bool scaled = (PREC == kPrecNvfp4);
        const float ss = scaled ? __fmul_rn(*a.x_scale, *a.w_scale) : 1.0f;
        const int64_t plane = (int64_t)a.M * a.rank;
        float* mine = a.partials + (((int64_t)rb * a.splits + split) * qa::kRows + row) * a.rank;
        for (int c0 = 0; c0 < a.rank; c0 += 16) {
            uint32_t r16[16], s16[16];
            tmem_ld_32x32b_x16(tmem + ((32u * q) << 16) + (uint32_t)c0, r16);              // x . hi
            tmem_ld_32x32b_x16(tmem + ((32u * q) << 16) + (uint32_t)(a.rank + c0), s16);   // x . lo
            tmem_ld_wait();
            float v16[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v16[i] = ok ? __fadd_rn(__uint_as_float(r16[i]), __uint_as_float(s16[i])) : 0.0f;
            if (a.splits == 1) {
                if (grow < a.M) store_lowrank_row(a.lowrank + c0, plane, grow, a.rank, v16, 16, ss, scaled);
            } else {
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4*>(mine + c0 + i) = make_float4(v16[i], v16[i + 1], v16[i + 2], v16[i + 3]);
            }
        }
        if (a.splits > 1) {
            __threadfence();
            named_bar_sync(1, 128);
            if (threadIdx.x == 32 * qa::kWorker0) {
                const unsigned int prev = atomicAdd(a.counters + rb, 1u);
                s_last = (prev == (unsigned int)(a.splits - 1)) ? 1 : 0;
            }
            named_bar_sync(1, 128);
            if (s_last) {
                // the last CTA of this row block adds the partials in split order
                __threadfence();
                for (int c0 = 0; c0 < a.rank; c0 += 16) {
                    float v16[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v16[i] = 0.0f;
                    for (int p = 0; p < a.splits; ++p) {
                        const float* src = a.partials + (((int64_t)rb * a.splits + p) * qa::kRows + row) * a.rank + c0;
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            const float4 f = __ldcg(reinterpret_cast<const float4*>(src + i));
                            v16[i] += f.x;
                            v16[i + 1] += f.y;
                            v16[i + 2] += f.z;
                            v16[i + 3] += f.w;
                        }
                    }
                    if (grow < a.M) store_lowrank_row(a.lowrank + c0, plane, grow, a.rank, v16, 16, ss, scaled);
                }
                if (threadIdx.x == 32 * qa::kWorker0) a.counters[rb] = 0u;   // ready for the next call
            }
        }
    }

    __syncthreads();
    // on a timeout, let the copies already issued land before the CTA exits
    if (s_failed && warp == 0 && lane == 0) {
        for (int s = 0; s < nst; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteQaDrain);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && has_lr) {
        tc_fence_after();
        tmem_dealloc(tmem, a.tmem_cols);
    }
}

}  // namespace svdq
