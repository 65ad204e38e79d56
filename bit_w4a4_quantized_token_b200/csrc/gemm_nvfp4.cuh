// gemm_nvfp4.cuh -- block-scaled FP4 GEMM of the SVDQ W4A4 layer (sm_100a).
//
//   acc[m, n]  = sum_k (q_x[m,k] e_x[m,k/16]) (q_w[n,k] e_w[n,k/16])   FP4 x FP4, fp32 in TMEM
//   acc[m, n] += sum_j L'[m, j] L_up[j, n]       rank-r branch: bf16 MMAs of the hi and lo
//                                                parts of L' into the same accumulator
//   y[m, n]    = bf16( S_x S_w acc[m, n] + b[n] )
// where L' = ((x/lambda) . L_down) / (S_x S_w) comes from the quantizer.  The
// "NVFP4 runtime kernel with SVDQ low-rank correction" of the Diffusers docs
// page "Nunchaku Lite" ("Supported quantization types" table).
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles taken round-robin.
// Three producer warps fill a ring of stages that runs across tile
// boundaries: warp 0 loads the activation codes (TMA, 128-byte swizzle),
// warp 1 the weight codes, warp 3 the two operands' scale blocks (bulk
// copies); one issuing thread cannot keep the tensor core fed on its own.
// Warp 2 copies each stage's scale blocks into TMEM and issues tcgen05.mma
// (kind::mxf4nvf4, K = 64 per instruction; kind::f16 for the rank-r chunks).
// Eight epilogue warps (4..11) pull the finished accumulator out of TMEM into
// registers, hand TMEM back to the MMA warp at once, and then scale, add the
// bias and store bf16 while the next tile's MMAs run.
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {
namespace gm {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;                 // 256 FP4 values of K per row per stage
constexpr int kStages = 4;
constexpr int A_BYTES = BM * BK_BYTES;        // 16 KB (also holds a 128 x 64 bf16 rank-r tile)
constexpr int B_BYTES = BN * BK_BYTES;        // 32 KB (also holds a 256 x 64 bf16 L_up tile)
constexpr int SFA_BYTES = 4 * 512;            // 4 scale blocks: 128 rows x 16 groups
constexpr int SFB_BYTES = 8 * 512;            // 2 row blocks x 4 scale blocks
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int kEpiWarps = 8;                  // 2 per TMEM lane quadrant, 128 columns each
constexpr int kEpiWarp0 = 4;                  // first epilogue warp (a multiple of 4)
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr uint32_t kMmaWarp = 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;               // 256 fp32 columns
constexpr uint32_t SF_COL = 256;              // scale factors of ring stage s at SF_COL + 48 s:
constexpr uint32_t SF_STAGE_COLS = 48;        //   4 k-steps x 4 columns (A), then 4 k-steps x 8 columns (B)
static_assert(SF_COL + kStages * SF_STAGE_COLS <= TMEM_COLS, "scale-factor columns do not fit in TMEM");
constexpr size_t SMEM_BYTES = 1024 + (size_t)kStages * STAGE_BYTES + 256;
}  // namespace gm

struct GemmArgs {
    const uint8_t* x_scales;
    const uint8_t* w_scales;
    const float* x_scale;
    const float* w_scale;
    const __nv_bfloat16* bias;   // may be null
    __nv_bfloat16* y;
    int M, N, K, rank;
    int kg4;                     // K / 64: scale blocks per 128 rows
    int n_sf_blocks;             // ceil(N / 128): 128-row blocks present in w_scales
    int m_tiles, n_tiles;
    // Fused QKV + RMSNorm + RoPE epilogue (pair kernel only; qk_cols == 0
    // disables it): columns [0, q_cols) are the Q heads and [q_cols, qk_cols)
    // the K heads (128 columns each) of a to_qkv projection.
    const __nv_bfloat16* norm_q;   // [128] RMSNorm weights of the Q heads
    const __nv_bfloat16* norm_k;   // [128] RMSNorm weights of the K heads
    const float* rope_cos;         // [M, 64] per-token rotary tables
    const float* rope_sin;
    float eps;
    int q_cols, qk_cols;
    // Fused GELU + next-layer activation epilogue (pair kernel, kEpiGelu):
    // h = bf16(GELU(y)) is not stored; the next layer's activation step is
    // done on it instead (gelu_mlp.cuh).
    int gelu_approx;                 // 0: x Phi(x); 1: tanh form
    const float* nx_inv_lambda;      // [N] 1 / lambda of the next layer
    const __nv_bfloat16* nx_ldt;     // [2, nx_rank, N] hi/lo planes of L_down / lambda (next layer)
    int nx_rank;                     // 0, 16 or 32
    const float* nx_x_scale;         // the next layer's static activation tensor scale
    uint8_t* nx_codes;               // [M, N / 2] nvfp4 codes of h / lambda
    uint8_t* nx_scales;              // their E4M3 group scales, tensor-core layout, K = N
    float* nx_acc;                   // [M, nx_rank] fp32 sums of h (L_down / lambda), zero on entry
    int nx_rows_pad;                 // rows of nx_scales: M rounded up to 128
};

enum : uint32_t { kSiteGmEmpty = 16, kSiteGmFull = 17, kSiteGmAcc = 18, kSiteGmDrain = 19, kSiteGmAccEmpty = 20 };

__global__ void __launch_bounds__(gm::kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_wc,
                      const __grid_constant__ CUtensorMap tm_L, const __grid_constant__ CUtensorMap tm_Lup,
                      GemmArgs a) {
    using namespace gm;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * STAGE_BYTES);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
    __shared__ int s_failed;
    __shared__ int s_issued[gm::kStages];   // phases started in each stage (by the A-code producer)

    const uint32_t warp = warp_id(), lane = lane_id();
    const int n_kb = (a.K + 255) / 256;
    const int n_lr = a.rank > 0 ? 2 * ((a.rank + 63) / 64) : 0;   // hi and lo part of each 64-column chunk
    const int per_tile = n_kb + n_lr;
    const int total_tiles = a.m_tiles * a.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 3);               // one arrival per producer warp
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kEpiWarps);
        for (int s = 0; s < kStages; ++s) s_issued[s] = 0;
        s_failed = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_xc);
        prefetch_tensormap(&tm_wc);
        if (a.rank > 0) {
            prefetch_tensormap(&tm_L);
            prefetch_tensormap(&tm_Lup);
        }
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 1 || warp == 3) {
        // ----------------------------------------------------------- producers
        if (lane == 0) {
            const int role = warp == 0 ? 0 : (warp == 1 ? 1 : 2);   // A codes, B codes, scale blocks
            int it = 0;   // position in the stage ring, continued across tiles
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const int m_tile = tile % a.m_tiles, n_tile = tile / a.m_tiles;
                const int m0 = m_tile * BM, n0 = n_tile * BN;
                const int nb0 = 2 * n_tile;
                const int nbv = (nb0 < a.n_sf_blocks ? 1 : 0) + (nb0 + 1 < a.n_sf_blocks ? 1 : 0);
                for (int kk = 0; kk < per_tile; ++kk, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, kSiteGmEmpty)) {
                        s_failed = 1;
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + (size_t)s * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    uint8_t* sfa = sb + B_BYTES;
                    uint8_t* sfb = sfa + SFA_BYTES;
                    if (kk < n_kb) {
                        const int kb = kk;
                        if (role == 0) {
                            mbar_arrive_expect_tx(&full[s], A_BYTES);
                            tma_load_2d(sa, &tm_xc, &full[s], kb * BK_BYTES, m0);
                            reinterpret_cast<volatile int*>(s_issued)[s] += 1;
                        } else if (role == 1) {
                            mbar_arrive_expect_tx(&full[s], B_BYTES);
                            tma_load_2d(sb, &tm_wc, &full[s], kb * BK_BYTES, n0);
                        } else {
                            const int natoms = min(4, a.kg4 - 4 * kb);
                            const uint32_t sf_bytes = (uint32_t)natoms * 512u;
                            mbar_arrive_expect_tx(&full[s], sf_bytes * (1u + (uint32_t)nbv));
                            bulk_load(sfa, a.x_scales + ((int64_t)m_tile * a.kg4 + 4 * kb) * 512, sf_bytes, &full[s]);
                            for (int rb = 0; rb < nbv; ++rb)
                                bulk_load(sfb + rb * 2048, a.w_scales + ((int64_t)(nb0 + rb) * a.kg4 + 4 * kb) * 512,
                                          sf_bytes, &full[s]);
                        }
                    } else {
                        const int c = (kk - n_kb) >> 1, part = (kk - n_kb) & 1;
                        if (role == 0) {
                            mbar_arrive_expect_tx(&full[s], A_BYTES);
                            tma_load_3d(sa, &tm_L, &full[s], c * 64, m0, part);
                            reinterpret_cast<volatile int*>(s_issued)[s] += 1;
                        } else if (role == 1) {
                            mbar_arrive_expect_tx(&full[s], B_BYTES);
                            tma_load_2d(sb, &tm_Lup, &full[s], c * 64, n0);
                        } else {
                            mbar_arrive(&full[s]);
                        }
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_fp4 = idesc_nvfp4(BN);
            const uint32_t idesc_lr = idesc_bf16_f32(BN);
            bool ok = true;
            int it = 0, local = 0;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++local) {
                // the epilogue must have pulled the previous tile out of TMEM
                if (!mbar_wait(acc_empty, ((uint32_t)local & 1u) ^ 1u, kSiteGmAccEmpty)) {
                    s_failed = 1;
                    break;
                }
                tc_fence_after();
                for (int kk = 0; kk < per_tile; ++kk, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    if (!mbar_wait(&full[s], ph, kSiteGmFull)) {
                        ok = false;
                        s_failed = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + (size_t)s * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    if (kk < n_kb) {
                        const uint32_t sfa = sb + B_BYTES;
                        const uint32_t sfb = sfa + SFA_BYTES;
                        const int nks = min(4, a.kg4 - 4 * kk);
                        // Scale blocks go to this stage's own TMEM columns, and the
                        // copies for K-step j + 1 are issued before the MMA of step j:
                        // the tensor pipe runs its instructions in order, so copies
                        // queued behind an MMA overlap it, while a batch of copies in
                        // front of the MMAs would not.
                        const uint32_t t_sfa = tmem + SF_COL + SF_STAGE_COLS * (uint32_t)s;
                        const uint32_t t_sfb = t_sfa + 16u;
                        auto copy_scales = [&](int j) {
                            tmem_cp_32x128b_x4(t_sfa + 4u * j, desc_sf_block(sfa + 512u * j));
                            tmem_cp_32x128b_x4(t_sfb + 8u * j, desc_sf_block(sfb + 512u * j));
                            tmem_cp_32x128b_x4(t_sfb + 8u * j + 4u, desc_sf_block(sfb + 2048u + 512u * j));
                        };
                        copy_scales(0);
                        for (int j = 0; j < nks; ++j) {
                            if (j + 1 < nks) copy_scales(j + 1);
                            mma_nvfp4(tmem + ACC_COL, desc_sw128(sa + 32u * j), desc_sw128(sb + 32u * j), idesc_fp4,
                                      t_sfa + 4u * j, t_sfb + 8u * j, (kk > 0 || j > 0) ? 1u : 0u);
                        }
                    } else {
                        const int c = (kk - n_kb) >> 1;
                        const int nks = min(4, (a.rank - 64 * c + 15) / 16);
                        for (int j = 0; j < nks; ++j)
                            mma_bf16(tmem + ACC_COL, desc_sw128(sa + 32u * j), desc_sw128(sb + 32u * j), idesc_lr,
                                     1u);
                    }
                    tc_commit(&empty[s]);
                }
                if (ok) tc_commit(acc_full);
            }
        }
    } else if (warp >= (uint32_t)kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        const uint32_t q = warp & 3u;                 // TMEM lane quadrant this warp may read
        const int half = (int)(warp - kEpiWarp0) >> 2;   // which 128 of the 256 columns
        const int row = (int)(32u * q + lane);
        const float S = __fmul_rn(*a.x_scale, *a.w_scale);
        int local = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++local) {
            const int m_tile = tile % a.m_tiles, n_tile = tile / a.m_tiles;
            const int64_t grow = (int64_t)m_tile * BM + row;
            const int nbase = n_tile * BN + 128 * half;
            const bool ok = mbar_wait(acc_full, (uint32_t)local & 1u, kSiteGmAcc);
            if (!ok) {
                s_failed = 1;
                break;
            }
            tc_fence_after();
            uint32_t acc[128];
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 0u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 0));
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 32u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 32));
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 64u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 64));
            tmem_ld_32x32b_x32(tmem + ((32u * q) << 16) + ACC_COL + 128u * half + 96u,
                               *reinterpret_cast<uint32_t(*)[32]>(acc + 96));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);     // TMEM is free for the next tile
            if (grow >= a.M) continue;
            __nv_bfloat16* yrow = a.y + grow * (int64_t)a.N;
#pragma unroll
            for (int c = 0; c < 8; ++c) {              // 16 columns at a time
                const int n = nbase + 16 * c;
                if (n >= a.N) break;                   // N % 16 == 0
                float bv[16];
                if (a.bias) {
                    const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(a.bias + n));
                    const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(a.bias + n) + 1);
                    const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        bv[2 * p] = bf16lo_to_f32(ws[p]);
                        bv[2 * p + 1] = bf16hi_to_f32(ws[p]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) bv[i] = 0.0f;
                }
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float o0 = fmaf(__uint_as_float(acc[16 * c + 2 * i]), S, bv[2 * i]);
                    const float o1 = fmaf(__uint_as_float(acc[16 * c + 2 * i + 1]), S, bv[2 * i + 1]);
                    const __nv_bfloat162 h = __floats2bfloat162_rn(o0, o1);
                    packed[i] = *reinterpret_cast<const uint32_t*>(&h);
                }
                uint4* dst = reinterpret_cast<uint4*>(yrow + n);
                dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
        }
    }

    __syncthreads();
    if (s_failed && warp == 0 && lane == 0) {
        // on a timeout, let the loads already issued land before the CTA exits
        for (int s = 0; s < kStages; ++s) {
            const int n = reinterpret_cast<volatile int*>(s_issued)[s];
            if (n > 0) mbar_wait(&full[s], (uint32_t)(n - 1) & 1u, kSiteGmDrain);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace svdq
