// svd_split.cuh -- the offline SVDQuant split of a linear layer's weight
// (sm_100a), feeding svdq_pack_weight.
//
// The SVDQuant paper that the Diffusers docs page "Nunchaku Lite" builds on
// (its introduction), and the tutorial's offline quantization step
// (quantize_hf.py --rank 32): the smoothed weight W_hat = W diag(lambda),
// [N, K], is split into a rank-r part and a residual,
//     W_hat = L_up^T L_down^T + R,    L_down [K, r], L_up [r, N],
// with the rank-r part the best one (the truncated SVD), so that only R is
// quantized to 4 bits.  Here the truncated SVD comes from a randomized range
// finder with subspace iteration (Halko, Martinsson and Tropp, "Finding
// structure with randomness", 2011, algorithms 4.4 and 5.1):
//     Y = W_hat Omega           Omega: [K, l] Gaussian test matrix (an input), l = r + p
//     Q = orth(Y); q times:  Q = orth(W_hat orth(W_hat^T Q))
//     Z = W_hat^T Q             (= B^T with B = Q^T W_hat, [l, K])
//     Z^T Z = U diag(s^2) U^T   (eigen-decomposition of the l x l Gram matrix)
//     L_up^T = Q U_r diag(s_r),  L_down = Z U_r diag(1 / s_r)
//     R = W_hat - L_up^T L_down^T   (with the bf16-rounded factors)
// orth() is CholeskyQR2 (two rounds of Gram matrix -> Cholesky -> triangular
// solve, Gram matrices in fp64); the small l x l eigen-problem is cyclic
// Jacobi in fp64.  Every kernel here is an offline, once-per-layer step.
#pragma once
#include "sm100_ptx.cuh"

namespace svdq {
namespace sv {
constexpr int kMaxL = 64;       // rank + oversampling
constexpr int kTileR = 32;      // output rows per block of the products
constexpr int kTileK = 64;      // reduction chunk
constexpr int kGramBlocks = 64;
}  // namespace sv

// Y[N, l] = W_hat X with W_hat[n, k] = W[n, k] lambda[k] and X [K, l] (fp32).
// Block: 32 rows of W; 256 threads; thread t owns output (row t / 8, columns
// t % 8 + 8 j).
__global__ void __launch_bounds__(256) svd_w_times_kernel(const __nv_bfloat16* __restrict__ W,
                                                          const float* __restrict__ lambda, int64_t N, int64_t K,
                                                          const float* __restrict__ X, int l, float* __restrict__ Y) {
    __shared__ float ws[sv::kTileR][sv::kTileK + 1];
    __shared__ float xs[sv::kTileK][sv::kMaxL];
    const int t = threadIdx.x;
    const int64_t n0 = (int64_t)blockIdx.x * sv::kTileR;
    const int r = t >> 3, c0 = t & 7;
    float acc[sv::kMaxL / 8];
#pragma unroll
    for (int j = 0; j < sv::kMaxL / 8; ++j) acc[j] = 0.0f;
    for (int64_t k0 = 0; k0 < K; k0 += sv::kTileK) {
        for (int i = t; i < sv::kTileR * sv::kTileK; i += 256) {
            const int rr = i / sv::kTileK, kk = i % sv::kTileK;
            const int64_t n = n0 + rr, k = k0 + kk;
            ws[rr][kk] = (n < N && k < K) ? __bfloat162float(W[n * K + k]) * lambda[k] : 0.0f;
        }
        for (int i = t; i < sv::kTileK * l; i += 256) {
            const int kk = i / l, j = i % l;
            const int64_t k = k0 + kk;
            xs[kk][j] = k < K ? X[k * l + j] : 0.0f;
        }
        __syncthreads();
        for (int kk = 0; kk < sv::kTileK; ++kk) {
            const float w = ws[r][kk];
#pragma unroll
            for (int j = 0; j < sv::kMaxL / 8; ++j)
                if (c0 + 8 * j < l) acc[j] = fmaf(w, xs[kk][c0 + 8 * j], acc[j]);
        }
        __syncthreads();
    }
    const int64_t n = n0 + r;
    if (n < N)
#pragma unroll
        for (int j = 0; j < sv::kMaxL / 8; ++j)
            if (c0 + 8 * j < l) Y[n * l + c0 + 8 * j] = acc[j];
}

// Z[K, l] = W_hat^T Q with Q [N, l].  Block: 32 columns k of W.
__global__ void __launch_bounds__(256) svd_wt_times_kernel(const __nv_bfloat16* __restrict__ W,
                                                           const float* __restrict__ lambda, int64_t N, int64_t K,
                                                           const float* __restrict__ Qm, int l, float* __restrict__ Z) {
    __shared__ float ws[sv::kTileK][sv::kTileR + 1];   // [n][k]
    __shared__ float qs[sv::kTileK][sv::kMaxL];
    const int t = threadIdx.x;
    const int64_t kb = (int64_t)blockIdx.x * sv::kTileR;
    const int r = t >> 3, c0 = t & 7;
    float acc[sv::kMaxL / 8];
#pragma unroll
    for (int j = 0; j < sv::kMaxL / 8; ++j) acc[j] = 0.0f;
    for (int64_t nn0 = 0; nn0 < N; nn0 += sv::kTileK) {
        for (int i = t; i < sv::kTileK * sv::kTileR; i += 256) {
            const int nn = i / sv::kTileR, kk = i % sv::kTileR;
            const int64_t n = nn0 + nn, k = kb + kk;
            ws[nn][kk] = (n < N && k < K) ? __bfloat162float(W[n * K + k]) : 0.0f;
        }
        for (int i = t; i < sv::kTileK * l; i += 256) {
            const int nn = i / l, j = i % l;
            const int64_t n = nn0 + nn;
            qs[nn][j] = n < N ? Qm[n * l + j] : 0.0f;
        }
        __syncthreads();
        for (int nn = 0; nn < sv::kTileK; ++nn) {
            const float w = ws[nn][r];
#pragma unroll
            for (int j = 0; j < sv::kMaxL / 8; ++j)
                if (c0 + 8 * j < l) acc[j] = fmaf(w, qs[nn][c0 + 8 * j], acc[j]);
        }
        __syncthreads();
    }
    const int64_t k = kb + r;
    if (k < K) {
        const float lk = lambda[k];
#pragma unroll
        for (int j = 0; j < sv::kMaxL / 8; ++j)
            if (c0 + 8 * j < l) Z[k * l + c0 + 8 * j] = acc[j] * lk;
    }
}

// Partial Gram matrices of A [rows, l]: block b adds rows b, b + B, ... into
// part[b] (fp64, upper triangle and diagonal).
__global__ void __launch_bounds__(256) svd_gram_partial_kernel(const float* __restrict__ A, int64_t rows, int l,
                                                               double* __restrict__ part) {
    double* G = part + (int64_t)blockIdx.x * sv::kMaxL * sv::kMaxL;
    const int npairs = l * (l + 1) / 2;
    for (int p = threadIdx.x; p < npairs; p += blockDim.x) {
        // pair p -> (i, j) with i <= j
        int i = 0, rem = p;
        while (rem >= l - i) {
            rem -= l - i;
            ++i;
        }
        const int j = i + rem;
        double s = 0.0;
        for (int64_t row = blockIdx.x; row < rows; row += gridDim.x)
            s += (double)A[row * l + i] * (double)A[row * l + j];
        G[i * sv::kMaxL + j] = s;
    }
}

// Adds the partial Gram matrices in block order and returns, in one thread,
// Rinv = R^-1 for the Cholesky factor G = R^T R (R upper triangular).  A pivot
// that is not clearly positive drops its direction (row of Rinv zero).
__global__ void svd_chol_inv_kernel(const double* __restrict__ part, int nparts, int l, double* __restrict__ Rinv) {
    __shared__ double R[sv::kMaxL][sv::kMaxL];   // G, overwritten row by row with its Cholesky factor
    for (int p = threadIdx.x; p < l * l; p += blockDim.x) {
        const int i = p / l, j = p % l;
        double s = 0.0;
        if (i <= j)
            for (int b = 0; b < nparts; ++b) s += part[((int64_t)b * sv::kMaxL + i) * sv::kMaxL + j];
        R[i][j] = s;
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    double dmax = 0.0;
    for (int i = 0; i < l; ++i) dmax = fmax(dmax, R[i][i]);
    const double tiny = dmax * 1e-28 + 1e-300;
    for (int i = 0; i < l; ++i) {
        double d = R[i][i];
        for (int k = 0; k < i; ++k) d -= R[k][i] * R[k][i];
        const bool ok = d > tiny;
        R[i][i] = ok ? sqrt(d) : 0.0;
        for (int j = i + 1; j < l; ++j) {
            double s = R[i][j];
            for (int k = 0; k < i; ++k) s -= R[k][i] * R[k][j];
            R[i][j] = ok ? s / R[i][i] : 0.0;
        }
    }
    // inverse of the upper-triangular R by back substitution, column by column
    for (int j = 0; j < l; ++j) {
        for (int i = j; i >= 0; --i) {
            double s = (i == j) ? 1.0 : 0.0;
            for (int k = i + 1; k <= j; ++k) s -= R[i][k] * Rinv[k * sv::kMaxL + j];
            Rinv[i * sv::kMaxL + j] = R[i][i] > 0.0 ? s / R[i][i] : 0.0;
        }
        for (int i = j + 1; i < l; ++i) Rinv[i * sv::kMaxL + j] = 0.0;
    }
}

// A[row, :] <- A[row, :] Rinv (one thread per row).
__global__ void __launch_bounds__(256) svd_apply_rinv_kernel(float* __restrict__ A, int64_t rows, int l,
                                                             const double* __restrict__ Rinv) {
    __shared__ float Rs[sv::kMaxL * sv::kMaxL];
    for (int p = threadIdx.x; p < l * l; p += blockDim.x)
        Rs[p] = (float)Rinv[(p / l) * sv::kMaxL + (p % l)];
    __syncthreads();
    const int64_t row = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (row >= rows) return;
    float a[sv::kMaxL];
#pragma unroll
    for (int i = 0; i < sv::kMaxL; ++i) a[i] = i < l ? A[row * l + i] : 0.0f;
    for (int j = 0; j < l; ++j) {
        float s = 0.0f;
        for (int i = 0; i <= j; ++i) s = fmaf(a[i], Rs[i * l + j], s);
        A[row * l + j] = s;
    }
}

// Eigen-decomposition of the symmetric l x l matrix assembled from the
// partial Gram matrices, by cyclic Jacobi rotations (one warp, fp64).
// Outputs: evals[l] in decreasing order and the matching eigenvectors as the
// columns of U (row-major [l][kMaxL]).
constexpr size_t kJacobiSmem = 2 * sizeof(double) * sv::kMaxL * (sv::kMaxL + 1);

__global__ void svd_jacobi_kernel(const double* __restrict__ part, int nparts, int l, double* __restrict__ evals,
                                  double* __restrict__ U) {
    extern __shared__ double jac_smem[];   // kJacobiSmem bytes
    auto A = reinterpret_cast<double(*)[sv::kMaxL + 1]>(jac_smem);
    auto V = reinterpret_cast<double(*)[sv::kMaxL + 1]>(jac_smem + sv::kMaxL * (sv::kMaxL + 1));
    const int lane = threadIdx.x;
    for (int p = lane; p < l * l; p += 32) {
        const int i = p / l, j = p % l;
        const int a = min(i, j), b = max(i, j);
        double s = 0.0;
        for (int q = 0; q < nparts; ++q) s += part[((int64_t)q * sv::kMaxL + a) * sv::kMaxL + b];
        A[i][j] = s;
        V[i][j] = (i == j) ? 1.0 : 0.0;
    }
    __syncwarp();
    for (int sweep = 0; sweep < 30; ++sweep) {
        double off = 0.0, tot = 0.0;
        for (int p = lane; p < l * l; p += 32) {
            const int i = p / l, j = p % l;
            if (i != j) off += A[i][j] * A[i][j];
            tot += A[i][j] * A[i][j];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            off += __shfl_xor_sync(0xffffffffu, off, o);
            tot += __shfl_xor_sync(0xffffffffu, tot, o);
        }
        if (off <= 1e-30 * tot) break;
        for (int p = 0; p < l - 1; ++p)
            for (int q = p + 1; q < l; ++q) {
                const double apq = A[p][q];
                if (fabs(apq) <= 1e-300) continue;
                const double app = A[p][p], aqq = A[q][q];
                const double theta = (aqq - app) / (2.0 * apq);
                const double tt = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
                const double c = 1.0 / sqrt(tt * tt + 1.0), s = tt * c;
                __syncwarp();
                // rows p and q, then columns p and q (A <- J^T A J), and V <- V J
                for (int k = lane; k < l; k += 32) {
                    const double akp = A[p][k], akq = A[q][k];
                    A[p][k] = c * akp - s * akq;
                    A[q][k] = s * akp + c * akq;
                }
                __syncwarp();
                for (int k = lane; k < l; k += 32) {
                    const double apk = A[k][p], aqk = A[k][q];
                    A[k][p] = c * apk - s * aqk;
                    A[k][q] = s * apk + c * aqk;
                    const double vkp = V[k][p], vkq = V[k][q];
                    V[k][p] = c * vkp - s * vkq;
                    V[k][q] = s * vkp + c * vkq;
                }
                __syncwarp();
            }
    }
    __syncwarp();
    if (lane == 0) {
        // order by decreasing eigenvalue (selection sort of column indices)
        int idx[sv::kMaxL];
        for (int i = 0; i < l; ++i) idx[i] = i;
        for (int i = 0; i < l; ++i) {
            int best = i;
            for (int j = i + 1; j < l; ++j)
                if (A[idx[j]][idx[j]] > A[idx[best]][idx[best]]) best = j;
            const int tmp = idx[i];
            idx[i] = idx[best];
            idx[best] = tmp;
        }
        for (int i = 0; i < l; ++i) {
            evals[i] = A[idx[i]][idx[i]];
            for (int k = 0; k < l; ++k) U[k * sv::kMaxL + i] = V[k][idx[i]];
        }
    }
}

// L_up[j, n] = bf16(s_j sum_i Q[n, i] U[i, j]) and L_down[k, j] =
// bf16(sum_i Z[k, i] U[i, j] / s_j) for j < r (one thread per output row).
__global__ void __launch_bounds__(256) svd_factors_kernel(const float* __restrict__ Qm, int64_t N,
                                                          const float* __restrict__ Z, int64_t K, int l, int r,
                                                          const double* __restrict__ evals,
                                                          const double* __restrict__ U,
                                                          __nv_bfloat16* __restrict__ L_up,
                                                          __nv_bfloat16* __restrict__ L_down,
                                                          float* __restrict__ sv_out) {
    __shared__ float Us[sv::kMaxL * sv::kMaxL];
    __shared__ float sv_s[sv::kMaxL];
    for (int p = threadIdx.x; p < l * l; p += blockDim.x) Us[p] = (float)U[(p / l) * sv::kMaxL + (p % l)];
    for (int j = threadIdx.x; j < l; j += blockDim.x) sv_s[j] = (float)sqrt(fmax(evals[j], 0.0));
    __syncthreads();
    if (blockIdx.x == 0 && sv_out)
        for (int j = threadIdx.x; j < l; j += blockDim.x) sv_out[j] = sv_s[j];
    const int64_t row = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (row < N) {
        for (int j = 0; j < r; ++j) {
            float s = 0.0f;
            for (int i = 0; i < l; ++i) s = fmaf(Qm[row * l + i], Us[i * l + j], s);
            L_up[(int64_t)j * N + row] = __float2bfloat16_rn(s * sv_s[j]);
        }
    }
    if (row < K) {
        for (int j = 0; j < r; ++j) {
            float s = 0.0f;
            for (int i = 0; i < l; ++i) s = fmaf(Z[row * l + i], Us[i * l + j], s);
            L_down[row * r + j] = __float2bfloat16_rn(sv_s[j] > 0.0f ? s / sv_s[j] : 0.0f);
        }
    }
}

// R[n, k] = bf16(W[n, k] lambda[k] - sum_j L_up[j, n] L_down[k, j]) with the
// bf16 factors (fp32 sums).  Block: 32 rows n x 64 columns k.
__global__ void __launch_bounds__(256) svd_residual_kernel(const __nv_bfloat16* __restrict__ W,
                                                           const float* __restrict__ lambda, int64_t N, int64_t K,
                                                           const __nv_bfloat16* __restrict__ L_up,
                                                           const __nv_bfloat16* __restrict__ L_down, int r,
                                                           __nv_bfloat16* __restrict__ R) {
    __shared__ float us[sv::kMaxL][32];   // L_up[j, n0 + i]
    __shared__ float ds[64][sv::kMaxL];   // L_down[k0 + kk, j]
    const int64_t n0 = (int64_t)blockIdx.y * 32, k0 = (int64_t)blockIdx.x * 64;
    for (int p = threadIdx.x; p < r * 32; p += blockDim.x) {
        const int j = p / 32, i = p % 32;
        us[j][i] = n0 + i < N ? __bfloat162float(L_up[(int64_t)j * N + n0 + i]) : 0.0f;
    }
    for (int p = threadIdx.x; p < 64 * r; p += blockDim.x) {
        const int kk = p / r, j = p % r;
        ds[kk][j] = k0 + kk < K ? __bfloat162float(L_down[(k0 + kk) * r + j]) : 0.0f;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < 32 * 64; p += blockDim.x) {
        const int i = p / 64, kk = p % 64;
        const int64_t n = n0 + i, k = k0 + kk;
        if (n >= N || k >= K) continue;
        float s = 0.0f;
        for (int j = 0; j < r; ++j) s = fmaf(us[j][i], ds[kk][j], s);
        R[n * K + k] = __float2bfloat16_rn(__bfloat162float(W[n * K + k]) * lambda[k] - s);
    }
}

}  // namespace svdq
