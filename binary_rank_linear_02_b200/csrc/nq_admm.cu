// nq_admm.cu -- the LB-ADMM initialiser of the binary factorisation on the device.
//
// NanoQuant initialises the binary factors and scales of a layer by ADMM: a closed-form
// least-squares step for the continuous parameters alternates with a projection onto the
// binary constraint by the sign operation, and magnitude balancing of the scales follows
// (hardwired.dev, "NanoQuant jednoduse: 70B model na herni grafice", section "Trikrokovy
// pipeline", step 2; the routines power_iteration, rank1_approx, svid and
// factorize_admm_nanoquant are named in the codewithpapers.app record of arXiv 2602.06694).
// The pages give no formula; this file implements the library's reading of it:
//
//   W ~= A B^T, A (m x r) and B (n x r) latent, constrained to row-scaled sign matrices
//   Z = diag(s) S (S in {+1,-1}), so that Z_A Z_B^T = diag(s1) U V^T diag(s2) is the stored
//   form.  One iteration (Gauss-Seidel, scaled duals L):
//     rho_A = lam_k tr(B^T B) / r
//     A     = (W B + rho_A (Z_A - L_A)) (B^T B + rho_A I)^-1        least squares, closed form
//     Z_A   = Pi(A + L_A): per row, signs and the scale mean |.|     projection
//     L_A  += A - Z_A                                               dual
//     the same for B with W^T and the new A;  lam_{k+1} = growth lam_k.
//   Start: block power iteration from a caller-given n x r Gaussian Omega, Q = orth(W Omega)
//   then q times Q = orth(W (W^T Q)), orth by Cholesky-QR; A0 = Q, B0 = W^T Q with each
//   column pair rescaled to equal norms; Z = Pi(A0), Pi(B0), L = 0.
//   Result: U, s_A from Z_A, V, s_B from Z_B; s1 = c s_A, s2 = s_B / c with
//   c = sqrt(rms(s_B) / rms(s_A)) (magnitude balancing: equal root-mean-squares).
//
// On the device every dense step is an fp32 GEMM with a fused epilogue (gemm_f32_kernel:
// strided, optionally transposed operands, W read as bfloat16), the r x r systems are
// solved by a blocked right-looking Cholesky factorisation (diagonal block in shared
// memory, panel by triangular solve, trailing update by the GEMM) and blocked triangular
// solves whose updates are again GEMMs.  All reductions run in a fixed order, so a run is
// deterministic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include <vector>

#include "nq_internal.cuh"

namespace nq {
namespace {

// ------------------------------------------------------------------ fp32 GEMM
// C[i][j] = alpha * sum_k opA[i][k] opB[k][j] + sc * (beta D[i][j] + gamma E[i][j] + delta [i == j])
// with sc = *scale (a device scalar) when `scale` is set, else 1.  opA[i][k] = A[i*lda + k]
// (TA_T: A[k*lda + i]); opB[k][j] = B[k*ldb + j] (TB_T: B[j*ldb + k]).  D may alias C
// (each element is read and then written by the same thread).  With `sq` set nothing is
// stored: the tile's sum of squares of the C values goes to sq[tile] (fixed order).
constexpr int kGM = 128, kGN = 128, kGK = 16, kGThreads = 256;

template <typename TA, typename TD = float>
struct GemmF32 {
    int64_t M, N, K;
    float alpha, beta, gamma, delta;
    const TA* A;
    int64_t lda;
    const float* B;
    int64_t ldb;
    const TD* D;
    int64_t ldd;
    const float* E;
    int64_t lde;
    float* C;
    int64_t ldc;
    const float* scale;
    double* sq;
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename TA, typename TD, bool TA_T, bool TB_T>
__global__ void __launch_bounds__(kGThreads) gemm_f32_kernel(const __grid_constant__ GemmF32<TA, TD> g) {
    __shared__ __align__(16) float As[2][kGK][kGM + 4];
    __shared__ __align__(16) float Bs[2][kGK][kGN + 4];
    const int t = threadIdx.x;
    const int64_t i0 = (int64_t)blockIdx.y * kGM, j0 = (int64_t)blockIdx.x * kGN;
    const int ty = t >> 4, tx = t & 15;

    float ra[8], rb[8];
    // global -> registers for k-block kb (8 elements of A and of B per thread)
    auto load = [&](int64_t k0) {
        if (!TA_T) {  // A row-major M x K: a thread takes 8 consecutive k of one row
            const int ii = t >> 1, kk = (t & 1) * 8;
            const int64_t gi = i0 + ii;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int64_t gk = k0 + kk + q;
                ra[q] = (gi < g.M && gk < g.K) ? to_f32(g.A[gi * g.lda + gk]) : 0.f;
            }
        } else {  // A stored K x M: 8 consecutive i of one k
            const int kk = t >> 4, ii = (t & 15) * 8;
            const int64_t gk = k0 + kk;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int64_t gi = i0 + ii + q;
                ra[q] = (gi < g.M && gk < g.K) ? to_f32(g.A[gk * g.lda + gi]) : 0.f;
            }
        }
        if (!TB_T) {  // B row-major K x N: 8 consecutive j of one k
            const int kk = t >> 4, jj = (t & 15) * 8;
            const int64_t gk = k0 + kk;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int64_t gj = j0 + jj + q;
                rb[q] = (gj < g.N && gk < g.K) ? g.B[gk * g.ldb + gj] : 0.f;
            }
        } else {  // B stored N x K: 8 consecutive k of one j
            const int jj = t >> 1, kk = (t & 1) * 8;
            const int64_t gj = j0 + jj;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int64_t gk = k0 + kk + q;
                rb[q] = (gj < g.N && gk < g.K) ? g.B[gj * g.ldb + gk] : 0.f;
            }
        }
    };
    auto store = [&](int buf) {
        if (!TA_T) {
            const int ii = t >> 1, kk = (t & 1) * 8;
#pragma unroll
            for (int q = 0; q < 8; ++q) As[buf][kk + q][ii] = ra[q];
        } else {
            const int kk = t >> 4, ii = (t & 15) * 8;
#pragma unroll
            for (int q = 0; q < 8; ++q) As[buf][kk][ii + q] = ra[q];
        }
        if (!TB_T) {
            const int kk = t >> 4, jj = (t & 15) * 8;
#pragma unroll
            for (int q = 0; q < 8; ++q) Bs[buf][kk][jj + q] = rb[q];
        } else {
            const int jj = t >> 1, kk = (t & 1) * 8;
#pragma unroll
            for (int q = 0; q < 8; ++q) Bs[buf][kk + q][jj] = rb[q];
        }
    };

    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

    const int64_t nk = (g.K + kGK - 1) / kGK;
    if (nk > 0) {
        load(0);
        store(0);
    }
    __syncthreads();
    for (int64_t kb = 0; kb < nk; ++kb) {
        const int buf = (int)(kb & 1);
        if (kb + 1 < nk) load((kb + 1) * kGK);
#pragma unroll
        for (int k = 0; k < kGK; ++k) {
            // rows ty*4 .. +3 and 64 + ty*4 .. +3; columns tx*4 .. +3 and 64 + tx*4 .. +3
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][k][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][k][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
        }
        if (kb + 1 < nk) store(buf ^ 1);
        __syncthreads();
    }

    const float sc = g.scale ? *g.scale : 1.f;
    const float beta = g.beta * sc, gamma = g.gamma * sc, delta = g.delta * sc;
    double sq = 0.0;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int64_t i = i0 + (a < 4 ? ty * 4 + a : 64 + ty * 4 + a - 4);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int64_t j = j0 + (b < 4 ? tx * 4 + b : 64 + tx * 4 + b - 4);
            if (i < g.M && j < g.N) {
                float v = g.alpha * acc[a][b];
                if (g.D) v += beta * to_f32(g.D[i * g.ldd + j]);
                if (g.E) v += gamma * g.E[i * g.lde + j];
                if (i == j) v += delta;
                if (g.sq)
                    sq += (double)v * (double)v;
                else
                    g.C[i * g.ldc + j] = v;
            }
        }
    }
    if (g.sq) {
        __shared__ double red[kGThreads];
        red[t] = sq;
        __syncthreads();
        for (int s = kGThreads / 2; s > 0; s >>= 1) {
            if (t < s) red[t] += red[t + s];
            __syncthreads();
        }
        if (t == 0) g.sq[blockIdx.y * gridDim.x + blockIdx.x] = red[0];
    }
}

template <typename TA, bool TA_T, bool TB_T, typename TD = float>
int gemm(const GemmF32<TA, TD>& g, cudaStream_t s) {
    if (g.M <= 0 || g.N <= 0) return NQ_OK;
    const dim3 grid((unsigned)((g.N + kGN - 1) / kGN), (unsigned)((g.M + kGM - 1) / kGM));
    gemm_f32_kernel<TA, TD, TA_T, TB_T><<<grid, kGThreads, 0, s>>>(g);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

template <typename TA, typename TD = float>
GemmF32<TA, TD> gemm_args(int64_t M, int64_t N, int64_t K, const TA* A, int64_t lda, const float* B, int64_t ldb,
                          float* C, int64_t ldc) {
    GemmF32<TA, TD> g;
    g.M = M; g.N = N; g.K = K;
    g.alpha = 1.f; g.beta = 0.f; g.gamma = 0.f; g.delta = 0.f;
    g.A = A; g.lda = lda; g.B = B; g.ldb = ldb;
    g.D = nullptr; g.ldd = 0; g.E = nullptr; g.lde = 0;
    g.C = C; g.ldc = ldc; g.scale = nullptr; g.sq = nullptr;
    return g;
}

// ------------------------------------------------------------------ Cholesky and triangular solves
constexpr int kNB = 64;  // block size of the blocked factorisation and solves

// Factor the nb x nb diagonal block at (k0, k0) of the symmetric positive definite H
// (lower triangle used) in place: H_kk = L_kk L_kk^T.  One CTA; a pivot that is not
// positive (H not positive definite in fp32) sets *flag.
__global__ void __launch_bounds__(256) potrf_diag_kernel(float* H, int64_t ld, int64_t k0, int nb, int* flag) {
    __shared__ float a[kNB][kNB + 1];
    for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) a[e / nb][e % nb] = H[(k0 + e / nb) * ld + k0 + e % nb];
    __syncthreads();
    for (int j = 0; j < nb; ++j) {
        if (threadIdx.x == 0) {
            const float d = a[j][j];
            if (!(d > 0.f)) *flag = 1;
            a[j][j] = sqrtf(fmaxf(d, 1e-30f));
        }
        __syncthreads();
        const float djj = a[j][j];
        for (int i = j + 1 + threadIdx.x; i < nb; i += blockDim.x) a[i][j] /= djj;
        __syncthreads();
        // trailing update of the block: a[i][k] -= a[i][j] a[k][j] for j < k <= i
        const int rem = nb - j - 1;
        for (int e = threadIdx.x; e < rem * rem; e += blockDim.x) {
            const int i = j + 1 + e / rem, k = j + 1 + e % rem;
            if (k <= i) a[i][k] -= a[i][j] * a[k][j];
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) {
        const int i = e / nb, k = e % nb;
        H[(k0 + i) * ld + k0 + k] = k <= i ? a[i][k] : 0.f;
    }
}

// For rows row0 .. row0+rows-1 of X (leading dimension ldx), columns c0 .. c0+nb-1:
//   UPPER = false:  x L_d^T = b  (forward: x_j = (b_j - sum_{k<j} x_k L_d[j][k]) / L_d[j][j])
//   UPPER = true:   x L_d   = b  (backward: x_j = (b_j - sum_{k>j} x_k L_d[k][j]) / L_d[j][j])
// with L_d the nb x nb lower-triangular block at (d0, d0) of L (leading dimension ldl).
// In place; one thread per row, L_d in shared memory.
template <bool UPPER>
__global__ void __launch_bounds__(128) trsm_rows_kernel(float* X, int64_t ldx, int64_t row0, int64_t rows, int64_t c0,
                                                        const float* L, int64_t ldl, int64_t d0) {
    __shared__ float ld_[kNB][kNB + 1];
    for (int e = threadIdx.x; e < kNB * kNB; e += blockDim.x) ld_[e / kNB][e % kNB] = L[(d0 + e / kNB) * ldl + d0 + e % kNB];
    __syncthreads();
    const int64_t i = row0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= row0 + rows) return;
    float* x = X + i * ldx + c0;
    float v[kNB];
#pragma unroll
    for (int j = 0; j < kNB; ++j) v[j] = x[j];
    if (!UPPER) {
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
            float s = v[j];
#pragma unroll
            for (int k = 0; k < j; ++k) s -= v[k] * ld_[j][k];
            v[j] = s / ld_[j][j];
        }
    } else {
#pragma unroll
        for (int j = kNB - 1; j >= 0; --j) {
            float s = v[j];
#pragma unroll
            for (int k = j + 1; k < kNB; ++k) s -= v[k] * ld_[k][j];
            v[j] = s / ld_[j][j];
        }
    }
#pragma unroll
    for (int j = 0; j < kNB; ++j) x[j] = v[j];
}

// H (r x r, lower triangle) = L L^T in place.
int cholesky(float* H, int64_t r, int* flag, cudaStream_t s) {
    for (int64_t k0 = 0; k0 < r; k0 += kNB) {
        potrf_diag_kernel<<<1, 256, 0, s>>>(H, r, k0, kNB, flag);
        const int64_t below = r - k0 - kNB;
        if (below <= 0) break;
        trsm_rows_kernel<false><<<(unsigned)((below + 127) / 128), 128, 0, s>>>(H, r, k0 + kNB, below, k0, H, r, k0);
        // H22 -= L21 L21^T (full square of the trailing block; only its lower triangle is read)
        GemmF32<float> g = gemm_args<float>(below, below, kNB, H + (k0 + kNB) * r + k0, r, H + (k0 + kNB) * r + k0, r,
                                            H + (k0 + kNB) * r + k0 + kNB, r);
        g.alpha = -1.f;
        g.beta = 1.f;
        g.D = g.C;
        g.ldd = r;
        if (gemm<float, false, true>(g, s) != NQ_OK) return NQ_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

// X (rows x r, leading dimension r) <- X L^-T: the forward half of a solve with L L^T.
int solve_lower_T(float* X, int64_t rows, const float* L, int64_t r, cudaStream_t s) {
    for (int64_t c0 = 0; c0 < r; c0 += kNB) {
        trsm_rows_kernel<false><<<(unsigned)((rows + 127) / 128), 128, 0, s>>>(X, r, 0, rows, c0, L, r, c0);
        const int64_t rest = r - c0 - kNB;
        if (rest <= 0) break;
        // X[:, c0+nb:] -= X[:, c0:c0+nb] L[c0+nb:, c0:c0+nb]^T
        GemmF32<float> g = gemm_args<float>(rows, rest, kNB, X + c0, r, L + (c0 + kNB) * r + c0, r, X + c0 + kNB, r);
        g.alpha = -1.f;
        g.beta = 1.f;
        g.D = g.C;
        g.ldd = r;
        if (gemm<float, false, true>(g, s) != NQ_OK) return NQ_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

// X (rows x r) <- X L^-1: the backward half.
int solve_lower(float* X, int64_t rows, const float* L, int64_t r, cudaStream_t s) {
    for (int64_t c0 = r - kNB; c0 >= 0; c0 -= kNB) {
        trsm_rows_kernel<true><<<(unsigned)((rows + 127) / 128), 128, 0, s>>>(X, r, 0, rows, c0, L, r, c0);
        if (c0 == 0) break;
        // X[:, :c0] -= X[:, c0:c0+nb] L[c0:c0+nb, :c0]
        GemmF32<float> g = gemm_args<float>(rows, c0, kNB, X + c0, r, L + c0 * r, r, X, r);
        g.alpha = -1.f;
        g.beta = 1.f;
        g.D = g.C;
        g.ldd = r;
        if (gemm<float, false, false>(g, s) != NQ_OK) return NQ_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

// ------------------------------------------------------------------ element-wise steps
// H += rho I with rho = lam * tr(H) / r (tr summed in index order by one thread); rho is
// kept in *rho_out for the least-squares right-hand side.
__global__ void add_penalty_kernel(float* H, int64_t r, float lam, float* rho_out) {
    __shared__ float rho;
    if (threadIdx.x == 0) {
        double tr = 0.0;
        for (int64_t k = 0; k < r; ++k) tr += (double)H[k * r + k];
        rho = (float)((double)lam * tr / (double)r);
        *rho_out = rho;
    }
    __syncthreads();
    for (int64_t k = threadIdx.x; k < r; k += blockDim.x) H[k * r + k] += rho;
}

// Pi and the dual: per row of M = X + L (or of X alone when `dual` is 0), the scale
// s = mean |M| (lanes add in a fixed order), Z = s sign(M) (sign(0) = +1) and
// L = M - Z (dual 1), or L = 0 (dual 0, the start).  One warp per row.
__global__ void project_kernel(const float* X, float* L, float* Z, float* sc, int64_t rows, int64_t r, int dual) {
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* x = X + row * r;
    float* l = L + row * r;
    float s = 0.f;
    for (int64_t k = lane; k < r; k += 32) s += fabsf(dual ? x[k] + l[k] : x[k]);
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    s /= (float)r;
    if (lane == 0) sc[row] = s;
    float* z = Z + row * r;
    for (int64_t k = lane; k < r; k += 32) {
        const float mv = dual ? x[k] + l[k] : x[k];
        const float zv = mv >= 0.f ? s : -s;
        z[k] = zv;
        l[k] = dual ? mv - zv : 0.f;
    }
}

// Column norms of A (m x r) and B (n x r), then A[:, k] *= c_k, B[:, k] /= c_k with
// c_k = sqrt(|B_k| / |A_k|).  One thread per column, rows in order.
__global__ void balance_columns_kernel(float* A, int64_t m, float* B, int64_t n, int64_t r) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= r) return;
    double na = 0.0, nb = 0.0;
    for (int64_t i = 0; i < m; ++i) na += (double)A[i * r + k] * A[i * r + k];
    for (int64_t j = 0; j < n; ++j) nb += (double)B[j * r + k] * B[j * r + k];
    const double c = (na > 0.0 && nb > 0.0) ? sqrt(sqrt(nb) / sqrt(na)) : 1.0;
    const float cf = (float)c, ci = (float)(1.0 / c);
    for (int64_t i = 0; i < m; ++i) A[i * r + k] *= cf;
    for (int64_t j = 0; j < n; ++j) B[j * r + k] *= ci;
}

// Magnitude balancing and the stored scales: c = sqrt(rms(sB) / rms(sA)) (sums of squares
// in index order), s1 = fp16(c sA), s2 = fp16(sB / c); the balanced fp32 values are kept
// in sA / sB.  One CTA.
__global__ void balance_scales_kernel(float* sA, int64_t m, float* sB, int64_t n, uint16_t* s1, uint16_t* s2) {
    __shared__ float cs[2];
    if (threadIdx.x == 0) {
        double a = 0.0, b = 0.0;
        for (int64_t i = 0; i < m; ++i) a += (double)sA[i] * sA[i];
        for (int64_t j = 0; j < n; ++j) b += (double)sB[j] * sB[j];
        const double ra = sqrt(a / (double)m), rb = sqrt(b / (double)n);
        const double c = (ra > 0.0 && rb > 0.0) ? sqrt(rb / ra) : 1.0;
        cs[0] = (float)c;
        cs[1] = (float)(1.0 / c);
    }
    __syncthreads();
    for (int64_t i = threadIdx.x; i < m; i += blockDim.x) {
        sA[i] *= cs[0];
        s1[i] = __half_as_ushort(__float2half_rn(sA[i]));
    }
    for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
        sB[j] *= cs[1];
        s2[j] = __half_as_ushort(__float2half_rn(sB[j]));
    }
}

// Z (rows x r) with its row scales rebuilt from the fp16 scales: Z[i][k] = s16[i] sign(Z[i][k]).
__global__ void rescale_rows_kernel(float* Z, const uint16_t* s16, int64_t rows, int64_t r) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= rows * r) return;
    const float s = __half2float(__ushort_as_half(s16[e / r]));
    Z[e] = Z[e] >= 0.f ? s : -s;
}

// Packed signs of Z (rows x r): bit b of word w of row i is Z[i][32w + b] >= 0.
__global__ void pack_rows_kernel(const float* Z, int64_t rows, int64_t r, uint32_t* out) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t wpr = r / 32;
    if (e >= rows * wpr) return;
    const float* z = Z + (e / wpr) * r + (e % wpr) * 32;
    uint32_t w = 0;
#pragma unroll
    for (int b = 0; b < 32; ++b) w |= (z[b] >= 0.f ? 1u : 0u) << b;
    out[e] = w;
}

// Sum of squares of a bf16 matrix, per CTA (fixed order), for the relative error.
__global__ void sumsq_bf16_kernel(const __nv_bfloat16* W, int64_t count, double* part) {
    __shared__ double red[256];
    double s = 0.0;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x) {
        const double v = (double)__bfloat162float(W[e]);
        s += v * v;
    }
    red[threadIdx.x] = s;
    __syncthreads();
    for (int k = 128; k > 0; k >>= 1) {
        if (threadIdx.x < k) red[threadIdx.x] += red[threadIdx.x + k];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[blockIdx.x] = red[0];
}

// ------------------------------------------------------------------ the steps on device state
struct AdmmState {
    int64_t m, n, r;
    const __nv_bfloat16* W;
    float *A, *B, *ZA, *ZB, *LA, *LB, *sA, *sB;
    float* R;     // max(m, n) x r
    float* H;     // r x r
    float* rho;   // device scalar
    int* flag;    // device: a Cholesky pivot was not positive
    // the iterations' products of W on the tensor cores (set when the call iterates)
    void* dscr = nullptr;          // a factor split into three bf16 parts: 3 max(m, n) x r
    unsigned* status = nullptr;    // bounded-wait timeouts of those products
};

int project(float* X, float* L, float* Z, float* sc, int64_t rows, int64_t r, int dual, cudaStream_t s) {
    project_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(X, L, Z, sc, rows, r, dual);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

// X = (Wop F + rho (Zx - Lx)) (F^T F + rho I)^-1 with rho = lam tr(F^T F) / r, then
// Zx = Pi(X + Lx), Lx += X - Zx.  TRANS: Wop = W^T (the B update).
template <bool TRANS>
int half_step(AdmmState& st, const float* F, int64_t frows, float* X, int64_t xrows, float* Zx, float* Lx, float* sx,
              float lam, cudaStream_t s) {
    const int64_t r = st.r;
    // H = F^T F + rho I
    GemmF32<float> g = gemm_args<float>(r, r, frows, F, r, F, r, st.H, r);
    if (gemm<float, true, false>(g, s) != NQ_OK) return NQ_ERR_CUDA;
    add_penalty_kernel<<<1, 256, 0, s>>>(st.H, r, lam, st.rho);
    int rc = cholesky(st.H, r, st.flag, s);
    if (rc != NQ_OK) return rc;
    // R = Wop F + rho (Zx - Lx), on the tensor cores: W in bf16 as given (exact), F as the
    // sum of three bf16 parts (fp32's precision), fp32 accumulation in a fixed order
    // (W^T read in place: W's rows are its columns)
    const int64_t K = TRANS ? st.m : st.n;
    if ((rc = dense_af(reinterpret_cast<const uint16_t*>(st.W), !TRANS, xrows, K, F, r, X, Zx, Lx, st.rho, st.dscr,
                       st.status, s)) != NQ_OK)
        return rc;
    if ((rc = solve_lower_T(X, xrows, st.H, r, s)) != NQ_OK) return rc;
    if ((rc = solve_lower(X, xrows, st.H, r, s)) != NQ_OK) return rc;
    return project(X, Lx, Zx, sx, xrows, r, 1, s);
}

int iterate(AdmmState& st, int iters, double lam0, double growth, cudaStream_t s) {
    double lam = lam0;
    for (int it = 0; it < iters; ++it) {
        int rc = half_step<false>(st, st.B, st.n, st.A, st.m, st.ZA, st.LA, st.sA, (float)lam, s);
        if (rc != NQ_OK) return rc;
        rc = half_step<true>(st, st.A, st.m, st.B, st.n, st.ZB, st.LB, st.sB, (float)lam, s);
        if (rc != NQ_OK) return rc;
        lam *= growth;
    }
    return NQ_OK;
}

// Q (rows x r) <- Q L^-T with L L^T = Q^T Q (Cholesky-QR).
int orthonormalize(AdmmState& st, float* Q, int64_t rows, cudaStream_t s) {
    GemmF32<float> g = gemm_args<float>(st.r, st.r, rows, Q, st.r, Q, st.r, st.H, st.r);
    if (gemm<float, true, false>(g, s) != NQ_OK) return NQ_ERR_CUDA;
    int rc = cholesky(st.H, st.r, st.flag, s);
    if (rc != NQ_OK) return rc;
    return solve_lower_T(Q, rows, st.H, st.r, s);
}

int init(AdmmState& st, const float* Omega, int q, cudaStream_t s) {
    const int64_t m = st.m, n = st.n, r = st.r;
    // A = orth(W Omega)
    GemmF32<__nv_bfloat16> g = gemm_args<__nv_bfloat16>(m, r, n, st.W, n, Omega, r, st.A, r);
    if (gemm<__nv_bfloat16, false, false>(g, s) != NQ_OK) return NQ_ERR_CUDA;
    int rc = orthonormalize(st, st.A, m, s);
    for (int k = 0; k < q && rc == NQ_OK; ++k) {
        GemmF32<__nv_bfloat16> t = gemm_args<__nv_bfloat16>(n, r, m, st.W, n, st.A, r, st.B, r);
        if (gemm<__nv_bfloat16, true, false>(t, s) != NQ_OK) return NQ_ERR_CUDA;
        GemmF32<__nv_bfloat16> y = gemm_args<__nv_bfloat16>(m, r, n, st.W, n, st.B, r, st.A, r);
        if (gemm<__nv_bfloat16, false, false>(y, s) != NQ_OK) return NQ_ERR_CUDA;
        rc = orthonormalize(st, st.A, m, s);
    }
    if (rc != NQ_OK) return rc;
    // B = W^T A, then equal column norms
    GemmF32<__nv_bfloat16> b = gemm_args<__nv_bfloat16>(n, r, m, st.W, n, st.A, r, st.B, r);
    if (gemm<__nv_bfloat16, true, false>(b, s) != NQ_OK) return NQ_ERR_CUDA;
    balance_columns_kernel<<<(unsigned)((r + 127) / 128), 128, 0, s>>>(st.A, m, st.B, n, r);
    if ((rc = project(st.A, st.LA, st.ZA, st.sA, m, r, 0, s)) != NQ_OK) return rc;
    return project(st.B, st.LB, st.ZB, st.sB, n, r, 0, s);
}

bool device_ptr(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeManaged || (a.type == cudaMemoryTypeDevice && a.device == dev);
}

int check_shape(int64_t m, int64_t n, int64_t r) {
    if (m <= 0 || n <= 0 || r <= 0 || m % 128 || n % 128 || r % 128 || m > (1 << 20) || n > (1 << 20) ||
        r > m || r > n || r > 16384)
        return NQ_ERR_SHAPE;
    return NQ_OK;
}

// Scratch owned by one call: R, H and the device scalars.
struct Scratch {
    char* base = nullptr;
    ~Scratch() {
        if (base) cudaFree(base);
    }
};

// dense: also the split-factor buffer of the iterations' tensor-core products.
int bind_scratch(AdmmState& st, Scratch& sc, bool dense = false) {
    const int64_t rows = st.m > st.n ? st.m : st.n;
    const size_t base_bytes = sizeof(float) * (size_t)(rows * st.r + st.r * st.r) + 256;
    const size_t d_bytes = dense ? (size_t)dense_af_scratch_bytes(rows, st.r) : 0;
    const size_t bytes = base_bytes + 256 + d_bytes;
    if (cudaMalloc(&sc.base, bytes) != cudaSuccess) {
        cudaGetLastError();
        sc.base = nullptr;
        return NQ_ERR_NOMEM;
    }
    st.R = reinterpret_cast<float*>(sc.base);
    st.H = st.R + rows * st.r;
    st.rho = st.H + st.r * st.r;
    st.flag = reinterpret_cast<int*>(st.rho + 4);
    st.status = reinterpret_cast<unsigned*>(st.flag + 1);
    if (dense) st.dscr = sc.base + (base_bytes + 255) / 256 * 256;
    return cudaMemset(st.flag, 0, 2 * sizeof(int)) == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;  // flag and status
}

int finish_flag(AdmmState& st, cudaStream_t s) {
    int flag[2] = {0, 0};  // the Cholesky flag, then the dense products' timeout word
    if (cudaMemcpyAsync(flag, st.flag, sizeof(flag), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return NQ_ERR_CUDA;
    if (flag[1]) return NQ_ERR_TIMEOUT;
    return flag[0] ? NQ_ERR_VALUE : NQ_OK;
}

}  // namespace
}  // namespace nq

using namespace nq;

extern "C" int nq_admm_iterate(const void* W, int64_t m, int64_t n, int64_t r, float* A, float* B, float* ZA, float* ZB,
                               float* LA, float* LB, float* sA, float* sB, int iters, double lam0, double growth,
                               void* stream) {
    int rc = check_shape(m, n, r);
    if (rc != NQ_OK) return rc;
    if (iters < 0 || !(lam0 > 0.0) || !(growth > 0.0)) return NQ_ERR_VALUE;
    if (!W || !A || !B || !ZA || !ZB || !LA || !LB || !sA || !sB) return NQ_ERR_NULL;
    const void* ptrs[] = {W, A, B, ZA, ZB, LA, LB, sA, sB};
    for (const void* p : ptrs)
        if (reinterpret_cast<uintptr_t>(p) & 15u) return NQ_ERR_ALIGN;
    for (const void* p : ptrs)
        if (!device_ptr(p)) return NQ_ERR_PTRKIND;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    AdmmState st{m, n, r, static_cast<const __nv_bfloat16*>(W), A, B, ZA, ZB, LA, LB, sA, sB, nullptr, nullptr, nullptr, nullptr};
    Scratch sc;
    if ((rc = bind_scratch(st, sc, true)) != NQ_OK) return rc;
    if ((rc = iterate(st, iters, lam0, growth, s)) != NQ_OK) return rc;
    return finish_flag(st, s);
}

extern "C" int nq_admm_init(const void* W, int64_t m, int64_t n, int64_t r, const float* Omega, int power_iters,
                            float* A, float* B, float* ZA, float* ZB, float* LA, float* LB, float* sA, float* sB,
                            void* stream) {
    int rc = check_shape(m, n, r);
    if (rc != NQ_OK) return rc;
    if (power_iters < 0 || power_iters > 64) return NQ_ERR_VALUE;
    if (!W || !Omega || !A || !B || !ZA || !ZB || !LA || !LB || !sA || !sB) return NQ_ERR_NULL;
    const void* ptrs[] = {W, Omega, A, B, ZA, ZB, LA, LB, sA, sB};
    for (const void* p : ptrs)
        if (reinterpret_cast<uintptr_t>(p) & 15u) return NQ_ERR_ALIGN;
    for (const void* p : ptrs)
        if (!device_ptr(p)) return NQ_ERR_PTRKIND;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    AdmmState st{m, n, r, static_cast<const __nv_bfloat16*>(W), A, B, ZA, ZB, LA, LB, sA, sB, nullptr, nullptr, nullptr, nullptr};
    Scratch sc;
    if ((rc = bind_scratch(st, sc)) != NQ_OK) return rc;
    if ((rc = init(st, Omega, power_iters, s)) != NQ_OK) return rc;
    return finish_flag(st, s);
}

extern "C" int nq_admm_factorize(const void* W, int64_t m, int64_t n, int64_t r, const float* Omega, int power_iters,
                                 int iters, double lam0, double growth, uint32_t* Upk, uint32_t* Vpk, void* s1,
                                 void* s2, double* rel_err, void* stream) {
    int rc = check_shape(m, n, r);
    if (rc != NQ_OK) return rc;
    if (power_iters < 0 || power_iters > 64 || iters < 0 || !(lam0 > 0.0) || !(growth > 0.0)) return NQ_ERR_VALUE;
    if (!W || !Omega || !Upk || !Vpk || !s1 || !s2) return NQ_ERR_NULL;
    const void* ptrs[] = {W, Omega, Upk, Vpk, s1, s2};
    for (const void* p : ptrs)
        if (reinterpret_cast<uintptr_t>(p) & 15u) return NQ_ERR_ALIGN;
    for (const void* p : ptrs)
        if (!device_ptr(p)) return NQ_ERR_PTRKIND;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the factors, projections, duals and scales of both sides, then R, H, scalars
    const size_t fa = (size_t)(m * r), fb = (size_t)(n * r);
    char* state = nullptr;
    const size_t tiles = (size_t)((m + kGM - 1) / kGM) * (size_t)((n + kGN - 1) / kGN);
    const size_t bytes = sizeof(float) * (3 * fa + 3 * fb + (size_t)m + (size_t)n) + sizeof(double) * (tiles + 1024) + 1024;
    if (cudaMalloc(&state, bytes) != cudaSuccess) {
        cudaGetLastError();
        return NQ_ERR_NOMEM;
    }
    struct Free {
        char* p;
        ~Free() { cudaFree(p); }
    } free_state{state};
    float* A = reinterpret_cast<float*>(state);
    float* ZA = A + fa;
    float* LA = ZA + fa;
    float* B = LA + fa;
    float* ZB = B + fb;
    float* LB = ZB + fb;
    float* sA = LB + fb;
    float* sB = sA + m;
    // m, n multiples of 128: sB + n is 512-byte aligned from the 256-byte aligned base
    double* part = reinterpret_cast<double*>(sB + n);
    AdmmState st{m, n, r, static_cast<const __nv_bfloat16*>(W), A, B, ZA, ZB, LA, LB, sA, sB, nullptr, nullptr, nullptr, nullptr};
    Scratch sc;
    if ((rc = bind_scratch(st, sc, true)) != NQ_OK) return rc;
    if ((rc = init(st, Omega, power_iters, s)) != NQ_OK) return rc;
    if ((rc = iterate(st, iters, lam0, growth, s)) != NQ_OK) return rc;
    balance_scales_kernel<<<1, 256, 0, s>>>(sA, m, sB, n, static_cast<uint16_t*>(s1), static_cast<uint16_t*>(s2));
    // the stored form: signs of Z_A (U, m x r/32) and of Z_B (V, n x r/32, then transposed
    // into the forward's layout V^T: r x n/32 in Vpk)
    pack_rows_kernel<<<(unsigned)((m * (r / 32) + 255) / 256), 256, 0, s>>>(ZA, m, r, Upk);
    uint32_t* Vrows = reinterpret_cast<uint32_t*>(st.R);  // n x r/32 words fit in R
    pack_rows_kernel<<<(unsigned)((n * (r / 32) + 255) / 256), 256, 0, s>>>(ZB, n, r, Vrows);
    if (cudaGetLastError() != cudaSuccess) return NQ_ERR_CUDA;
    if ((rc = transpose_device(Vrows, n, r, Vpk, s)) != NQ_OK) return rc;
    if (rel_err) {
        // ||W - diag(s1) U V^T diag(s2)||_F / ||W||_F with the stored fp16 scales: the
        // residual W - Z_A Z_B^T by a GEMM whose epilogue adds W and keeps only the tiles'
        // sums of squares; ||W||^2 by a reduction; both added up in double, in order
        rescale_rows_kernel<<<(unsigned)((fa + 255) / 256), 256, 0, s>>>(ZA, static_cast<const uint16_t*>(s1), m, r);
        rescale_rows_kernel<<<(unsigned)((fb + 255) / 256), 256, 0, s>>>(ZB, static_cast<const uint16_t*>(s2), n, r);
        GemmF32<float, __nv_bfloat16> e = gemm_args<float, __nv_bfloat16>(m, n, r, ZA, r, ZB, r, nullptr, 0);
        e.alpha = -1.f;
        e.beta = 1.f;
        e.D = static_cast<const __nv_bfloat16*>(W);
        e.ldd = n;
        e.sq = part;
        if (gemm<float, false, true, __nv_bfloat16>(e, s) != NQ_OK) return NQ_ERR_CUDA;
        constexpr int kSumBlocks = 1024;
        sumsq_bf16_kernel<<<kSumBlocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(W), m * n, part + tiles);
        if (cudaGetLastError() != cudaSuccess) return NQ_ERR_CUDA;
        std::vector<double> h(tiles + kSumBlocks);
        if (cudaMemcpyAsync(h.data(), part, sizeof(double) * h.size(), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return NQ_ERR_CUDA;
        double res = 0.0, tot = 0.0;
        for (size_t i = 0; i < tiles; ++i) res += h[i];
        for (size_t i = tiles; i < h.size(); ++i) tot += h[i];
        *rel_err = tot > 0.0 ? sqrt(res / tot) : 0.0;
    }
    return finish_flag(st, s);
}
