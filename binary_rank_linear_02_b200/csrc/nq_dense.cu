// nq_dense.cu -- dense tcgen05 GEMM for the factor gradients at calibration batch sizes.
//
// The straight-through refinement of the factorised components (hardwired.dev, "NanoQuant
// jednoduse", section "Krok 3") needs, per layer and per batch of calibration tokens,
//     dU[i][k] = s1_i sum_b dy[b][i] t[b][k]        (t = V^T (s2 (.) x), batch x r fp32)
//     dV[j][k] = s2_j sum_b x[b][j]  u[b][k]        (u = U^T (s1 (.) dy))
// a dense contraction over the tokens.  Here it runs on the 5th-generation tensor cores:
// out (M x R) = diag(s) . A . B^T with A = a^T (M x K, bfloat16, exact: a is bf16 input) and
// B = the rank vectors transposed (R x K).  The rank vectors are fp32, so B holds each as
// the sum of two bfloat16 numbers, hi = bf16(v) and lo = bf16(v - hi), in the two halves of
// a doubled K (the A tile is the same for both halves: its TMA coordinate wraps): a
// bf16 x bf16 product is exact in fp32, so the products carry ~2^-17 relative error of v.
// One CTA per 128 x 128 output tile: warp 0 loads A and B tiles by TMA (128-byte swizzle,
// K-major), warp 1 issues tcgen05.mma kind::f16 (bf16 operands, fp32 accumulators in tensor
// memory), warps 2-5 read the accumulators back (tcgen05.ld) and write s_i * acc.  Every
// mbarrier wait is bounded (NQ_ERR_TIMEOUT in the status word; the CTA drains and exits).
// The same kernel serves the LB-ADMM initialiser's products of W (bf16 input, exact) with a
// factor F (fp32, split into three bf16 parts: fp32's precision), out = W F + rho (D - E),
// the penalty term of the least-squares step folded into the epilogue.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "nq_internal.cuh"
#include "nq_sm100.cuh"

namespace nq {
namespace {

constexpr int kDM = 128, kDN = 128, kDK = 64;     // tile M, N; K per stage (128 bytes of bf16)
constexpr int kDStages = 3;
constexpr int kDTileBytes = kDM * kDK * 2;        // 16 KB (A and B tiles are the same size)
constexpr int kDStageBytes = 2 * kDTileBytes;
constexpr int kDThreads = 192;
constexpr int kDSmem = kDStages * kDStageBytes + 1024 /*barriers*/ + 1024 /*alignment slack*/;
constexpr int kDPad = 64;                         // tokens are padded to a multiple of this

// kind::f16 instruction descriptor: bf16 A and B (format 1), K-major both, fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

struct DenseBarriers {
    unsigned long long full[kDStages], empty[kDStages];
    unsigned long long tmem_full, drain;
    uint32_t tmem_base;
    int abort_flag;
};

// out[(m0 + i) * ldo + n0 + j] = s[m0 + i] * sum_k A[m0 + i][k] B[n0 + j][k] over nkb stages;
// A's stage kb reads K block kb % ka_blocks.
__global__ void __launch_bounds__(kDThreads, 2)
dense_gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap, int nkb,
                  int ka_blocks, float* __restrict__ out, int64_t ldo, const uint16_t* __restrict__ s,
                  const float* __restrict__ D, const float* __restrict__ E, const float* __restrict__ rho,
                  unsigned* __restrict__ status) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    DenseBarriers& bar = *reinterpret_cast<DenseBarriers*>(gbase + kDStages * kDStageBytes);
    volatile int* abort_flag = &bar.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // column tiles fastest: the CTAs resident at once share a few row panels of A, and all of
    // B (R x 2Bp bf16, 40 MB at r = 2432 and 4096 tokens) stays in L2 while A streams once
    const int n0 = blockIdx.x * kDN, m0 = blockIdx.y * kDM;

    if (threadIdx.x == 0) {
        for (int st = 0; st < kDStages; ++st) {
            mbar_init(smem_u32(&bar.full[st]), 1);
            mbar_init(smem_u32(&bar.empty[st]), 1);
        }
        mbar_init(smem_u32(&bar.tmem_full), 1);
        mbar_init(smem_u32(&bar.drain), 1);
        bar.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&amap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&bmap)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&bar.tmem_base)), "r"((uint32_t)kDN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            pdl_wait();  // A and B are written by the kernels before this one
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int st = kb % kDStages;
                const uint32_t ph = (uint32_t)(kb / kDStages) & 1u;
                if (!mbar_wait(smem_u32(&bar.empty[st]), ph ^ 1u, abort_flag, status)) break;
                const uint32_t full = smem_u32(&bar.full[st]);
                mbar_expect_tx(full, (uint32_t)kDStageBytes);
                const uint32_t dst = base + (uint32_t)(st * kDStageBytes);
                // x coordinates in 32-bit words of the maps (two bf16 each)
                tma_load_2d(dst, &amap, (kb % ka_blocks) * (kDK / 2), m0, full);
                tma_load_2d(dst + kDTileBytes, &bmap, kb * (kDK / 2), n0, full);
                ++issued;
            }
            if (*abort_flag) {
                for (int kb = issued - kDStages < 0 ? 0 : issued - kDStages; kb < issued; ++kb)
                    mbar_drain(smem_u32(&bar.full[kb % kDStages]), (uint32_t)(kb / kDStages) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kDM, kDN);
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int st = kb % kDStages;
                const uint32_t ph = (uint32_t)(kb / kDStages) & 1u;
                if (!mbar_wait(smem_u32(&bar.full[st]), ph, abort_flag, status)) break;
                tc_fence_after();
                const uint64_t ad = sw128_desc(base + (uint32_t)(st * kDStageBytes));
                const uint64_t bd = sw128_desc(base + (uint32_t)(st * kDStageBytes + kDTileBytes));
#pragma unroll
                for (int k = 0; k < kDK / 16; ++k)
                    umma_f16(tmem, ad + (uint64_t)(k * 16 * 2 / 16), bd + (uint64_t)(k * 16 * 2 / 16), idesc,
                             (kb > 0 || k > 0) ? 1u : 0u);
                umma_commit(smem_u32(&bar.empty[st]));
            }
            if (kb == nkb) {
                umma_commit(smem_u32(&bar.tmem_full));
            } else {
                umma_commit(smem_u32(&bar.drain));
                mbar_drain(smem_u32(&bar.drain), 0);
            }
        }
    } else {
        // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 = rows of the tile
        if (mbar_wait(smem_u32(&bar.tmem_full), 0, abort_flag, status)) {
            tc_fence_after();
            pdl_trigger();
            const int quad = warp & 3;
            const int row = m0 + quad * 32 + lane;
            const float sv = s ? __half2float(__ushort_as_half(s[row])) : 1.f;
            float* orow = out + (int64_t)row * ldo + n0;
#pragma unroll 1
            for (int c0 = 0; c0 < kDN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c0, v);
                if (D) {  // + rho (D - E), D and E laid out as out
                    const float rv = *rho;
                    const float* drow = D + (int64_t)row * ldo + n0 + c0;
                    const float* erow = E + (int64_t)row * ldo + n0 + c0;
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 d = *reinterpret_cast<const float4*>(drow + j);
                        const float4 e = *reinterpret_cast<const float4*>(erow + j);
                        *reinterpret_cast<float4*>(orow + c0 + j) = make_float4(
                            fmaf(rv, d.x - e.x, sv * __uint_as_float(v[j])), fmaf(rv, d.y - e.y, sv * __uint_as_float(v[j + 1])),
                            fmaf(rv, d.z - e.z, sv * __uint_as_float(v[j + 2])),
                            fmaf(rv, d.w - e.w, sv * __uint_as_float(v[j + 3])));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(orow + c0 + j) =
                            make_float4(sv * __uint_as_float(v[j]), sv * __uint_as_float(v[j + 1]),
                                        sv * __uint_as_float(v[j + 2]), sv * __uint_as_float(v[j + 3]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kDN));
    }
}

// dst[c][b] = src[b][c] (bf16) for b < B, 0 for B <= b < Bp: the K-major A operand from
// token-major activations.  64 x 64 tiles through shared memory (row pitch 65 halves: the
// column reads of the write-out fall in distinct banks), each thread moving two adjacent
// elements per access so that a warp reads and writes 128 contiguous bytes.
constexpr int kTT = 64;
__global__ void __launch_bounds__(256) transpose_pad_kernel(const uint16_t* __restrict__ src, int64_t B, int64_t C,
                                                            int64_t Bp, uint16_t* __restrict__ dst) {
    __shared__ uint16_t tile[kTT][kTT + 1];
    const int64_t c0 = (int64_t)blockIdx.x * kTT, b0 = (int64_t)blockIdx.y * kTT;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int k = ty; k < kTT; k += 8) {
        const int64_t b = b0 + k, c = c0 + 2 * tx;
        uint32_t v = 0;
        if (b < B && c < C) v = *reinterpret_cast<const uint32_t*>(src + b * C + c);
        tile[k][2 * tx] = (uint16_t)(v & 0xFFFFu);
        tile[k][2 * tx + 1] = (uint16_t)(v >> 16);
    }
    __syncthreads();
    for (int k = ty; k < kTT; k += 8) {
        const int64_t c = c0 + k, b = b0 + 2 * tx;
        if (c < C && b < Bp)
            *reinterpret_cast<uint32_t*>(dst + c * Bp + b) = (uint32_t)tile[2 * tx][k] | ((uint32_t)tile[2 * tx + 1][k] << 16);
    }
}

// dst[c][b] = bf16(v), dst[c][Bp + b] = bf16(v - bf16(v)) with v = src[b][c] (fp32), zeros for
// B <= b < Bp: the K-major B operand, each fp32 value as the sum of two bf16 numbers.  64 x 64
// tiles as above (row pitch 65 floats).
__global__ void __launch_bounds__(256) transpose_split_kernel(const float* __restrict__ src, int64_t B, int64_t C,
                                                              int64_t Bp, uint16_t* __restrict__ dst) {
    __shared__ float tile[kTT][kTT + 1];
    const int64_t c0 = (int64_t)blockIdx.x * kTT, b0 = (int64_t)blockIdx.y * kTT;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int k = ty; k < kTT; k += 8) {
        const int64_t b = b0 + k, c = c0 + 2 * tx;
        float2 v = make_float2(0.f, 0.f);
        if (b < B && c < C) v = *reinterpret_cast<const float2*>(src + b * C + c);
        tile[k][2 * tx] = v.x;
        tile[k][2 * tx + 1] = v.y;
    }
    __syncthreads();
    for (int k = ty; k < kTT; k += 8) {
        const int64_t c = c0 + k, b = b0 + 2 * tx;
        if (c < C && b < Bp) {
            uint32_t hi2 = 0, lo2 = 0;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float v = tile[2 * tx + e][k];
                const __nv_bfloat16 hi = __float2bfloat16_rn(v);
                const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
                hi2 |= (uint32_t)__bfloat16_as_ushort(hi) << (16 * e);
                lo2 |= (uint32_t)__bfloat16_as_ushort(lo) << (16 * e);
            }
            *reinterpret_cast<uint32_t*>(dst + c * 2 * Bp + b) = hi2;
            *reinterpret_cast<uint32_t*>(dst + c * 2 * Bp + Bp + b) = lo2;
        }
    }
}

// dst[c][b], dst[c][K + b], dst[c][2K + b] = the three bf16 parts of v = src[b][c] (fp32):
// hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi - mid), whose sum carries v to ~2^-25
// relative (fp32's own precision): for the ADMM products, whose sign projections and
// small-penalty solves amplify the two-part error.  B rows (K) a multiple of 64.
__global__ void __launch_bounds__(256) transpose_split3_kernel(const float* __restrict__ src, int64_t K, int64_t C,
                                                               uint16_t* __restrict__ dst) {
    __shared__ float tile[kTT][kTT + 1];
    const int64_t c0 = (int64_t)blockIdx.x * kTT, b0 = (int64_t)blockIdx.y * kTT;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int k = ty; k < kTT; k += 8) {
        const int64_t b = b0 + k, c = c0 + 2 * tx;
        float2 v = make_float2(0.f, 0.f);
        if (c < C) v = *reinterpret_cast<const float2*>(src + b * C + c);
        tile[k][2 * tx] = v.x;
        tile[k][2 * tx + 1] = v.y;
    }
    __syncthreads();
    for (int k = ty; k < kTT; k += 8) {
        const int64_t c = c0 + k, b = b0 + 2 * tx;
        if (c < C) {
            uint32_t p[3] = {0u, 0u, 0u};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float v = tile[2 * tx + e][k];
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const __nv_bfloat16 h = __float2bfloat16_rn(v);
                    p[q] |= (uint32_t)__bfloat16_as_ushort(h) << (16 * e);
                    v -= __bfloat162float(h);
                }
            }
#pragma unroll
            for (int q = 0; q < 3; ++q) *reinterpret_cast<uint32_t*>(dst + c * 3 * K + q * K + b) = p[q];
        }
    }
}

bool make_map_bf16(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols) {
    // encode_map_u32_sw128 takes 32-bit words: a bf16 row of `cols` is cols / 2 words, the
    // 64-element box 32 words; TMA copies bytes, so the element type only sets the units
    return encode_map_u32_sw128(map, ptr, rows, cols / 2, kDK / 2, kDM);
}

}  // namespace

int64_t outer_tc_scratch_bytes(int64_t batch, int64_t M, int64_t R) {
    const int64_t Bp = (batch + kDPad - 1) / kDPad * kDPad;
    return 2 * (M * Bp + R * 2 * Bp) + 256;
}

namespace {
int dense_prepare() {
    static unsigned long long init_mask = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NQ_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (cudaFuncSetAttribute(dense_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmem) != cudaSuccess)
            return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    return NQ_OK;
}

// out (M x R, pitch R) = diag(s) A (sum of the parts of Bt)^T [+ rho (D - E)]: A is M x Kp
// bf16 (K-major), Bt is R x parts Kp bf16 (the parts side by side), Kp a multiple of kDK.
int dense_launch(const uint16_t* A, const uint16_t* Bt, int parts, int64_t M, int64_t Kp, int64_t R, float* out,
                 const uint16_t* s, const float* D, const float* E, const float* rho, unsigned* status,
                 cudaStream_t stream) {
    CUtensorMap amap, bmap;
    if (!make_map_bf16(&amap, A, M, Kp) || !make_map_bf16(&bmap, Bt, R, parts * Kp)) return NQ_ERR_CUDA;
    const int nkb = (int)(parts * Kp / kDK), ka_blocks = (int)(Kp / kDK);
    return launch_pdl(dense_gemm_kernel, dim3((unsigned)(R / kDN), (unsigned)(M / kDM)), dim3(kDThreads), (size_t)kDSmem,
                      stream, amap, bmap, nkb, ka_blocks, out, R, s, D, E, rho, status) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}
}  // namespace

int outer_tc(const uint16_t* a, const uint16_t* s, const float* t, int64_t batch, int64_t M, int64_t R, float* out,
             void* scratch, unsigned* status, cudaStream_t stream) {
    if (M % kDM || R % kDN || batch <= 0) return NQ_ERR_SHAPE;
    const int64_t Bp = (batch + kDPad - 1) / kDPad * kDPad;
    uint16_t* At = static_cast<uint16_t*>(scratch);                      // M x Bp
    uint16_t* Bt = At + ((M * Bp + 127) / 128) * 128;                    // R x 2 Bp (hi | lo)
    int rc = dense_prepare();
    if (rc != NQ_OK) return rc;
    transpose_pad_kernel<<<dim3((unsigned)((M + kTT - 1) / kTT), (unsigned)(Bp / kTT)), 256, 0, stream>>>(a, batch, M,
                                                                                                       Bp, At);
    transpose_split_kernel<<<dim3((unsigned)((R + kTT - 1) / kTT), (unsigned)(Bp / kTT)), 256, 0, stream>>>(t, batch, R,
                                                                                                         Bp, Bt);
    if (cudaGetLastError() != cudaSuccess) return NQ_ERR_CUDA;
    return dense_launch(At, Bt, 2, M, Bp, R, out, s, nullptr, nullptr, nullptr, status, stream);
}

int64_t dense_af_scratch_bytes(int64_t K, int64_t R) { return 2 * (R * 3 * K) + 256; }

int dense_af(const uint16_t* A, int64_t M, int64_t K, const float* F, int64_t R, float* out, const float* D,
             const float* E, const float* rho, void* scratch, unsigned* status, cudaStream_t stream) {
    if (M % kDM || R % kDN || K % kDK || K <= 0) return NQ_ERR_SHAPE;
    uint16_t* Bt = static_cast<uint16_t*>(scratch);  // R x 3K (hi | mid | lo)
    int rc = dense_prepare();
    if (rc != NQ_OK) return rc;
    transpose_split3_kernel<<<dim3((unsigned)((R + kTT - 1) / kTT), (unsigned)(K / kTT)), 256, 0, stream>>>(F, K, R, Bt);
    if (cudaGetLastError() != cudaSuccess) return NQ_ERR_CUDA;
    return dense_launch(A, Bt, 3, M, K, R, out, nullptr, D, E, rho, status, stream);
}

int transpose_bf16_device(const uint16_t* src, int64_t rows, int64_t cols, uint16_t* dst, cudaStream_t stream) {
    if (rows % kTT || cols % kTT) return NQ_ERR_SHAPE;
    transpose_pad_kernel<<<dim3((unsigned)(cols / kTT), (unsigned)(rows / kTT)), 256, 0, stream>>>(src, rows, cols, rows,
                                                                                                dst);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

}  // namespace nq
