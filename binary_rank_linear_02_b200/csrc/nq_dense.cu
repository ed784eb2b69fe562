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
// Both operands are read where they lie, token-major ([K][M] and [K][R] rows): the tensor
// cores take MN-major shared-memory tiles (rows of 64 M or R elements along K), so neither
// a nor the split rank vectors are transposed.
// One CTA per 128 x 128 output tile: warp 0 loads A and B tiles by TMA (128-byte swizzle),
// warp 1 issues tcgen05.mma kind::f16 (bf16 operands, fp32 accumulators in tensor memory),
// warps 2-5 read the accumulators back (tcgen05.ld) and write s_i * acc.  Every mbarrier
// wait is bounded (NQ_ERR_TIMEOUT in the status word; the CTA drains and exits).
// The same kernel serves the LB-ADMM initialiser's products of W (bf16 input, exact; K-major
// for W F, MN-major for W^T F) with a factor F (fp32, split into three bf16 parts: fp32's
// precision), out = Wop F + rho (D - E), the penalty term folded into the epilogue.
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
constexpr int kDHalf = kDTileBytes / 2;           // one TMA box of an MN-major tile: 64 rows x 64 elements

// kind::f16 instruction descriptor: bf16 A and B (format 1), fp32 D, M x N; A and B K-major
// (0) or MN-major (1, bits 15 and 16).
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool amn, bool bmn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((amn ? 1u : 0u) << 15) | ((bmn ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// SW128 MN-major shared-memory operand descriptor: rows of 64 elements (128 B) along K,
// 8-row groups 1024 B apart (stride byte offset), the second 64-element block of the tile's
// 128 M (or N) elements one TMA box (8 KB) further (leading byte offset).
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)(kDHalf >> 4) << 16;  // leading byte offset: next 64-element block
    d |= (uint64_t)(1024 >> 4) << 32;    // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;              // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;              // 128-byte swizzle
    return d;
}

struct DenseBarriers {
    unsigned long long full[kDStages], empty[kDStages];
    unsigned long long tmem_full, drain;
    uint32_t tmem_base;
    int abort_flag;
};

// out[(m0 + i) * ldo + n0 + j] = s[m0 + i] * sum_k A[m0 + i][k] B[n0 + j][k] over nkb stages;
// A's stage kb reads K block kb % ka_blocks.  AMN / BMN: the operand's map is over [K][M]
// ([K][N]) rows, each stage two 64 x 64 boxes (MN-major), else over [M][K] ([N][K]) rows,
// one 128 x 64 box (K-major).
template <bool AMN, bool BMN>
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
                const int ka = kb % ka_blocks;
                if constexpr (AMN) {
                    tma_load_2d(dst, &amap, m0 / 2, ka * kDK, full);
                    tma_load_2d(dst + kDHalf, &amap, m0 / 2 + kDK / 2, ka * kDK, full);
                } else {
                    tma_load_2d(dst, &amap, ka * (kDK / 2), m0, full);
                }
                if constexpr (BMN) {
                    tma_load_2d(dst + kDTileBytes, &bmap, n0 / 2, kb * kDK, full);
                    tma_load_2d(dst + kDTileBytes + kDHalf, &bmap, n0 / 2 + kDK / 2, kb * kDK, full);
                } else {
                    tma_load_2d(dst + kDTileBytes, &bmap, kb * (kDK / 2), n0, full);
                }
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
            constexpr uint32_t idesc = idesc_bf16(kDM, kDN, AMN, BMN);
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int st = kb % kDStages;
                const uint32_t ph = (uint32_t)(kb / kDStages) & 1u;
                if (!mbar_wait(smem_u32(&bar.full[st]), ph, abort_flag, status)) break;
                tc_fence_after();
                const uint32_t aaddr = base + (uint32_t)(st * kDStageBytes), baddr = aaddr + kDTileBytes;
                const uint64_t ad = AMN ? sw128_desc_mn(aaddr) : sw128_desc(aaddr);
                const uint64_t bd = BMN ? sw128_desc_mn(baddr) : sw128_desc(baddr);
                // a K step of 16: 32 bytes along a K-major row, 16 rows (2 KB) of an MN-major tile
                constexpr uint64_t astep = AMN ? 2048 / 16 : 32 / 16, bstep = BMN ? 2048 / 16 : 32 / 16;
#pragma unroll
                for (int k = 0; k < kDK / 16; ++k)
                    umma_f16(tmem, ad + (uint64_t)k * astep, bd + (uint64_t)k * bstep, idesc, (kb > 0 || k > 0) ? 1u : 0u);
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

// The rank vectors (batch x R fp32, token-major) as the B operand's rows: dst[b][c] =
// bf16(v), dst[Bp + b][c] = bf16(v - bf16(v)) with v = src[b][c], zero rows for
// B <= b < Bp.  Two columns per thread.
__global__ void __launch_bounds__(256) split2_kernel(const float* __restrict__ src, int64_t B, int64_t C, int64_t Bp,
                                                     uint16_t* __restrict__ dst) {
    const int64_t pairs = Bp * C / 2;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < pairs; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = p / (C / 2), c = 2 * (p % (C / 2));
        const float2 v = b < B ? *reinterpret_cast<const float2*>(src + b * C + c) : make_float2(0.f, 0.f);
        const __nv_bfloat16 h0 = __float2bfloat16_rn(v.x), h1 = __float2bfloat16_rn(v.y);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(v.x - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(v.y - __bfloat162float(h1));
        *reinterpret_cast<uint32_t*>(dst + b * C + c) =
            (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        *reinterpret_cast<uint32_t*>(dst + (Bp + b) * C + c) =
            (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
}

// A factor (K x C fp32, row-major) as the B operand's rows in three bf16 parts: dst[q K + k][c]
// for q = 0, 1, 2 holds hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi - mid), whose sum
// carries v to ~2^-25 relative (fp32's own precision): for the ADMM products, whose sign
// projections and small-penalty solves amplify a two-part error.  Two columns per thread.
__global__ void __launch_bounds__(256) split3_kernel(const float* __restrict__ src, int64_t K, int64_t C,
                                                     uint16_t* __restrict__ dst) {
    const int64_t pairs = K * C / 2;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < pairs; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t k = p / (C / 2), c = 2 * (p % (C / 2));
        float2 v = *reinterpret_cast<const float2*>(src + k * C + c);
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(v.x), h1 = __float2bfloat16_rn(v.y);
            *reinterpret_cast<uint32_t*>(dst + ((int64_t)q * K + k) * C + c) =
                (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
            v.x -= __bfloat162float(h0);
            v.y -= __bfloat162float(h1);
        }
    }
}

// Maps over bf16 matrices (rows x cols elements, row pitch cols): encode_map_u32_sw128 takes
// 32-bit words (a row is cols / 2 words); TMA copies bytes, so the element type only sets
// the units.  K-major operand ([M][K] rows): boxes of 64 elements x 128 rows.  MN-major
// operand ([K][M] rows): boxes of 64 elements x 64 rows.
bool make_map_bf16(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols) {
    return encode_map_u32_sw128(map, ptr, rows, cols / 2, kDK / 2, kDM);
}
bool make_map_bf16_mn(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols) {
    return encode_map_u32_sw128(map, ptr, rows, cols / 2, kDK / 2, kDK);
}

}  // namespace

int64_t outer_tc_scratch_bytes(int64_t batch, int64_t M, int64_t R) {
    const int64_t Bp = (batch + kDPad - 1) / kDPad * kDPad;
    return 2 * (2 * Bp * R) + 256;
}

namespace {
template <bool AMN, bool BMN>
int dense_prepare() {
    static unsigned long long init_mask = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NQ_ERR_CUDA;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (cudaFuncSetAttribute(dense_gemm_kernel<AMN, BMN>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmem) !=
            cudaSuccess)
            return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    return NQ_OK;
}

// out (M x R, pitch R) = diag(s) A (sum of the parts of B)^T [+ rho (D - E)] over K = Kp per
// part.  A: AMN ? rows_a x M ([K][M], rows_a >= 1, rows past it read as zeros) : M x Kp
// ([M][K]); B: parts Kp x R ([K][R]) bf16.  M, R multiples of 128, Kp of 64.
template <bool AMN>
int dense_launch(const uint16_t* A, int64_t rows_a, const uint16_t* B, int parts, int64_t M, int64_t Kp, int64_t R,
                 float* out, const uint16_t* s, const float* D, const float* E, const float* rho, unsigned* status,
                 cudaStream_t stream) {
    int rc = dense_prepare<AMN, true>();
    if (rc != NQ_OK) return rc;
    CUtensorMap amap, bmap;
    if (!(AMN ? make_map_bf16_mn(&amap, A, rows_a, M) : make_map_bf16(&amap, A, M, Kp)) ||
        !make_map_bf16_mn(&bmap, B, parts * Kp, R))
        return NQ_ERR_CUDA;
    const int nkb = (int)(parts * Kp / kDK), ka_blocks = (int)(Kp / kDK);
    return launch_pdl(dense_gemm_kernel<AMN, true>, dim3((unsigned)(R / kDN), (unsigned)(M / kDM)), dim3(kDThreads),
                      (size_t)kDSmem, stream, amap, bmap, nkb, ka_blocks, out, R, s, D, E, rho, status) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}

unsigned split_grid(int64_t pairs) {
    const int64_t g = (pairs + 255) / 256, cap = 8 * (int64_t)sm_count();
    return (unsigned)(g < cap ? g : cap);
}
}  // namespace

int outer_tc(const uint16_t* a, const uint16_t* s, const float* t, int64_t batch, int64_t M, int64_t R, float* out,
             void* scratch, unsigned* status, cudaStream_t stream) {
    if (M % kDM || R % kDN || batch <= 0) return NQ_ERR_SHAPE;
    const int64_t Bp = (batch + kDPad - 1) / kDPad * kDPad;
    uint16_t* Bs = static_cast<uint16_t*>(scratch);  // 2 Bp x R: rows of hi, then rows of lo
    split2_kernel<<<split_grid(Bp * R / 2), 256, 0, stream>>>(t, batch, R, Bp, Bs);
    if (cudaGetLastError() != cudaSuccess) return NQ_ERR_CUDA;
    // a (batch x M, token-major) read in place: the token rows from batch to Bp are outside
    // the map and read as zeros
    return dense_launch<true>(a, batch, Bs, 2, M, Bp, R, out, s, nullptr, nullptr, nullptr, status, stream);
}

int64_t dense_af_scratch_bytes(int64_t K, int64_t R) { return 2 * (3 * K * R) + 256; }

int dense_af(const uint16_t* A, bool a_kmajor_rows, int64_t M, int64_t K, const float* F, int64_t R, float* out,
             const float* D, const float* E, const float* rho, void* scratch, unsigned* status, cudaStream_t stream) {
    if (M % kDM || R % kDN || K % kDK || K <= 0) return NQ_ERR_SHAPE;
    uint16_t* Bs = static_cast<uint16_t*>(scratch);  // 3K x R: rows of hi, mid, lo
    split3_kernel<<<split_grid(K * R / 2), 256, 0, stream>>>(F, K, R, Bs);
    if (cudaGetLastError() != cudaSuccess) return NQ_ERR_CUDA;
    return a_kmajor_rows ? dense_launch<false>(A, M, Bs, 3, M, K, R, out, nullptr, D, E, rho, status, stream)
                         : dense_launch<true>(A, K, Bs, 3, M, K, R, out, nullptr, D, E, rho, status, stream);
}

}  // namespace nq
