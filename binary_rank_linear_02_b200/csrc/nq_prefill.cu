// nq_prefill.cu -- prefill path (batch > 8): the factorised linear as two dense
// tensor-core GEMMs on tcgen05 (hardwired.dev section "Cisla": binary GEMM kernels).
//
//   prescale : x'[b][.] = fp16(s2 (.) x[b])                    (elementwise, K-permuted)
//   GEMM 1   : T[b][k]  = sum_j V^T[k][j] x'[b][j]             M = r, N = batch, K = n
//   GEMM 2   : y[b][i]  = s1_i * sum_k U[i][k] T[b][k]         M = m, N = batch, K = r
//
// Weights are the MMA's A operand (M = 128 rows per CTA), tokens its B operand (N = BN
// per CTA).  A is never stored expanded in memory: four "expander" warps read the packed
// sign words of their row, turn them into fp16 +1/-1 in registers and write the 128B-
// swizzled K-major tile the UMMA descriptor expects; B (x' or T, fp16) arrives by TMA.
// One thread issues tcgen05.mma (kind::f16, fp32 accumulators in tensor memory); the
// expander warps then read the accumulators back (tcgen05.ld) for the epilogue, which
// writes T as fp16 (GEMM 1) or y = s1 * acc as fp32 (GEMM 2).
//
// fp16, not bf16, operands: bf16 x is exact in fp16 over the normal range, +1/-1 are
// exact, and fp16 keeps 3 more mantissa bits of x' and T than bf16 would.  Dense fp16
// and bf16 rates are the same on tcgen05.
//
// K order.  A word holds 32 consecutive columns, bit b = column b.  One left shift by
// (15 - q) brings bit q to bit 15 and bit q+16 to bit 31, and one LOP3 turns those two
// sign positions into the fp16 pair (+-1, +-1): register q holds columns (q, q+16).  The
// MMA therefore sees each 32-column group in the order c0, c16, c1, c17, ..., c15, c31,
// and the B operands are stored in that order: the prescale writes x' permuted and
// GEMM 1's epilogue writes T permuted, so no extra pass is needed.
//
// Every wait on an mbarrier is bounded by the global timer (about 2 s); a wait that
// expires records NQ_ERR_TIMEOUT in the library's device status word, the CTA drains
// what it issued and returns (tensor memory is always freed).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "nq_internal.cuh"

namespace nq {
namespace {

constexpr int kBM = 128;          // rows of A per CTA (tcgen05 M)
constexpr int kBK = 64;           // K elements per stage: one 128-byte swizzle atom of fp16
constexpr int kUmmaK = 16;        // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192;     // warp 0 TMA, warp 1 MMA, warps 2..5 expand + epilogue
constexpr int kSmemBudget = 200 * 1024;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: false if the CTA aborted or the limit expired (then the CTA aborts).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* status) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicExch(status, (unsigned)(-NQ_ERR_TIMEOUT));
            return false;
        }
    }
}

// Time-bounded wait that ignores the abort flag: used to drain what this CTA issued.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = global_ns();
    while (!mbar_try(bar, parity) && global_ns() - t0 < kWaitLimitNs) {
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// SW128 K-major shared-memory operand descriptor: 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;            // leading byte offset 16 B (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;            // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;            // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: fp16 A and B, K-major both, fp32 D, M = 128, N = bn.
__host__ __device__ constexpr uint32_t idesc_f16(int bn) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Sixteen fp16 pairs (+-1) from one packed word: pair q = (column q, column q + 16).
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t (&h)[16]) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const uint32_t sh = w << (15 - q);
        // (sh & 0x80008000) ^ 0xBC00BC00: stored bit 1 -> 0x3C00 (+1), bit 0 -> 0xBC00 (-1).
        // LOP3 truth table of (a & b) ^ c with a = 0xF0, b = 0xCC, c = 0xAA: 0x6A.
        asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(h[q]) : "r"(sh), "r"(0x80008000u), "r"(0xBC00BC00u));
    }
}

// Position of natural column c inside its 32-group in the MMA's K order.
__host__ __device__ __forceinline__ int kperm(int c) { return c < 16 ? 2 * c : 2 * (c - 16) + 1; }

template <int BN>
struct Geometry {
    static constexpr int kABytes = kBM * kBK * 2;          // 16 KB per stage
    static constexpr int kBBytes = BN * kBK * 2;           // BN rows x 128 B
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = (kSmemBudget - 2048) / kStageBytes > 8 ? 8 : (kSmemBudget - 2048) / kStageBytes;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*barriers*/ + 1024 /*alignment slack*/;
    static constexpr int kTmemCols = BN < 32 ? 32 : BN;
};

struct Barriers {
    unsigned long long full_a[8], full_b[8], empty[8];
    unsigned long long tmem_full, drain;
    uint32_t tmem_base;
    int abort_flag;
};

// One CTA computes a 128 x BN tile of D = A . B^T with A = expanded signs (rows
// m0..m0+127 of `Wpk`, K = kdim) and B = TMA tiles of `bmap` (rows n0..n0+BN-1).
// EPI 0: T[b][perm(k)] = fp16(D) (GEMM 1);  EPI 1: y[b][i] = s1_i * D (GEMM 2).
template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap bmap, const uint32_t* __restrict__ Wpk, int64_t kdim,
            int64_t mdim, int64_t batch, uint16_t* __restrict__ T_out, float* __restrict__ y_out,
            const uint16_t* __restrict__ s1, unsigned* __restrict__ status) {
    using G = Geometry<BN>;
    constexpr int S = G::kStages;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    Barriers& bar = *reinterpret_cast<Barriers*>(gbase + S * G::kStageBytes);
    const uint32_t a_smem = base;                        // S stages of A
    const uint32_t b_smem = base + S * G::kABytes;       // S stages of B
    volatile int* abort_flag = &bar.abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.x * kBM;
    const int64_t n0 = (int64_t)blockIdx.y * BN;
    const int nkb = (int)(kdim / kBK);
    const int64_t wpr = kdim / 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&bar.full_a[s]), 128);
            mbar_init(smem_u32(&bar.full_b[s]), 1);
            mbar_init(smem_u32(&bar.empty[s]), 1);
        }
        mbar_init(smem_u32(&bar.tmem_full), 1);
        mbar_init(smem_u32(&bar.drain), 1);
        bar.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&bmap)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&bar.tmem_base)), "r"((uint32_t)G::kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer of the B tiles (activations)
        if (lane == 0) {
            pdl_wait();  // B comes from the previous kernel (prescale or GEMM 1)
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (uint32_t)(kb / S) & 1u;
                if (!mbar_wait(smem_u32(&bar.empty[s]), ph ^ 1u, abort_flag, status)) break;
                mbar_expect_tx(smem_u32(&bar.full_b[s]), (uint32_t)G::kBBytes);
                tma_load_2d(b_smem + s * G::kBBytes, &bmap, kb * kBK, (int)n0, smem_u32(&bar.full_b[s]));
                ++issued;
            }
            if (*abort_flag) {
                // let the loads already issued land before the CTA's shared memory goes away
                for (int kb = issued - S < 0 ? 0 : issued - S; kb < issued; ++kb)
                    mbar_drain(smem_u32(&bar.full_b[kb % S]), (uint32_t)(kb / S) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(BN);
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (uint32_t)(kb / S) & 1u;
                if (!mbar_wait(smem_u32(&bar.full_a[s]), ph, abort_flag, status)) break;
                if (!mbar_wait(smem_u32(&bar.full_b[s]), ph, abort_flag, status)) break;
                tc_fence_after();
                const uint64_t ad = sw128_desc(a_smem + s * G::kABytes);
                const uint64_t bd = sw128_desc(b_smem + s * G::kBBytes);
#pragma unroll
                for (int k = 0; k < kBK / kUmmaK; ++k)
                    umma_f16(tmem, ad + (uint64_t)(k * kUmmaK * 2 / 16), bd + (uint64_t)(k * kUmmaK * 2 / 16), idesc,
                             (kb > 0 || k > 0) ? 1u : 0u);
                umma_commit(smem_u32(&bar.empty[s]));
            }
            if (kb == nkb) {
                umma_commit(smem_u32(&bar.tmem_full));
            } else {
                // aborted: make sure the MMAs already issued are finished before teardown
                umma_commit(smem_u32(&bar.drain));
                mbar_drain(smem_u32(&bar.drain), 0);
            }
        }
    } else {
        // ---------------- expanders: one thread per A row, then the epilogue
        const int row = threadIdx.x - 64;                // 0..127
        const uint32_t* wrow = Wpk + (m0 + row) * wpr;
        const uint32_t a_row_off = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
        uint4 cur = make_uint4(0, 0, 0, 0), nxt = make_uint4(0, 0, 0, 0);
        // the packed row is read 4 words (two stages) at a time, one load ahead
        if (nkb > 0) cur = __ldg(reinterpret_cast<const uint4*>(wrow));
        if (nkb > 2) nxt = __ldg(reinterpret_cast<const uint4*>(wrow) + 1);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % S;
            const uint32_t ph = (uint32_t)(kb / S) & 1u;
            if (!mbar_wait(smem_u32(&bar.empty[s]), ph ^ 1u, abort_flag, status)) { ok = false; break; }
            const uint32_t w0 = (kb & 1) ? cur.z : cur.x;
            const uint32_t w1 = (kb & 1) ? cur.w : cur.y;
            uint32_t h0[16], h1[16];
            expand_word(w0, h0);
            expand_word(w1, h1);
            const uint32_t dst = a_smem + s * G::kABytes + a_row_off;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t* h = c < 4 ? h0 : h1;
                const int q = (c & 3) * 4;
                const uint32_t addr = dst + (uint32_t)(((c ^ (row & 7)) * 16));
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(h[q]), "r"(h[q + 1]),
                             "r"(h[q + 2]), "r"(h[q + 3])
                             : "memory");
            }
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(&bar.full_a[s]));
            if (kb & 1) {
                cur = nxt;
                if (kb + 3 < nkb) nxt = __ldg(reinterpret_cast<const uint4*>(wrow) + (kb + 3) / 2);
            }
        }
        if (ok && mbar_wait(smem_u32(&bar.tmem_full), 0, abort_flag, status)) {
            tc_fence_after();
            pdl_trigger();
            // epilogue: this warp owns TMEM lanes 32*(warp%4) .. +31 = rows of the tile
            const int quad = warp & 3;
            const int r_in_tile = quad * 32 + lane;
            const int64_t grow = m0 + r_in_tile;
            float s1v = 1.f;
            if (EPI == 1) s1v = __half2float(__ushort_as_half(s1[grow]));
            int64_t tcol = 0;
            if (EPI == 0) tcol = (grow & ~31ll) + kperm((int)(grow & 31));
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)c0, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int64_t b = n0 + c0 + j;
                    if (b < batch) {
                        const float d = __uint_as_float(v[j]);
                        if (EPI == 0)
                            T_out[b * mdim + tcol] = __half_as_ushort(__float2half_rn(d));
                        else
                            y_out[b * mdim + grow] = s1v * d;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)G::kTmemCols));
    }
}

// x'[b][perm(j)] = fp16(bf16 x[b][j] * fp16 s2[j]); one thread per 32-column group.
__global__ void prescale_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ s2, int64_t n,
                                int64_t batch, uint16_t* __restrict__ xp) {
    const int64_t groups = n / 32;
    const int64_t total = batch * groups;
    pdl_wait();
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = idx / groups, g = idx % groups;
        const uint4* xs = reinterpret_cast<const uint4*>(x + b * n + g * 32);
        const uint4* ss = reinterpret_cast<const uint4*>(s2 + g * 32);
        uint32_t xv[16], sv[16], out[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 a = __ldg(xs + i), c = __ldg(ss + i);
            xv[4 * i] = a.x; xv[4 * i + 1] = a.y; xv[4 * i + 2] = a.z; xv[4 * i + 3] = a.w;
            sv[4 * i] = c.x; sv[4 * i + 1] = c.y; sv[4 * i + 2] = c.z; sv[4 * i + 3] = c.w;
        }
        // column c sits in half (c & 1) of word c / 2; output pair q = (column q, column q+16)
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            uint32_t pair = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = q + 16 * h;
                const uint16_t xb = (uint16_t)(xv[c >> 1] >> (16 * (c & 1)));
                const uint16_t sb = (uint16_t)(sv[c >> 1] >> (16 * (c & 1)));
                const float v = __uint_as_float((uint32_t)xb << 16) * __half2float(__ushort_as_half(sb));
                pair |= (uint32_t)__half_as_ushort(__float2half_rn(v)) << (16 * h);
            }
            out[q] = pair;
        }
        uint4* o = reinterpret_cast<uint4*>(xp + b * n + g * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
    }
    pdl_trigger();
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2D fp16 tensor [rows][cols] (row-major), box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN>
int run_gemms(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1, const uint16_t* s2,
              int64_t m, int64_t n, int64_t r, int64_t batch, float* y, Workspace* ws, cudaStream_t stream) {
    using G = Geometry<BN>;
    static unsigned long long init_mask = 0;
    const unsigned long long bit = 1ull << (ws->device & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (cudaFuncSetAttribute(gemm_kernel<BN, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmemBytes) !=
                cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<BN, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmemBytes) !=
                cudaSuccess)
            return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    CUtensorMap map_x, map_t;
    if (!make_map(&map_x, ws->xprime, batch, n, BN) || !make_map(&map_t, ws->T, batch, r, BN)) return NQ_ERR_CUDA;

    const int64_t groups = batch * (n / 32);
    int pblocks = (int)((groups + 255) / 256);
    if (pblocks > 4 * sm_count()) pblocks = 4 * sm_count();
    if (launch_pdl(prescale_kernel, dim3(pblocks), dim3(256), 0, stream, x, s2, n, batch, ws->xprime) != cudaSuccess)
        return NQ_ERR_CUDA;
    const unsigned ntiles = (unsigned)((batch + BN - 1) / BN);
    if (launch_pdl(gemm_kernel<BN, 0>, dim3((unsigned)(r / kBM), ntiles), dim3(kThreads), (size_t)G::kSmemBytes,
                   stream, map_x, Vpk, n, r, batch, ws->T, (float*)nullptr, (const uint16_t*)nullptr,
                   ws->status + 1) != cudaSuccess)
        return NQ_ERR_CUDA;
    if (launch_pdl(gemm_kernel<BN, 1>, dim3((unsigned)(m / kBM), ntiles), dim3(kThreads), (size_t)G::kSmemBytes,
                   stream, map_t, Upk, r, m, batch, (uint16_t*)nullptr, y, s1, ws->status + 1) != cudaSuccess)
        return NQ_ERR_CUDA;
    return NQ_OK;
}

}  // namespace

int prefill_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                    const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                    Workspace* ws, cudaStream_t stream) {
    if (batch <= 64) return run_gemms<64>(x, Upk, Vpk, s1, s2, m, n, r, batch, y, ws, stream);
    if (batch <= 1024) return run_gemms<128>(x, Upk, Vpk, s1, s2, m, n, r, batch, y, ws, stream);
    return run_gemms<256>(x, Upk, Vpk, s1, s2, m, n, r, batch, y, ws, stream);
}

}  // namespace nq
