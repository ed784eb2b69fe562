// nq_decode.cu -- decode path (1 <= batch <= 8): two binary GEMV stages.
//
//   stage 1:  t_k = sum_j V[j][k] * (s2_j x_j)          (rows k of V^T, r of them)
//   stage 2:  y_i = s1_i * sum_k U[i][k] * t_k          (rows i of U, m of them)
//
// The product with a +1/-1 row is the binary GEMV of hardwired.dev section "Cisla"
// (custom binary GEMV/GEMM kernels) for the factorised weight of section "Jak
// NanoQuant funguje".  Both stages run the same core: a row of signs against a vector.
//
// Why integer tensor-core instructions.  At HBM speed a B200 SM must retire ~190 packed
// sign bits per clock but can issue only 4 warp instructions per clock, so unpacking a
// bit and adding +/-x on the CUDA cores (shift, sign flip, add: >= 3 ops per bit per
// token) caps a GEMV at a fraction of the bandwidth.  Here one LOP3 turns a word into
// four bytes that are 0 or 2^s (s = bit position inside each byte, a mask selects the
// bits s, s+8, s+16, s+24), and mma.sync m16n8k32 (u8 x s8 -> s32) multiplies 16 rows
// x 32 such bytes against the activation, which is quantised per column range to 14
// bits and split into two int8 limbs (hi, lo) that sit in the MMA's N dimension next to
// up to four tokens.  Integer accumulation is exact; the only rounding is the 14-bit
// quantisation of the activation (relative step 2^-14 of the range's largest entry).
//
// Since the A bytes are 0/1 (times 2^s), the MMA yields sum_j b_j q_j; the signed sum is
// sum_j (2 b_j - 1) q_j = 2 * sum_j b_j q_j - sum_j q_j, with sum_j q_j counted while
// quantising.
//
// Layout in one column block (CB) of 128 columns = 4 words per row: lane (g, t) of a
// warp (g = lane/4, t = lane%4) reads word t of rows g and g+8 of a 16-row tile.  For s
// in 0..3, A = { w & M_s, w(g+8) & M_s, (w>>4) & M_s, (w(g+8)>>4) & M_s } with
// M_s = 0x01010101 << s.  MMA K column 4t+c maps to column 32t + s + 8c of the CB and K
// column 16+4t+c to column 32t + s + 4 + 8c; the B fragments are built in that order.
// N column n = 2*token + limb (limb 0 = hi, 1 = lo), four tokens per "token group".
#include <cuda_fp16.h>
#include <math.h>

#include "nq_internal.cuh"

namespace nq {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCB = 128;           // columns per column block
constexpr int kChunk = 2048;       // columns quantised and staged per pass
constexpr int kChunkCB = kChunk / kCB;
constexpr int kQBits = 14;         // |q| < 2^14

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
__device__ __forceinline__ float f16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Exponent E with max < 2^E (0 for max == 0): values are quantised as rint(v * 2^(14-E)).
__device__ __forceinline__ int range_exponent(float max_abs) {
    int e = 0;
    if (max_abs > 0.f) frexpf(max_abs, &e);
    return e;
}

__device__ __forceinline__ int quantise(float v, int e) {
    float q = rintf(scalbnf(v, kQBits - e));
    q = fminf(fmaxf(q, -16384.f), 16383.f);
    return (int)q;
}

// Shared-memory staging of one chunk: q values (int16) and the B fragments.
struct ChunkSmem {
    int16_t q[8][kChunk];                  // 32 KB
    uint4 frag[kChunkCB][2][2][32];        // [cb][token group][half][lane] = 32 KB
};

// Build the B fragments of `ncb` column blocks from sq (tokens >= batch are zero).
__device__ void build_fragments(ChunkSmem& sm, int ncb, int batch, int ntg) {
    const int total = ncb * ntg * 32 * 8;  // fragment words
    for (int idx = threadIdx.x; idx < total; idx += kThreads) {
        const int j = idx & 7;             // 2*s + h
        const int lane = (idx >> 3) & 31;
        const int tg = (idx >> 8) % ntg;
        const int cb = (idx >> 8) / ntg;
        const int s = j >> 1, h = j & 1;
        const int t = lane & 3, tok = 4 * tg + (lane >> 3), limb = (lane >> 2) & 1;
        uint32_t word = 0;
        if (tok < batch) {
            const int16_t* qrow = sm.q[tok] + cb * kCB + 32 * t + s + 4 * h;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                int q = qrow[8 * c];
                uint32_t byte = limb == 0 ? (uint32_t)((q >> 7) & 0xFF) : (uint32_t)(q & 0x7F);
                word |= byte << (8 * c);
            }
        }
        reinterpret_cast<uint32_t*>(&sm.frag[cb][tg][j >> 2][lane])[j & 3] = word;
    }
}

// Accumulate one 16-row tile against column blocks [cb0, cb1) of the staged chunk.
// W points at word 0 of the tile's row 0 for the chunk; wpr = words per row.
template <int NTG>
__device__ __forceinline__ void tile_mma(const uint32_t* __restrict__ W, int64_t wpr, const ChunkSmem& sm,
                                         int cb0, int cb1, int cbstep, int (&acc)[NTG][4][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t* rg = W + (int64_t)g * wpr + t;
    const uint32_t* rg8 = rg + 8 * wpr;
    int cb = cb0;
    for (; cb + 3 * cbstep < cb1; cb += 4 * cbstep) {
        uint32_t wa[4], wb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            wa[u] = __ldg(rg + 4 * (cb + u * cbstep));
            wb[u] = __ldg(rg8 + 4 * (cb + u * cbstep));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = cb + u * cbstep;
            const uint32_t a4 = wa[u] >> 4, b4 = wb[u] >> 4;
#pragma unroll
            for (int tg = 0; tg < NTG; ++tg) {
                const uint4 f0 = sm.frag[c][tg][0][lane], f1 = sm.frag[c][tg][1][lane];
                const uint32_t bf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint32_t M = 0x01010101u << s;
                    mma_u8s8(acc[tg][s], wa[u] & M, wb[u] & M, a4 & M, b4 & M, bf[2 * s], bf[2 * s + 1]);
                }
            }
        }
    }
    for (; cb < cb1; cb += cbstep) {
        const uint32_t wa = __ldg(rg + 4 * cb), wb = __ldg(rg8 + 4 * cb);
        const uint32_t a4 = wa >> 4, b4 = wb >> 4;
#pragma unroll
        for (int tg = 0; tg < NTG; ++tg) {
            const uint4 f0 = sm.frag[cb][tg][0][lane], f1 = sm.frag[cb][tg][1][lane];
            const uint32_t bf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint32_t M = 0x01010101u << s;
                mma_u8s8(acc[tg][s], wa & M, wb & M, a4 & M, b4 & M, bf[2 * s], bf[2 * s + 1]);
            }
        }
    }
}

// sum_j b_j q_j for (row g, token 4tg+t) and (row g+8, same token) from the accumulators.
template <int NTG>
__device__ __forceinline__ void combine(const int (&acc)[NTG][4][4], int tg, int& row_g, int& row_g8) {
    int hi0 = 0, lo0 = 0, hi8 = 0, lo8 = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        hi0 += acc[tg][s][0] >> s;
        lo0 += acc[tg][s][1] >> s;
        hi8 += acc[tg][s][2] >> s;
        lo8 += acc[tg][s][3] >> s;
    }
    row_g = hi0 * 128 + lo0;
    row_g8 = hi8 * 128 + lo8;
}

__device__ __forceinline__ float block_max_token(float v, float* sred) {
    // max over the block of v for one token; sred has kWarps floats
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) sred[threadIdx.x >> 5] = v;
    __syncthreads();
    float m = sred[0];
    for (int w = 1; w < kWarps; ++w) m = fmaxf(m, sred[w]);
    return m;
}

struct Stage1Smem {
    ChunkSmem chunk;
    float v[8][kChunk];                    // 64 KB: s2 * x of the chunk
    float res[8][128];                     // finished sums of the CTA's 128 rows
    float red[kWarps];
    int e[8];
    int qsum[8];
    int last;
};

struct Stage2Smem {
    ChunkSmem chunk;
    int bq[128][8];                        // per (row of the CTA, token) sum_k b q
    int e[8];
    int qsum[8];
};

// ------------------------------------------------------------------ stage 1
// grid = (r/128 row groups, nsplit).  CTA (rg, sp) handles rows [128 rg, 128 rg + 128)
// of V^T against column blocks [sp*cps, (sp+1)*cps), staged kChunk columns at a time;
// warp w owns rows
// 128 rg + 16 w .. +16.  Each chunk has its own quantisation exponent per token, so
// the warp converts its integer sums to fp32 after every chunk.  With nsplit > 1 the
// CTAs of a row group leave fp32 partials; the last to arrive adds them in split order
// (deterministic) and writes t and the row group's max |t| per token.
template <int NTG>
__global__ void __launch_bounds__(kThreads) stage1_kernel(const uint16_t* __restrict__ x,
                                                          const uint32_t* __restrict__ Vpk,
                                                          const uint16_t* __restrict__ s2, int64_t n, int64_t r,
                                                          int batch, int nsplit, int cps, float* __restrict__ t,
                                                          float* __restrict__ tgmax, float* __restrict__ partials,
                                                          int* __restrict__ counters) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Stage1Smem& sm = *reinterpret_cast<Stage1Smem*>(smem_raw);
    const int rg = blockIdx.x, sp = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int64_t wpr = n / 32;
    const int64_t row0 = (int64_t)rg * 128 + 16 * warp;
    const int ncb_total = (int)(n / kCB);
    const int cbA = sp * cps, cbB = min(ncb_total, cbA + cps);

    float part[NTG][2];
#pragma unroll
    for (int tg = 0; tg < NTG; ++tg) part[tg][0] = part[tg][1] = 0.f;

    pdl_wait();  // x may come from the previous kernel on the stream

    for (int cbc = cbA; cbc < cbB; cbc += kChunkCB) {
        const int ncb = min(kChunkCB, cbB - cbc);
        const int64_t col0 = (int64_t)cbc * kCB;
        const int ccols = ncb * kCB;
        // stage s2 * x (exact in fp32) and its per-token max
        for (int tok = 0; tok < batch; ++tok) {
            float mx = 0.f;
            for (int c = threadIdx.x; c < ccols; c += kThreads) {
                float v = bf16_to_f32(x[(int64_t)tok * n + col0 + c]) * f16_to_f32(s2[col0 + c]);
                sm.v[tok][c] = v;
                mx = fmaxf(mx, fabsf(v));
            }
            mx = block_max_token(mx, sm.red);
            if (threadIdx.x == 0) {
                sm.e[tok] = range_exponent(mx);
                sm.qsum[tok] = 0;
            }
        }
        __syncthreads();
        for (int tok = 0; tok < batch; ++tok) {
            const int e = sm.e[tok];
            int qs = 0;
            for (int c = threadIdx.x; c < ccols; c += kThreads) {
                int q = quantise(sm.v[tok][c], e);
                sm.chunk.q[tok][c] = (int16_t)q;
                qs += q;
            }
            for (int o = 16; o > 0; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
            if (lane == 0) atomicAdd(&sm.qsum[tok], qs);
        }
        __syncthreads();
        build_fragments(sm.chunk, ncb, batch, NTG);
        __syncthreads();

        int acc[NTG][4][4];
#pragma unroll
        for (int tg = 0; tg < NTG; ++tg)
#pragma unroll
            for (int s = 0; s < 4; ++s)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[tg][s][i] = 0;
        tile_mma<NTG>(Vpk + row0 * wpr + col0 / 32, wpr, sm.chunk, 0, ncb, 1, acc);

#pragma unroll
        for (int tg = 0; tg < NTG; ++tg) {
            const int tok = 4 * tg + tq;
            if (tok < batch) {
                int bq0, bq8;
                combine<NTG>(acc, tg, bq0, bq8);
                const int64_t qs = sm.qsum[tok];
                const int e = sm.e[tok] - kQBits;
                part[tg][0] += scalbnf((float)(2 * (int64_t)bq0 - qs), e);
                part[tg][1] += scalbnf((float)(2 * (int64_t)bq8 - qs), e);
            }
        }
        __syncthreads();  // before the next chunk overwrites the staging
    }
    pdl_trigger();

#pragma unroll
    for (int tg = 0; tg < NTG; ++tg) {
        const int tok = 4 * tg + tq;
        if (tok < batch) {
            sm.res[tok][16 * warp + g] = part[tg][0];
            sm.res[tok][16 * warp + g + 8] = part[tg][1];
        }
    }
    __syncthreads();

    const int ngroups = (int)(r / 128);
    if (nsplit == 1) {
        for (int tok = 0; tok < batch; ++tok) {
            float mx = 0.f;
            for (int i = threadIdx.x; i < 128; i += kThreads) {
                float v = sm.res[tok][i];
                t[(int64_t)tok * r + (int64_t)rg * 128 + i] = v;
                mx = fmaxf(mx, fabsf(v));
            }
            mx = block_max_token(mx, sm.red);
            if (threadIdx.x == 0) tgmax[(int64_t)tok * ngroups + rg] = mx;
        }
        return;
    }

    for (int idx = threadIdx.x; idx < batch * 128; idx += kThreads) {
        const int tok = idx / 128, i = idx % 128;
        partials[((int64_t)sp * 8 + tok) * r + (int64_t)rg * 128 + i] = sm.res[tok][i];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        int prev = atomicAdd(&counters[rg], 1);
        sm.last = (prev == nsplit - 1);
    }
    __syncthreads();
    if (!sm.last) return;
    __threadfence();
    for (int tok = 0; tok < batch; ++tok) {
        float mx = 0.f;
        for (int i = threadIdx.x; i < 128; i += kThreads) {
            float sum = 0.f;
            for (int s = 0; s < nsplit; ++s)
                sum += __ldcg(&partials[((int64_t)s * 8 + tok) * r + (int64_t)rg * 128 + i]);
            t[(int64_t)tok * r + (int64_t)rg * 128 + i] = sum;
            mx = fmaxf(mx, fabsf(sum));
        }
        mx = block_max_token(mx, sm.red);
        if (threadIdx.x == 0) tgmax[(int64_t)tok * ngroups + rg] = mx;
    }
    if (threadIdx.x == 0) counters[rg] = 0;
}

// ------------------------------------------------------------------ stage 2
// CTA = RT row tiles x KS k-parts (RT * KS = 8 warps), rows [RT*16*blockIdx.x, +RT*16).
// One quantisation exponent per token for the whole of t (from the row-group maxima of
// stage 1), so integer sums run across all chunks and k-parts and are converted once.
template <int NTG, int RT>
__global__ void __launch_bounds__(kThreads) stage2_kernel(const float* __restrict__ t,
                                                          const float* __restrict__ tgmax,
                                                          const uint32_t* __restrict__ Upk,
                                                          const uint16_t* __restrict__ s1, int64_t m, int64_t r,
                                                          int batch, float* __restrict__ y) {
    constexpr int KS = kWarps / RT;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Stage2Smem& sm = *reinterpret_cast<Stage2Smem*>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int rt = warp / KS, kp = warp % KS;
    const int64_t wpr = r / 32;
    const int64_t rowc = (int64_t)blockIdx.x * RT * 16;
    const int64_t row0 = rowc + 16 * rt;
    const int ngroups = (int)(r / 128);
    const int nchunks = (int)((r + kChunk - 1) / kChunk);

    for (int i = threadIdx.x; i < 128 * 8; i += kThreads) (&sm.bq[0][0])[i] = 0;

    pdl_wait();  // t and tgmax come from stage 1

    if (threadIdx.x < 8) {
        const int tok = threadIdx.x;
        float mx = 0.f;
        if (tok < batch)
            for (int gi = 0; gi < ngroups; ++gi) mx = fmaxf(mx, tgmax[(int64_t)tok * ngroups + gi]);
        sm.e[tok] = range_exponent(mx);
        sm.qsum[tok] = 0;
    }
    __syncthreads();

    int acc[NTG][4][4];
#pragma unroll
    for (int tg = 0; tg < NTG; ++tg)
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[tg][s][i] = 0;

    for (int ch = 0; ch < nchunks; ++ch) {
        const int64_t col0 = (int64_t)ch * kChunk;
        const int ccols = (int)min((int64_t)kChunk, r - col0);
        const int ncb = ccols / kCB;
        for (int tok = 0; tok < batch; ++tok) {
            const int e = sm.e[tok];
            int qs = 0;
            for (int c = threadIdx.x; c < ccols; c += kThreads) {
                int q = quantise(t[(int64_t)tok * r + col0 + c], e);
                sm.chunk.q[tok][c] = (int16_t)q;
                qs += q;
            }
            for (int o = 16; o > 0; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
            if (lane == 0) atomicAdd(&sm.qsum[tok], qs);
        }
        __syncthreads();
        build_fragments(sm.chunk, ncb, batch, NTG);
        __syncthreads();
        if (row0 < m) tile_mma<NTG>(Upk + row0 * wpr + col0 / 32, wpr, sm.chunk, kp, ncb, KS, acc);
        __syncthreads();
    }
    pdl_trigger();

    if (row0 < m) {
#pragma unroll
        for (int tg = 0; tg < NTG; ++tg) {
            const int tok = 4 * tg + tq;
            if (tok < batch) {
                int bq0, bq8;
                combine<NTG>(acc, tg, bq0, bq8);
                atomicAdd(&sm.bq[16 * rt + g][tok], bq0);
                atomicAdd(&sm.bq[16 * rt + g + 8][tok], bq8);
            }
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < RT * 16 * batch; idx += kThreads) {
        const int tok = idx / (RT * 16), i = idx % (RT * 16);
        const int64_t row = rowc + i;
        if (row < m) {
            const float v = scalbnf((float)(2 * (int64_t)sm.bq[i][tok] - sm.qsum[tok]), sm.e[tok] - kQBits);
            y[(int64_t)tok * m + row] = f16_to_f32(s1[row]) * v;
        }
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

// Column split of stage 1: about two CTAs per SM over the r/128 row groups; returns the
// number of column blocks per split (cps) and the split count.
void decode_split(int64_t n, int64_t r, int* nsplit, int* cps) {
    const int64_t ncb = n / kCB;
    const int64_t groups = r / 128;
    int64_t want = (2 * (int64_t)sm_count() + groups - 1) / groups;
    if (want > 64) want = 64;
    if (want > ncb) want = ncb;
    if (want < 1) want = 1;
    int64_t c = (ncb + want - 1) / want;
    *cps = (int)c;
    *nsplit = (int)((ncb + c - 1) / c);
}

namespace {

template <int NTG>
int decode_launch(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                  const uint16_t* s2, int64_t m, int64_t n, int64_t r, int batch, float* y, Workspace* ws,
                  cudaStream_t stream) {
    static unsigned long long init_mask = 0;  // devices whose kernel attributes are set
    const size_t smem1 = sizeof(Stage1Smem), smem2 = sizeof(Stage2Smem);
    const unsigned long long bit = 1ull << (ws->device & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (set_smem(stage1_kernel<NTG>, smem1) != cudaSuccess || set_smem(stage2_kernel<NTG, 1>, smem2) != cudaSuccess ||
            set_smem(stage2_kernel<NTG, 2>, smem2) != cudaSuccess || set_smem(stage2_kernel<NTG, 4>, smem2) != cudaSuccess)
            return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    int nsplit = 1, cps = 1;
    decode_split(n, r, &nsplit, &cps);
    dim3 grid1((unsigned)(r / 128), (unsigned)nsplit);
    cudaError_t err = launch_pdl(stage1_kernel<NTG>, grid1, dim3(kThreads), smem1, stream, x, Vpk, s2, n, r, batch,
                                 nsplit, cps, ws->t, ws->tgmax, ws->partials, ws->counters);
    if (err != cudaSuccess) return NQ_ERR_CUDA;
    // stage 2: fewer rows (more k-parts) per CTA when m is small
    const int64_t tiles = m / 16, sms = sm_count();
    const int rt = tiles >= 8 * sms ? 4 : (tiles >= 2 * sms ? 2 : 1);
    dim3 grid2((unsigned)((m + 16 * rt - 1) / (16 * rt)));
    const float* t = ws->t;
    const float* tgmax = ws->tgmax;
    if (rt == 1)
        err = launch_pdl(stage2_kernel<NTG, 1>, grid2, dim3(kThreads), smem2, stream, t, tgmax, Upk, s1, m, r, batch, y);
    else if (rt == 2)
        err = launch_pdl(stage2_kernel<NTG, 2>, grid2, dim3(kThreads), smem2, stream, t, tgmax, Upk, s1, m, r, batch, y);
    else
        err = launch_pdl(stage2_kernel<NTG, 4>, grid2, dim3(kThreads), smem2, stream, t, tgmax, Upk, s1, m, r, batch, y);
    return err == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

}  // namespace

int decode_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                   const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                   Workspace* ws, cudaStream_t stream) {
    if (batch <= 4) return decode_launch<1>(x, Upk, Vpk, s1, s2, m, n, r, (int)batch, y, ws, stream);
    return decode_launch<2>(x, Upk, Vpk, s1, s2, m, n, r, (int)batch, y, ws, stream);
}

}  // namespace nq
