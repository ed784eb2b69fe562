// nq_decode.cu -- decode path (1 <= batch <= 8): two binary GEMV stages per layer.
//
//   stage 1:  t_k = sum_j V[j][k] * (s2_j x_j)          (rows k of V^T, r of them)
//   stage 2:  y_i = s1_i * sum_k U[i][k] * t_k          (rows i of U, m of them)
//
// The product with a +1/-1 row is the binary GEMV of hardwired.dev section "Cisla"
// (custom binary GEMV/GEMM kernels) for the factorised weight of section "Jak
// NanoQuant funguje".  Both stages run the same core: 16 rows of signs against a vector.
//
// Why integer tensor-core instructions.  At HBM speed a B200 SM must retire ~190 packed
// sign bits per clock but issues only 4 warp instructions per clock (and logic ops at
// half that rate), so unpacking a bit and adding +/-x on the CUDA cores (shift, sign
// flip, add: >= 3 ops per bit per token) caps a GEMV at a fraction of the bandwidth.
// Here one LOP3 turns a word into four bytes that are 0 or 2^s (a mask selects bits s,
// s+8, s+16, s+24), and mma.sync m16n8k32 (u8 x s8 -> s32) multiplies 16 rows x 32 such
// bytes against the activation, which is quantised per column chunk to 14 bits and split
// into two int8 limbs (hi, lo) that sit in the MMA's N dimension beside up to four
// tokens.  Integer accumulation is exact; the only rounding is the 14-bit quantisation of
// the activation (relative step 2^-14 of the chunk's largest entry).  Measured on a B200
// (sign bits multiplied per clock per SM): this path 189; mma.sync b1 AND-popc on the
// packed words ~41 once the activation's bit-planes are counted; tcgen05.mma kind::i8 with
// the sign bytes in tensor memory and N = 16 ~32 (a 16-wide N leaves it mostly idle).
//
// Since the A bytes are 0/1 (times 2^s), the MMA yields sum_j b_j q_j; the signed sum is
// sum_j (2 b_j - 1) q_j = 2 * sum_j b_j q_j - sum_j q_j, with sum_j q_j counted while
// quantising.
//
// Fragment layout in one column block (CB) of 128 columns = 4 words per row: lane (g, t)
// of a warp (g = lane/4, t = lane%4) takes word t of rows g and g+8 of a 16-row tile.
// For s in 0..3, A = { w & M_s, w(g+8) & M_s, (w>>4) & M_s, (w(g+8)>>4) & M_s } with
// M_s = 0x01010101 << s.  MMA K column 4t+c is column 32t + s + 8c of the CB and K column
// 16+4t+c is column 32t + s + 4 + 8c; the B fragments are built in that order.  N column
// n = 2*token + limb (limb 0 = hi, 1 = lo), four tokens per token group.
//
// Latency.  A decode layer moves 0.4-18 MB, a few microseconds at HBM speed, so the
// fixed costs decide.  Every CTA copies its weight rows into shared memory (cp.async)
// before it waits on the previous kernel (programmatic dependent launch) and lets the next
// kernel launch at once, so weight streaming overlaps the dependency chain.  Stage 1
// splits each 128-row block's columns so that every CTA stages one chunk; the last CTA of a
// block adds the partial sums in a fixed order (deterministic), or, where all of t fits one
// stage-2 span and the splits are few, every stage-1 CTA just stores its partial and each
// stage-2 CTA adds the partials itself in the same order.  Stage 2 runs as one even
// wave where it fits: each layer gets CTAs in proportion to its work, each CTA holds its
// rows of U and the whole of t on chip.  Several independent layers share one launch, the
// slowest first in the grid.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "nq_internal.cuh"
#include "nq_sm100.cuh"

namespace nq {
namespace {

constexpr int kThreads = 256;          // stage 2: 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kCB = 128;               // columns per column block
constexpr int kChunk = 1024;           // columns per fragment chunk
constexpr int kChunkCB = kChunk / kCB;
constexpr int kChunkWords = kChunk / 32;
constexpr int kQBits = 14;             // |q| < 2^14
constexpr int kRowsS1 = 128;           // stage-1 rows per CTA (8 warps x 1 tile or 4 warps x 2 tiles of 16)
constexpr int kS1Stride = kChunkWords + 4;  // words per staged stage-1 row (36: bank-spread)
constexpr int kSumBatch = 16;          // stage-1 split partials loaded at once by the reducing CTA
constexpr int kMaxK2 = 8;              // stage-2 CTAs per SM tried for a launch that fits in one wave
constexpr size_t kSmemPerSM = 228 * 1024;  // shared memory of one SM
constexpr size_t kSmemReserve = 1024;      // taken by the system from it for every resident CTA
constexpr int kWaveTiles2 = 8;         // stage-2 tiles per CTA of a launch that needs several waves
constexpr int kColMajorMinBatch = 3;   // one token group: the column-major fragment build from this many tokens
constexpr int kSumSlots = 4;           // stage 2 adding the split partials: float4 columns per thread (r <= 4096)
constexpr int kS2SumMaxSplits = 12;    // ... for groups whose layers have at most this many stage-1 splits

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
__device__ __forceinline__ float f16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Not volatile: the instruction only writes its registers, so the compiler may schedule it
// freely against the loads around it.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Quantisation exponent E of a range whose largest |value| is max_abs: max_abs < 2^E,
// clamped to [-100, 113] so that both 2^(14-E) and 2^(E-14) are normal floats.  Values
// are quantised as q = rint(v * 2^(14-E)), |q| <= 2^14, and dequantised by 2^(E-14); both
// scalings are exact.  (Inputs whose largest magnitude is below 2^-100 lose precision.)
__device__ __forceinline__ int range_exponent(float max_abs) {
    int e = 0;
    if (max_abs > 0.f) frexpf(max_abs, &e);
    return min(max(e, -100), 113);
}

__device__ __forceinline__ float pow2f(int k) { return __int_as_float((k + 127) << 23); }  // k in [-126, 127]

// |v * up| < 2^14 by the choice of E, so rounding gives at most 2^14: clamp the top only.
__device__ __forceinline__ int quantise(float v, float up) { return min(__float2int_rn(v * up), 16383); }

__device__ __forceinline__ float warp_max(float v) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// One layer of a decode launch (device view).
struct DecLayer {
    const uint16_t* x;
    const uint32_t* Upk;
    const uint32_t* Vpk;
    const uint16_t* s1;
    const uint16_t* s2;
    float* y;
    float* t;        // workspace: batch x r
    float* tgmax;    // workspace: batch x r/128 (max |t| per 128-row block)
    float* partials; // workspace: nsplit x batch x r (stage-1 column splits)
    int* counters;   // workspace: r/128 arrival counters, zero between calls
    uint16_t* y_bf16;     // optional bf16(y)
    uint16_t* y_norm;     // optional bf16(y / rms(y)) per token
    float* norm_partials; // workspace: batch x (stage-2 CTAs of the layer), sums of y^2
    int* norm_counter;    // workspace: stage-2 arrivals of the layer, zero between calls
    int m, n, r;
    int nsplit;      // stage 1: CTAs per 128-row block (column splits)
    int cps;         // stage 1: column blocks per split
    int s2_ctas;     // stage 2: CTAs of the layer, each an even share of its 16-row tiles
    int s2sum;       // 1: stage 2 adds up the layer's stage-1 split partials itself
};

struct DecGroup {
    DecLayer L[kMaxGroup];
    int count;
    int batch;
    int depth1;       // stage-1 chunk ring depth (1 or 2)
    int r2;           // stage-2 columns held on chip at a time (a multiple of kCB)
    int w2words;      // stage-2 weight buffer: the most rows x words per row of one CTA
    int rows2;        // stage-2 rows held on chip: 16 x the most tiles of one CTA
    int per_sm2;      // stage-2 CTAs per SM of a one-wave plan (no more may share an SM), else 0
    int t_global;     // stage 2 builds its B fragments from t in global memory (no staged copy)
    // CTA ranges in launch order: range k holds CTAs s1_start[k] .. s1_start[k+1]-1 of layer
    // s1_layer[k] (likewise for stage 2); the host puts the slowest layers first
    int s1_start[kMaxGroup + 1];
    int s2_start[kMaxGroup + 1];
    unsigned char s1_layer[kMaxGroup];
    unsigned char s2_layer[kMaxGroup];
    // streaming stage 2 (stage2s_kernel): prefixes over the layers in their own order of
    // 128-row units (u_start) and of their 1024-column stages (st_start)
    int stream2;
    int u_start[kMaxGroup + 1];
    int st_start[kMaxGroup + 1];
};

// The range of `block` (an index into start[]).
__device__ __forceinline__ int find_range(const int* start, int count, int block) {
    int k = 0;
    while (k + 1 < count && block >= start[k + 1]) ++k;
    return k;
}

// ------------------------------------------------------------------ shared memory
// Sized per launch (ring depth, batch, ranks), so a CTA holds only what it uses.
struct Misc {
    float red[kWarps][8];
    int e[8];
    float up[8];             // 2^(14 - e): quantisation factor per token
    int qsum[8];
    int last;
};

// B fragments: per (column block, token group, half) one uint4 for each of the 32 lanes.
// (Storing only the lanes that hold tokens, and loading under a lane predicate, measured
// slower: the unconditional 16-byte loads keep the MMA loop free of branches.)
__host__ __device__ inline size_t frag_bytes(int ncb, int ntg) { return (size_t)ncb * ntg * 2 * 32 * 16; }

// stage 1: w [depth][128][36] | x [depth][batch + 1][1024] bf16 (slot batch = s2; after the
// last chunk its start holds res [batch][128] f32, the CTA's sums of its rows) | frag (8 CBs) | misc
__host__ __device__ inline size_t s1_w_bytes(int depth) { return (size_t)depth * kRowsS1 * kS1Stride * 4; }
__host__ __device__ inline size_t s1_x_bytes(int depth, int batch) { return (size_t)depth * (batch + 1) * kChunk * 2; }
__host__ __device__ inline size_t s1_bytes(int depth, int batch, int ntg) {
    return s1_w_bytes(depth) + s1_x_bytes(depth, batch) + frag_bytes(kChunkCB, ntg) + sizeof(Misc);
}
// stage 2: w [rows][stride(r)] | t [batch][r2] f32 | frag (all r2/128 CBs) | bq [rows2][batch] | s1 [rows2] | misc
// Words per staged row of a layer of rank r: the first span's words, plus 4 when that is an
// even number of 4-word groups (an odd number spreads the 8 rows a warp reads over all
// 32 banks).
__host__ __device__ inline int s2_stride(int r, int r2) {
    const int cols = r < r2 ? r : r2;
    return cols / 32 + (((cols / 128) % 2) ? 0 : 4);
}
// t is staged with 8 floats of padding after every 32, so that the four columns 32 apart
// that a fragment task reads fall in different banks
__host__ __device__ inline int s2_t_row(int r2) { return r2 + r2 / 4; }
__host__ __device__ inline size_t s2_t_bytes(int batch, int r2) { return (size_t)batch * s2_t_row(r2) * 4; }
__host__ __device__ inline size_t s2_bq_bytes(int rows2, int batch) { return ((size_t)rows2 * batch * 4 + 15) / 16 * 16; }
__host__ __device__ inline size_t s2_s1_bytes(int rows2) { return ((size_t)rows2 * 2 + 15) / 16 * 16; }
// (t_global: no staged copy of t)
__host__ __device__ inline size_t s2_bytes(int w2words, int rows2, int batch, int r2, int ntg, bool t_global = false) {
    return (size_t)w2words * 4 + (t_global ? 0 : s2_t_bytes(batch, r2)) + frag_bytes(r2 / kCB, ntg) +
           s2_bq_bytes(rows2, batch) + s2_s1_bytes(rows2) + sizeof(Misc);
}

template <int NTG>
__device__ __forceinline__ uint4* frag_ptr(uint4* frag, int cb, int tg, int half, int lane) {
    return frag + ((cb * NTG + tg) * 2 + half) * 32 + lane;
}

// Zero every slot: those of lanes without a token (tokens >= batch) are never written.
template <int NTG, int NT>
__device__ __forceinline__ void zero_fragments(uint4* frag, int ncb) {
    for (int i = threadIdx.x; i < ncb * NTG * 2 * 32; i += NT) frag[i] = make_uint4(0, 0, 0, 0);
}

// B fragments of `ncb` column blocks from the fp32 values val(tok, col) (col from the span's
// first column), quantised with up[tok]; adds each token's sum of q to qsum.  Per token,
// one task = (cb, word t of the CB, fragment word j = 2s + h): the 4 columns
// 32t + s + 4h + 8c (c in 0..3) give word j of two lanes, the hi-limb lane 8*tok' + t and
// the lo-limb lane 8*tok' + 4 + t (tok' = token within its group).  Each thread adds up its
// q's of the token; one warp reduction per token and warp.
template <int NTG, int NT, typename Val>
__device__ __forceinline__ void build_fragments(uint4* frag, Misc& mi, Val val, int ncb, int batch) {
    const int tasks = ncb * 32;
    for (int tok = 0; tok < batch; ++tok) {
        const float up = mi.up[tok];
        const int tg = tok >> 2, ti = tok & 3;
        int qs = 0;
        for (int task = threadIdx.x; task < tasks; task += NT) {
            const int j = task & 7, t = (task >> 3) & 3, cb = task >> 5;
            const int s4 = j >> 1, h = j & 1;
            const int col = cb * kCB + 32 * t + s4 + 4 * h;
            uint32_t wh = 0, wl = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int q = quantise(val(tok, col + 8 * c), up);
                qs += q;
                wh |= (uint32_t)((q >> 7) & 0xFF) << (8 * c);
                wl |= (uint32_t)(q & 0x7F) << (8 * c);
            }
            // word j lives in half j >> 2 at component j & 3
            reinterpret_cast<uint32_t*>(frag_ptr<NTG>(frag, cb, tg, j >> 2, 8 * ti + t))[j & 3] = wh;
            reinterpret_cast<uint32_t*>(frag_ptr<NTG>(frag, cb, tg, j >> 2, 8 * ti + 4 + t))[j & 3] = wl;
        }
        for (int o = 16; o > 0; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
        if ((threadIdx.x & 31) == 0 && qs != 0) atomicAdd(&mi.qsum[tok], qs);
    }
}

// The same fragments and sums for two token groups (5..8 tokens), column-major: a thread
// forms each of its columns' scale once and quantises every token of the column, with the
// per-token sums of q in registers and one warp reduction per token at the end (fewer
// instructions than one pass per token).  value = val(tok, col) * scale(col).
template <int NTG, int NT, typename Val, typename Scale>
__device__ __forceinline__ void build_fragments2(uint4* frag, Misc& mi, Val val, Scale scale, int ncb, int batch) {
    constexpr int kTok = 4 * NTG;
    const int tasks = ncb * 32;
    int qs[kTok];
    float up[kTok];
#pragma unroll
    for (int tok = 0; tok < kTok; ++tok) {
        qs[tok] = 0;
        up[tok] = tok < batch ? mi.up[tok] : 0.f;
    }
    for (int task = threadIdx.x; task < tasks; task += NT) {
        const int j = task & 7, t = (task >> 3) & 3, cb = task >> 5;
        const int s4 = j >> 1, h = j & 1;
        const int col = cb * kCB + 32 * t + s4 + 4 * h;
        float sc[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[c] = scale(col + 8 * c);
#pragma unroll
        for (int tok = 0; tok < kTok; ++tok) {
            if (tok < batch) {
                uint32_t wh = 0, wl = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int q = quantise(val(tok, col + 8 * c) * sc[c], up[tok]);
                    qs[tok] += q;
                    wh |= (uint32_t)((q >> 7) & 0xFF) << (8 * c);
                    wl |= (uint32_t)(q & 0x7F) << (8 * c);
                }
                const int tg = tok >> 2, ti = tok & 3;
                reinterpret_cast<uint32_t*>(frag_ptr<NTG>(frag, cb, tg, j >> 2, 8 * ti + t))[j & 3] = wh;
                reinterpret_cast<uint32_t*>(frag_ptr<NTG>(frag, cb, tg, j >> 2, 8 * ti + 4 + t))[j & 3] = wl;
            }
        }
    }
#pragma unroll
    for (int tok = 0; tok < kTok; ++tok) {
        if (tok < batch) {
            int v = qs[tok];
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if ((threadIdx.x & 31) == 0 && v != 0) atomicAdd(&mi.qsum[tok], v);
        }
    }
}

// build_fragments for one token, reading t from global memory instead of a staged copy:
// each thread takes up to four tasks per round and issues all their loads before
// quantising, so that the round costs one L2 round trip.  Same values, layout and sums as
// build_fragments at batch 1.
template <int NT>
__device__ __forceinline__ void build_fragments_t1(uint4* frag, Misc& mi, const float* __restrict__ t, int ncb) {
    const int tasks = ncb * 32;
    const float up = mi.up[0];
    int qs = 0;
    for (int t0 = threadIdx.x; t0 < tasks; t0 += 4 * NT) {
        float v[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int task = t0 + u * NT;
            const int j = task & 7, tt = (task >> 3) & 3, cb = task >> 5;
            const int col = cb * kCB + 32 * tt + (j >> 1) + 4 * (j & 1);
#pragma unroll
            for (int c = 0; c < 4; ++c) v[u][c] = task < tasks ? __ldcg(t + col + 8 * c) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int task = t0 + u * NT;
            if (task < tasks) {
                const int j = task & 7, tt = (task >> 3) & 3, cb = task >> 5;
                uint32_t wh = 0, wl = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int q = quantise(v[u][c], up);
                    qs += q;
                    wh |= (uint32_t)((q >> 7) & 0xFF) << (8 * c);
                    wl |= (uint32_t)(q & 0x7F) << (8 * c);
                }
                reinterpret_cast<uint32_t*>(frag_ptr<1>(frag, cb, 0, j >> 2, tt))[j & 3] = wh;
                reinterpret_cast<uint32_t*>(frag_ptr<1>(frag, cb, 0, j >> 2, 4 + tt))[j & 3] = wl;
            }
        }
    }
    for (int o = 16; o > 0; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
    if ((threadIdx.x & 31) == 0 && qs != 0) atomicAdd(&mi.qsum[0], qs);
}

// One column block of a 16-row tile into accumulator set `acc`.
template <int NTG>
__device__ __forceinline__ void cb_mma(const uint4* frag, uint32_t wa, uint32_t wb, int cb, int lane,
                                       int (&acc)[NTG][4][4]) {
    const uint32_t a4 = wa >> 4, b4 = wb >> 4;
#pragma unroll
    for (int tg = 0; tg < NTG; ++tg) {
        const uint4 f0 = *frag_ptr<NTG>(const_cast<uint4*>(frag), cb, tg, 0, lane);
        const uint4 f1 = *frag_ptr<NTG>(const_cast<uint4*>(frag), cb, tg, 1, lane);
        const uint32_t bf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint32_t M = 0x01010101u << s;
            mma_u8s8(acc[tg][s], wa & M, wb & M, a4 & M, b4 & M, bf[2 * s], bf[2 * s + 1]);
        }
    }
}

// Accumulate one 16-row tile against column blocks cb0 .. cb1-1 of the span's fragments.
// wrow points at the tile's row 0, word 0 of the span; rows are `stride` words apart.  Two
// accumulator sets alternate between consecutive column blocks so that dependent MMAs are
// two blocks apart.
template <int NTG>
__device__ __forceinline__ void tile_mma(const uint4* frag, const uint32_t* wrow, int stride, int cb0, int cb1,
                                         int (&acc)[NTG][4][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t* wa_row = wrow + g * stride + t;
    const uint32_t* wb_row = wa_row + 8 * stride;
    int acc2[NTG][4][4];
#pragma unroll
    for (int tg = 0; tg < NTG; ++tg)
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc2[tg][s][i] = 0;
    int cb = cb0;
    for (; cb + 1 < cb1; cb += 2) {
        const uint32_t wa0 = wa_row[4 * cb], wb0 = wb_row[4 * cb];
        const uint32_t wa1 = wa_row[4 * (cb + 1)], wb1 = wb_row[4 * (cb + 1)];
        cb_mma<NTG>(frag, wa0, wb0, cb, lane, acc);
        cb_mma<NTG>(frag, wa1, wb1, cb + 1, lane, acc2);
    }
    if (cb < cb1) cb_mma<NTG>(frag, wa_row[4 * cb], wb_row[4 * cb], cb, lane, acc);
#pragma unroll
    for (int tg = 0; tg < NTG; ++tg)
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[tg][s][i] += acc2[tg][s][i];
}

// Two 16-row tiles (rows wrow0.., wrow1..) against column blocks cb0 .. cb1-1 at once: each
// column block's B fragments are loaded once for both tiles, and the tiles' accumulators
// give eight independent MMA chains per column block.
template <int NTG>
__device__ __forceinline__ void tile_pair_mma(const uint4* frag, const uint32_t* wrow0, const uint32_t* wrow1,
                                              int stride, int cb0, int cb1, int (&acc0)[NTG][4][4],
                                              int (&acc1)[NTG][4][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t* a0 = wrow0 + g * stride + t;
    const uint32_t* a1 = wrow1 + g * stride + t;
    for (int cb = cb0; cb < cb1; ++cb) {
        const uint32_t wa0 = a0[4 * cb], wb0 = a0[8 * stride + 4 * cb];
        const uint32_t wa1 = a1[4 * cb], wb1 = a1[8 * stride + 4 * cb];
        const uint32_t x0 = wa0 >> 4, y0 = wb0 >> 4, x1 = wa1 >> 4, y1 = wb1 >> 4;
#pragma unroll
        for (int tg = 0; tg < NTG; ++tg) {
            const uint4 f0 = *frag_ptr<NTG>(const_cast<uint4*>(frag), cb, tg, 0, lane);
            const uint4 f1 = *frag_ptr<NTG>(const_cast<uint4*>(frag), cb, tg, 1, lane);
            const uint32_t bf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint32_t M = 0x01010101u << s;
                mma_u8s8(acc0[tg][s], wa0 & M, wb0 & M, x0 & M, y0 & M, bf[2 * s], bf[2 * s + 1]);
                mma_u8s8(acc1[tg][s], wa1 & M, wb1 & M, x1 & M, y1 & M, bf[2 * s], bf[2 * s + 1]);
            }
        }
    }
}

// sum_j b_j q_j for (row g, token 4tg+t) and (row g+8, same token).
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

template <int NTG>
__device__ __forceinline__ void zero_acc(int (&acc)[NTG][4][4]) {
#pragma unroll
    for (int tg = 0; tg < NTG; ++tg)
#pragma unroll
        for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[tg][s][i] = 0;
}

// ------------------------------------------------------------------ stage 1
// CTA = 128 rows of V^T of one layer x one column split (cps column blocks, staged kChunk
// columns at a time).  TPW = 1: eight warps, warp w owns the 16-row tile 16w..16w+15 (the
// launch fits in one wave at four CTAs per SM).  TPW = 2: four warps of fewer registers,
// warp w owns rows 32w..32w+31 as two tiles multiplied together, sharing each column
// block's B fragments (more CTAs per SM for launches of several waves, and for two token
// groups, where one tile per warp would need twice the registers).  Each chunk has its own
// quantisation exponent per token, so the warp converts its integer sums to fp32 after
// every chunk.  With several splits, the CTAs of a row block leave fp32 partials and the
// last to arrive adds them in split order (deterministic), then writes t and the block's
// max |t| per token (stage 2 builds its exponent from those maxima).
template <int TPW>
__host__ __device__ constexpr int s1_threads() { return 32 * kRowsS1 / (16 * TPW); }

// CM: the column-major fragment build (always for two token groups; for one token group the
// host picks it from kColMajorMinBatch tokens.  Measured per 7B step: 3 tokens 21.7 -> 21.3
// us, 4 tokens 23.9 -> 22.6 us, 70B block at 4 tokens 65.9 -> 63.1 us; 2 tokens 17.3 against
// 17.4 us, and a single token slower with it, so those keep the token-major build)
template <int NTG, int TPW, bool CM = false>
__global__ void __launch_bounds__(s1_threads<TPW>(), TPW == 1 ? 4 : (NTG == 1 ? 8 : 4))
stage1_kernel(const __grid_constant__ DecGroup grp) {
    constexpr int kThreads1 = s1_threads<TPW>(), kWarps1 = kThreads1 / 32;
    constexpr bool kColMajor1 = NTG == 2 || CM;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int batch = grp.batch, depth = grp.depth1;
    uint32_t* wbuf = reinterpret_cast<uint32_t*>(smem_raw);
    uint16_t* xbuf = reinterpret_cast<uint16_t*>(smem_raw + s1_w_bytes(depth));  // [depth][batch + 1][kChunk]
    uint4* frag = reinterpret_cast<uint4*>(smem_raw + s1_w_bytes(depth) + s1_x_bytes(depth, batch));
    Misc& mi = *reinterpret_cast<Misc*>(reinterpret_cast<unsigned char*>(frag) + frag_bytes(kChunkCB, NTG));
    float(*res)[kRowsS1] = reinterpret_cast<float(*)[kRowsS1]>(xbuf);  // after the last chunk

    const int rk = find_range(grp.s1_start, grp.count, blockIdx.x);
    const DecLayer& L = grp.L[grp.s1_layer[rk]];
    const int local = blockIdx.x - grp.s1_start[rk];
    const int rb = local / L.nsplit, sp = local % L.nsplit;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int n = L.n, r = L.r;
    const int64_t wpr = n / 32;
    const int64_t row0 = (int64_t)rb * kRowsS1;
    const uint32_t* W = L.Vpk + row0 * wpr;
    const int cbA = min(n / kCB, sp * L.cps), cbB = min(n / kCB, cbA + L.cps);
    const int nchunks = (cbB - cbA + kChunkCB - 1) / kChunkCB;
    auto chunk_cb = [&](int ch) { return min(kChunkCB, cbB - cbA - ch * kChunkCB); };
    auto wchunk = [&](int buf) { return wbuf + (size_t)buf * kRowsS1 * kS1Stride; };
    auto xchunk = [&](int buf, int tok) { return xbuf + ((size_t)buf * (batch + 1) + tok) * kChunk; };

    auto fetch_w = [&](int ch) {  // weight rows of chunk ch into buffer ch % depth: lane p of a warp takes piece p of a row
        const int per_row = chunk_cb(ch);  // 16-byte pieces (one per column block), at most 8
        uint32_t* dst = wchunk(ch % depth);
        const uint32_t* src = W + (int64_t)(cbA + ch * kChunkCB) * 4;
        const int p = threadIdx.x & 7;
        if (p < per_row)
            for (int row = threadIdx.x >> 3; row < kRowsS1; row += kThreads1 / 8)
                cp_async16(dst + row * kS1Stride + 4 * p, src + row * wpr + 4 * p);
    };
    // x rows (batch of them) of chunk ch, and (a weight, fetched with the sign words) s2 of
    // chunk ch in slot `batch`
    auto fetch_xs = [&](int ch, const uint16_t* base, int64_t tok_stride, int tok0, int tok1) {
        const int per_tok = chunk_cb(ch) * kCB / 8;
        const int col0 = (cbA + ch * kChunkCB) * kCB;
        for (int tok = tok0; tok < tok1; ++tok) {
            const uint16_t* src = base + (int64_t)(tok - tok0) * tok_stride + col0;
            for (int p = threadIdx.x; p < per_tok; p += kThreads1) cp_async16(xchunk(ch % depth, tok) + 8 * p, src + 8 * p);
        }
    };
    auto fetch_x = [&](int ch) { fetch_xs(ch, L.x, n, 0, batch); };
    auto fetch_s2 = [&](int ch) { fetch_xs(ch, L.s2, 0, batch, batch + 1); };

    // weights first: they do not depend on the previous kernel
    if (nchunks > 0) {
        fetch_w(0);
        fetch_s2(0);
    }
    cp_async_commit();
    if (nchunks > 1) {
        fetch_w(1);
        fetch_s2(1);
    }
    cp_async_commit();
    if (nchunks > 2 && threadIdx.x < kRowsS1)
        prefetch_l2(W + threadIdx.x * wpr + (cbA + 2 * kChunkCB) * 4, (uint32_t)((cbB - cbA - 2 * kChunkCB) * 16));
    zero_fragments<NTG, kThreads1>(frag, kChunkCB);
    pdl_trigger();
    pdl_wait();  // x may come from the previous kernel on the stream
    if (nchunks > 0) fetch_x(0);
    cp_async_commit();
    if (nchunks > 1) fetch_x(1);
    cp_async_commit();

    float part[TPW][NTG][2];  // [tile][token group][row g / g+8]
#pragma unroll
    for (int tl = 0; tl < TPW; ++tl)
#pragma unroll
        for (int tg = 0; tg < NTG; ++tg) part[tl][tg][0] = part[tl][tg][1] = 0.f;

    for (int ch = 0; ch < nchunks; ++ch) {
        const int buf = ch % depth;
        const int ncb = chunk_cb(ch);
        const int ccols = ncb * kCB;
        if (ch + 1 < nchunks) cp_async_wait<1>(); else cp_async_wait<0>();
        __syncthreads();
        // v = s2 * x (exact in fp32, formed again when the fragments are built) and its
        // per-token max: every thread takes a column stripe of every token, then the warps'
        // maxima are combined
        const uint16_t* ss = xchunk(buf, batch);
        auto val = [&](int tok, int c) { return bf16_to_f32(xchunk(buf, tok)[c]) * f16_to_f32(ss[c]); };
        if constexpr (kColMajor1) {  // column-major: each column's scale once for all tokens
            float mxv[4 * NTG];
#pragma unroll
            for (int tok = 0; tok < 4 * NTG; ++tok) mxv[tok] = 0.f;
            for (int c = threadIdx.x; c < ccols; c += kThreads1) {
                const float sc = f16_to_f32(ss[c]);
#pragma unroll
                for (int tok = 0; tok < 4 * NTG; ++tok)
                    if (tok < batch) mxv[tok] = fmaxf(mxv[tok], fabsf(bf16_to_f32(xchunk(buf, tok)[c]) * sc));
            }
#pragma unroll
            for (int tok = 0; tok < 4 * NTG; ++tok) {
                if (tok < batch) {
                    const float mx = warp_max(mxv[tok]);
                    if (lane == 0) mi.red[warp][tok] = mx;
                }
            }
        } else {
            for (int tok = 0; tok < batch; ++tok) {
                float mx = 0.f;
                for (int c = threadIdx.x; c < ccols; c += kThreads1) mx = fmaxf(mx, fabsf(val(tok, c)));
                mx = warp_max(mx);
                if (lane == 0) mi.red[warp][tok] = mx;
            }
        }
        __syncthreads();
        if (threadIdx.x < batch) {
            const int tok = threadIdx.x;
            float mx = mi.red[0][tok];
            for (int w = 1; w < kWarps1; ++w) mx = fmaxf(mx, mi.red[w][tok]);
            const int e = range_exponent(mx);
            mi.e[tok] = e;
            mi.up[tok] = pow2f(kQBits - e);
            mi.qsum[tok] = 0;
        }
        __syncthreads();
        if constexpr (kColMajor1)
            build_fragments2<NTG, kThreads1>(
                frag, mi, [&](int tok, int c) { return bf16_to_f32(xchunk(buf, tok)[c]); },
                [&](int c) { return f16_to_f32(ss[c]); }, ncb, batch);
        else
            build_fragments<NTG, kThreads1>(frag, mi, val, ncb, batch);
        __syncthreads();

        int acc[TPW][NTG][4][4];
        const uint32_t* wt = wchunk(buf) + 16 * TPW * warp * kS1Stride;  // the warp's first tile
        zero_acc<NTG>(acc[0]);
        if constexpr (TPW == 1) {
            tile_mma<NTG>(frag, wt, kS1Stride, 0, ncb, acc[0]);
        } else {
            zero_acc<NTG>(acc[1]);
            tile_pair_mma<NTG>(frag, wt, wt + 16 * kS1Stride, kS1Stride, 0, ncb, acc[0], acc[1]);
        }
#pragma unroll
        for (int tl = 0; tl < TPW; ++tl) {
#pragma unroll
            for (int tg = 0; tg < NTG; ++tg) {
                const int tok = 4 * tg + tq;
                if (tok < batch) {
                    int bq0, bq8;
                    combine<NTG>(acc[tl], tg, bq0, bq8);
                    const int64_t qs = mi.qsum[tok];
                    const float down = pow2f(mi.e[tok] - kQBits);
                    part[tl][tg][0] += (float)(2 * (int64_t)bq0 - qs) * down;
                    part[tl][tg][1] += (float)(2 * (int64_t)bq8 - qs) * down;
                }
            }
        }
        __syncthreads();  // buffers are free again
        if (ch + 2 < nchunks) {
            fetch_w(ch + 2);
            fetch_s2(ch + 2);
            fetch_x(ch + 2);
            cp_async_commit();
        }
    }

    // this CTA's sums for its 128 rows, into shared memory (over the x buffer, no longer read)
#pragma unroll
    for (int tl = 0; tl < TPW; ++tl)
#pragma unroll
        for (int tg = 0; tg < NTG; ++tg) {
            const int tok = 4 * tg + tq;
            if (tok < batch) {
                res[tok][16 * (TPW * warp + tl) + g] = part[tl][tg][0];
                res[tok][16 * (TPW * warp + tl) + g + 8] = part[tl][tg][1];
            }
        }
    __syncthreads();
    if (L.s2sum) {  // stage 2 adds the splits up: this CTA's sums are its split's partial of t
        float* dst = L.nsplit > 1 ? L.partials + (int64_t)sp * batch * r : L.t;
        for (int i = threadIdx.x; i < batch * kRowsS1; i += kThreads1) {
            const int tok = i / kRowsS1, k = i % kRowsS1;
            dst[(int64_t)tok * r + row0 + k] = res[tok][k];
        }
        return;
    }
    const int nrb = r / kRowsS1;
    if (L.nsplit > 1) {
        for (int i = threadIdx.x; i < batch * kRowsS1; i += kThreads1) {
            const int tok = i / kRowsS1, k = i % kRowsS1;
            L.partials[((int64_t)sp * batch + tok) * r + row0 + k] = res[tok][k];
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();  // the CTA's partials (ordered before by the barrier) are visible first
            mi.last = (atomicAdd(&L.counters[rb], 1) == L.nsplit - 1);
            if (mi.last) __threadfence();
        }
        __syncthreads();
        if (!mi.last) return;
        for (int i = threadIdx.x; i < batch * kRowsS1; i += kThreads1) {
            const int tok = i / kRowsS1, k = i % kRowsS1;
            const float* pp = L.partials + (int64_t)tok * r + row0 + k;
            const int64_t stride = (int64_t)batch * r;
            float sum = 0.f;
            for (int q0 = 0; q0 < L.nsplit; q0 += kSumBatch) {  // up to kSumBatch loads in flight
                float pv[kSumBatch];
#pragma unroll
                for (int q = 0; q < kSumBatch; ++q) pv[q] = q0 + q < L.nsplit ? __ldcg(pp + (q0 + q) * stride) : 0.f;
#pragma unroll
                for (int q = 0; q < kSumBatch; ++q)
                    if (q0 + q < L.nsplit) sum += pv[q];
            }
            res[tok][k] = sum;
        }
        if (threadIdx.x == 0) L.counters[rb] = 0;
        __syncthreads();
    }
    // t and the block's max |t| per token (one warp per token)
    for (int tok = warp; tok < batch; tok += kWarps1) {
        float v = 0.f;
#pragma unroll
        for (int q = 0; q < kRowsS1 / 32; ++q) {
            const float a = res[tok][lane + 32 * q];
            L.t[(int64_t)tok * r + row0 + lane + 32 * q] = a;
            v = fmaxf(v, fabsf(a));
        }
        v = warp_max(v);
        if (lane == 0) L.tgmax[(int64_t)tok * nrb + rb] = v;
    }
}

// ------------------------------------------------------------------ stage 2
// The launch has about k CTAs per SM (k = 2 when they fit); each layer gets CTAs in
// proportion to its work (16-row tiles x column blocks) and each CTA an even share of its
// layer's tiles, so that every CTA, and every SM, has about the same work.  The CTA's weight
// rows for up to r2 columns are copied on chip before the dependency wait, and t for those
// columns right after it; the warps split the CTA's (tile, column block) units into even
// runs.  One quantisation exponent per token for the whole of t (from stage 1's maxima), so
// integer sums run across all column blocks and warps and are converted once.
// Row-wise RMS normalisation of a layer's whole output, folded into stage 2: every CTA
// adds up y^2 over its rows per token (fixed order) into the workspace, and the CTA that
// arrives last adds those partial sums in CTA order (deterministic), then rounds
// y * (1 / sqrt(sum / m)) to bf16 for the whole layer.  Same result as rms_norm_kernel up
// to the order of the sum of squares.
template <typename YAt>
__device__ void rms_norm_epilogue(const DecLayer& L, int batch, int rows, int blk, Misc& mi, YAt y_at) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = L.s2_ctas;
    if (warp < batch) {  // one warp per token (batch <= 8 = warps)
        float ss = 0.f;
        for (int i = lane; i < rows; i += 32) {
            const float yv = y_at(warp, i);
            ss = fmaf(yv, yv, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) L.norm_partials[(int64_t)warp * nblk + blk] = ss;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        mi.last = atomicAdd(L.norm_counter, 1) == nblk - 1;
    }
    __syncthreads();
    if (!mi.last) return;
    __threadfence();
    if (warp < batch) {
        float ss = 0.f;
        for (int b = lane; b < nblk; b += 32) ss += __ldcg(L.norm_partials + (int64_t)warp * nblk + b);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) mi.up[warp] = ss > 0.f ? 1.0f / sqrtf(ss / (float)L.m) : 1.0f;
    }
    if (threadIdx.x == 0) *L.norm_counter = 0;  // ready for the next call
    __syncthreads();
    const int64_t m = L.m;
    for (int tok = 0; tok < batch; ++tok) {
        const float k = mi.up[tok];
        const float4* src = reinterpret_cast<const float4*>(L.y + tok * m);
        uint2* dst = reinterpret_cast<uint2*>(L.y_norm + tok * m);
        for (int64_t g = threadIdx.x; g < m / 4; g += kThreads) {
            const float4 v = __ldcg(src + g);
            const __nv_bfloat162 a = __floats2bfloat162_rn(v.x * k, v.y * k);
            const __nv_bfloat162 b = __floats2bfloat162_rn(v.z * k, v.w * k);
            dst[g] = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
        }
    }
}

template <int NTG, bool CM = false>
__global__ void __launch_bounds__(kThreads, NTG == 1 ? 3 : 2) stage2_kernel(const __grid_constant__ DecGroup grp) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int batch = grp.batch, r2 = grp.r2, rows2 = grp.rows2;
    uint32_t* wbuf = reinterpret_cast<uint32_t*>(smem_raw);
    float* tbuf = reinterpret_cast<float*>(smem_raw + (size_t)grp.w2words * 4);
    uint4* frag = reinterpret_cast<uint4*>(smem_raw + (size_t)grp.w2words * 4 +
                                           (grp.t_global ? 0 : s2_t_bytes(batch, r2)));
    int* bq = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(frag) + frag_bytes(r2 / kCB, NTG));
    uint16_t* s1buf = reinterpret_cast<uint16_t*>(reinterpret_cast<unsigned char*>(bq) + s2_bq_bytes(rows2, batch));
    Misc& mi = *reinterpret_cast<Misc*>(reinterpret_cast<unsigned char*>(s1buf) + s2_s1_bytes(rows2));

    const int rk = find_range(grp.s2_start, grp.count, blockIdx.x);
    const DecLayer& L = grp.L[grp.s2_layer[rk]];
    const int blk = blockIdx.x - grp.s2_start[rk];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int m = L.m, r = L.r;
    const int ws = s2_stride(r, r2);
    // this CTA's share of the layer's 16-row tiles
    const int ntl = m / 16;
    const int tile0 = (int)((int64_t)blk * ntl / L.s2_ctas), tile1 = (int)((int64_t)(blk + 1) * ntl / L.s2_ctas);
    const int ntiles = tile1 - tile0, rows = 16 * ntiles;
    const int64_t wpr = r / 32;
    const int64_t row0 = (int64_t)tile0 * 16;
    const uint32_t* W = L.Upk + row0 * wpr;
    const int nsc = (r + r2 - 1) / r2;  // column spans held on chip one after the other

    // consecutive threads take consecutive 16-byte pieces of the CTA's rows (whole warps per
    // instruction: measured faster than one row per warp)
    auto fetch_w = [&](int sc) {
        const int cols = min(r2, r - sc * r2);
        const int per_row = cols / 128;  // 16-byte pieces
        for (int i = threadIdx.x; i < rows * per_row; i += kThreads) {
            const int row = i / per_row, p = i % per_row;
            cp_async16(wbuf + row * ws + 4 * p, W + row * wpr + sc * (r2 / 32) + 4 * p);
        }
    };
    auto fetch_t = [&](int sc) {
        const int cols = min(r2, r - sc * r2);
        const int per_tok = cols / 4;
        for (int i = threadIdx.x; i < batch * per_tok; i += kThreads) {
            const int tok = i / per_tok, p = i % per_tok;
            cp_async16(tbuf + tok * s2_t_row(r2) + 4 * p + 8 * (p >> 3), L.t + (int64_t)tok * r + sc * r2 + 4 * p);
        }
    };

    fetch_w(0);
    for (int p = threadIdx.x; p < rows / 8; p += kThreads) cp_async16(s1buf + 8 * p, L.s1 + row0 + 8 * p);  // s1 of the rows
    cp_async_commit();
    if (nsc > 1)
        for (int row = threadIdx.x; row < rows; row += kThreads)
            prefetch_l2(W + row * wpr + r2 / 32, (uint32_t)((r - r2) / 8));
    for (int i = threadIdx.x; i < rows * batch; i += kThreads) bq[i] = 0;  // [row][batch]
    zero_fragments<NTG, kThreads>(frag, r2 / kCB);
    pdl_trigger();
    pdl_wait();  // t (or its split partials) and its maxima come from stage 1
    if (L.s2sum) {
        // t = the layer's stage-1 split partials added in split order (the order the reducing
        // stage-1 CTA uses otherwise), staged as fetch_t stages it, and each token's max |t|
        const float* src = L.nsplit > 1 ? L.partials : L.t;
        const int nq = L.nsplit > 1 ? L.nsplit : 1;
        const int64_t qstride = (int64_t)batch * r;
        const int n4 = r / 4;
        for (int tok = 0; tok < batch; ++tok) {
            const float4* s4 = reinterpret_cast<const float4*>(src + (int64_t)tok * r);
            float4 acc[kSumSlots];
#pragma unroll
            for (int j = 0; j < kSumSlots; ++j) {
                const int p = threadIdx.x + j * kThreads;
                acc[j] = p < n4 ? __ldcg(s4 + p) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            for (int q = 1; q < nq; ++q) {
#pragma unroll
                for (int j = 0; j < kSumSlots; ++j) {
                    const int p = threadIdx.x + j * kThreads;
                    if (p < n4) {
                        const float4 v = __ldcg(s4 + q * qstride / 4 + p);
                        acc[j].x += v.x;
                        acc[j].y += v.y;
                        acc[j].z += v.z;
                        acc[j].w += v.w;
                    }
                }
            }
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < kSumSlots; ++j) {
                const int p = threadIdx.x + j * kThreads;
                if (p < n4) {
                    *reinterpret_cast<float4*>(tbuf + tok * s2_t_row(r2) + 4 * p + 8 * (p >> 3)) = acc[j];
                    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(acc[j].x), fabsf(acc[j].y)), fmaxf(fabsf(acc[j].z), fabsf(acc[j].w))));
                }
            }
            mx = warp_max(mx);
            if (lane == 0) mi.red[warp][tok] = mx;
        }
        __syncthreads();
        for (int tok = warp; tok < batch; tok += kWarps) {
            float mx = lane < kWarps ? mi.red[lane][tok] : 0.f;
            mx = warp_max(mx);
            if (lane == 0) {
                const int e = range_exponent(mx);
                mi.e[tok] = e;
                mi.up[tok] = pow2f(kQBits - e);
                mi.qsum[tok] = 0;
            }
        }
    } else {
        if (!grp.t_global) {
            fetch_t(0);
            cp_async_commit();
        }

        // global max |t| per token from the per-block maxima (one warp per token)
        const int nrb = r / kRowsS1;
        for (int tok = warp; tok < batch; tok += kWarps) {
            float mx = 0.f;
            for (int gi = lane; gi < nrb; gi += 32) mx = fmaxf(mx, L.tgmax[(int64_t)tok * nrb + gi]);
            mx = warp_max(mx);
            if (lane == 0) {
                const int e = range_exponent(mx);
                mi.e[tok] = e;
                mi.up[tok] = pow2f(kQBits - e);
                mi.qsum[tok] = 0;
            }
        }
    }

    for (int sc = 0; sc < nsc; ++sc) {
        if (sc > 0) {
            __syncthreads();  // the previous span is consumed
            fetch_w(sc);
            fetch_t(sc);
            cp_async_commit();
        }
        cp_async_wait<0>();
        __syncthreads();
        // every column block of the span at once: one barrier, then an uninterrupted MMA loop
        const int ncb = min(r2, r - sc * r2) / kCB;
        auto tval = [&](int tok, int c) { return tbuf[tok * s2_t_row(r2) + c + 8 * (c >> 5)]; };
        if constexpr (NTG == 2 || CM)
            build_fragments2<NTG, kThreads>(frag, mi, tval, [](int) { return 1.0f; }, ncb, batch);
        else if (grp.t_global)
            build_fragments_t1<kThreads>(frag, mi, L.t, ncb);
        else
            build_fragments<NTG, kThreads>(frag, mi, tval, ncb, batch);
        __syncthreads();
        // the span's units (tile, column block) in tile-major order, an even run per warp;
        // a run covers the ends of up to a few tiles, each added into bq when done
        const int units = ntiles * ncb;
        const int u1 = (warp + 1) * units / kWarps;
        for (int u = warp * units / kWarps; u < u1;) {
            const int ti = u / ncb, cb0 = u % ncb;
            const int cb1 = min(ncb, cb0 + (u1 - u));
            int acc[NTG][4][4];
            zero_acc<NTG>(acc);
            tile_mma<NTG>(frag, wbuf + 16 * ti * ws, ws, cb0, cb1, acc);
#pragma unroll
            for (int tg = 0; tg < NTG; ++tg) {
                const int tok = 4 * tg + tq;
                if (tok < batch) {
                    int bq0, bq8;
                    combine<NTG>(acc, tg, bq0, bq8);
                    atomicAdd(&bq[(16 * ti + g) * batch + tok], bq0);
                    atomicAdd(&bq[(16 * ti + g + 8) * batch + tok], bq8);
                }
            }
            u += cb1 - cb0;
        }
    }
    __syncthreads();
    auto y_at = [&](int tok, int i) {
        const float v = (float)(2 * (int64_t)bq[i * batch + tok] - mi.qsum[tok]) * pow2f(mi.e[tok] - kQBits);
        return f16_to_f32(s1buf[i]) * v;
    };
    for (int idx = threadIdx.x; idx < rows * batch; idx += kThreads) {
        const int tok = idx / rows, i = idx % rows;
        const float yv = y_at(tok, i);
        L.y[(int64_t)tok * m + row0 + i] = yv;
        if (L.y_bf16) L.y_bf16[(int64_t)tok * m + row0 + i] = __bfloat16_as_ushort(__float2bfloat16_rn(yv));
    }
    if (L.y_norm) rms_norm_epilogue(L, batch, rows, blk, mi, y_at);
}

// ------------------------------------------------------------------ stage 2, streaming
// For launches whose weights do not fit on chip in one wave (the Llama-2-70B-shaped block:
// 36.5 MB of U against ~33 MB of shared memory on all SMs), one persistent CTA per SM streams
// an even share of all the layers' weight stages through a ring in shared memory, instead of
// waves of CTAs that each load, then compute.  A unit is one 256-row block of a layer over
// all r columns; a stage is 1024 columns of it (one TMA box of 256 rows x 32 words, 32 KB,
// 128-byte swizzle).  CTA c takes stages [c S / P, (c+1) S / P) of the S stages of all units
// in layer order, so every CTA streams the same number of bytes to within one stage.
// The last warp issues the TMA loads (the weights do not depend on stage 1, so the ring
// fills while the CTA waits for t); the 16 others multiply one 16-row tile each against B
// fragments of t built once per layer (t staged into shared memory in slices with one
// batch of asynchronous copies each; all of r, one exponent per token), loading fragment
// words only in the lanes that hold a token.  (Templated for two token groups as two tiles
// per warp, which measured slower than the classic kernel and is not launched.)
// A unit cut by a CTA boundary is finished by the last of its CTAs to arrive: each writes
// its integer row sums to its own slot, and the last adds the slots in CTA order (integer
// sums: exact, so the result does not depend on the arrival order).  Every wait on an
// mbarrier is bounded (NQ_ERR_TIMEOUT in the status word, then the CTA drains its loads).
constexpr int kS2sRows = 256;                                     // rows per unit
constexpr int kS2sBoxWords = 32;                                  // columns per stage / 32
constexpr int kS2sStageBytes = kS2sRows * kS2sBoxWords * 4;       // 32 KB
constexpr int kS2sStages = 4;
constexpr int kS2sMaxRank = 4096;                                 // fragments of all of r on chip
constexpr int kS2sMaxParts = 4;                                   // CTAs that may share a unit
__host__ __device__ constexpr int s2s_consumers(int ntg) { return ntg == 1 ? 16 : 8; }
__host__ __device__ constexpr int s2s_tpw(int ntg) { return ntg == 1 ? 1 : 2; }
__host__ __device__ constexpr int s2s_threads(int ntg) { return 32 * (s2s_consumers(ntg) + 1); }
__host__ __device__ constexpr int s2s_tstage_floats(int ntg) { return ntg == 1 ? 8192 : 4096; }

struct S2sMaps {
    CUtensorMap map[kMaxGroup];  // Upk of each layer: rows m, cols r/32 words
};

struct S2sBarriers {
    unsigned long long full[kS2sStages], empty[kS2sStages];
    int abort_flag;
    int last;
};

__host__ __device__ inline size_t s2s_frag_offset() { return (size_t)kS2sStages * kS2sStageBytes; }
__host__ __device__ inline size_t s2s_tstage_offset(int ntg) {
    return s2s_frag_offset() + frag_bytes(kS2sMaxRank / kCB, ntg);
}
__host__ __device__ inline size_t s2s_misc_offset(int ntg) {
    return s2s_tstage_offset(ntg) + (size_t)s2s_tstage_floats(ntg) * 4;
}
__host__ __device__ inline size_t s2s_bar_offset(int ntg) { return (s2s_misc_offset(ntg) + sizeof(Misc) + 15) / 16 * 16; }
__host__ __device__ inline size_t s2s_bytes(int ntg) {
    return s2s_bar_offset(ntg) + sizeof(S2sBarriers) + 1024 /*alignment slack*/;
}

template <int NTG, bool CM>
__global__ void __launch_bounds__(s2s_threads(NTG), 1)
stage2s_kernel(const __grid_constant__ DecGroup grp, const __grid_constant__ S2sMaps maps, unsigned* status,
               int* part, int* part_cnt) {
    constexpr int NC = s2s_consumers(NTG), TPW = s2s_tpw(NTG), NCT = 32 * NC;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle wants 1024-byte aligned stages
    unsigned char* gbase = smem_raw + (base - raw);
    uint4* frag = reinterpret_cast<uint4*>(gbase + s2s_frag_offset());
    float* tst = reinterpret_cast<float*>(gbase + s2s_tstage_offset(NTG));
    Misc& mi = *reinterpret_cast<Misc*>(gbase + s2s_misc_offset(NTG));
    S2sBarriers& bar = *reinterpret_cast<S2sBarriers*>(gbase + s2s_bar_offset(NTG));
    volatile int* abort_flag = &bar.abort_flag;
    const int batch = grp.batch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;

    // this CTA's stages [lo, hi) of all units' stages; unit u of layer k has stages
    // st_start[k] + (u - u_start[k]) * nst_k ..
    const int S = grp.st_start[grp.count];
    const int P = gridDim.x;
    const int lo = (int)((int64_t)blockIdx.x * S / P), hi = (int)((int64_t)(blockIdx.x + 1) * S / P);
    auto layer_of_stage = [&](int st) {
        int k = 0;
        while (k + 1 < grp.count && st >= grp.st_start[k + 1]) ++k;
        return k;
    };
    auto nst_of = [&](int k) { return (grp.L[k].r + 1023) / 1024; };
    auto cta_of_stage = [&](int st) {  // the CTA whose range holds stage st
        int c = (int)(((int64_t)st * P) / S);
        while (c + 1 < P && (int64_t)(c + 1) * S / P <= st) ++c;
        while (c > 0 && (int64_t)c * S / P > st) --c;
        return c;
    };

    if (threadIdx.x == 0) {
        for (int st = 0; st < kS2sStages; ++st) {
            mbar_init(smem_u32(&bar.full[st]), 1);
            mbar_init(smem_u32(&bar.empty[st]), NC);
        }
        bar.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == NC) {
        // ---------------- producer: the CTA's stages, in order
        if (lane == 0) {
            int slot = 0, issued = 0;
            uint32_t ph = 0;
            for (int st = lo; st < hi && !*abort_flag; ++st) {
                const int k = layer_of_stage(st);
                const int off = st - grp.st_start[k], nst = nst_of(k);
                const int rb = off / nst, c = off % nst;
                if (!mbar_wait(smem_u32(&bar.empty[slot]), ph ^ 1u, abort_flag, status)) break;
                mbar_expect_tx(smem_u32(&bar.full[slot]), (uint32_t)kS2sStageBytes);
                tma_load_2d(base + (uint32_t)(slot * kS2sStageBytes), &maps.map[k], c * kS2sBoxWords, rb * kS2sRows,
                            smem_u32(&bar.full[slot]));
                ++issued;
                if (++slot == kS2sStages) {
                    slot = 0;
                    ph ^= 1u;
                }
            }
            if (*abort_flag) {
                // let the loads already issued land before the shared memory goes away
                for (int q = issued - kS2sStages < 0 ? 0 : issued - kS2sStages; q < issued; ++q)
                    mbar_drain(smem_u32(&bar.full[q % kS2sStages]), (uint32_t)(q / kS2sStages) & 1u);
            }
        }
        pdl_trigger();
        return;
    }

    // ---------------- consumers (threads 0 .. NCT-1)
    pdl_trigger();
    zero_fragments<NTG, NCT>(frag, kS2sMaxRank / kCB);
    pdl_wait();  // t and its block maxima come from stage 1
    auto consumer_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(NCT) : "memory"); };
    int cur = -1, slot = 0;
    uint32_t ph = 0;
    int st = lo;
    while (st < hi) {
        const int k = layer_of_stage(st);
        const DecLayer& L = grp.L[k];
        const int r = L.r, ncb = r / kCB, nst = nst_of(k);
        const int off = st - grp.st_start[k];
        const int rb = off / nst, c_first = off % nst;
        const int c_last = min(nst, c_first + (hi - st));  // stages of this unit in this CTA: [c_first, c_last)
        if (k != cur) {
            // the layer's exponent per token (from stage 1's block maxima) and its fragments,
            // t staged into shared memory a slice of columns at a time
            consumer_sync();
            const int nrb = r / kRowsS1;
            for (int tok = warp; tok < batch; tok += NC) {
                float mx = 0.f;
                for (int gi = lane; gi < nrb; gi += 32) mx = fmaxf(mx, __ldcg(L.tgmax + (int64_t)tok * nrb + gi));
                mx = warp_max(mx);
                if (lane == 0) {
                    const int e = range_exponent(mx);
                    mi.e[tok] = e;
                    mi.up[tok] = pow2f(kQBits - e);
                    mi.qsum[tok] = 0;
                }
            }
            const int slice = min(r, s2s_tstage_floats(NTG) / batch / kCB * kCB);  // columns per slice
            for (int c0 = 0; c0 < r; c0 += slice) {
                const int cols = min(slice, r - c0);
                consumer_sync();  // the previous slice is consumed (and the maxima are written)
                for (int i = threadIdx.x; i < batch * cols / 4; i += NCT) {
                    const int tok = i / (cols / 4), p = i % (cols / 4);
                    cp_async16(tst + tok * slice + 4 * p, L.t + (int64_t)tok * r + c0 + 4 * p);
                }
                cp_async_commit();
                cp_async_wait<0>();
                consumer_sync();
                auto tval = [&](int tok, int cc) { return tst[tok * slice + cc]; };
                uint4* fslice = frag + (size_t)(c0 / kCB) * NTG * 2 * 32;
                if constexpr (NTG == 2 || CM)
                    build_fragments2<NTG, NCT>(fslice, mi, tval, [](int) { return 1.0f; }, cols / kCB, batch);
                else
                    build_fragments<NTG, NCT>(fslice, mi, tval, cols / kCB, batch);
            }
            consumer_sync();
            cur = k;
        }
        int acc[TPW][NTG][4][4], acc2[TPW][NTG][4][4];
#pragma unroll
        for (int tl = 0; tl < TPW; ++tl) {
            zero_acc<NTG>(acc[tl]);
            zero_acc<NTG>(acc2[tl]);
        }
        // rows 16 TPW warp + g (+ 8, + 16, + 24) of the stage: all have row & 7 == g
        const uint32_t row_off = (uint32_t)((16 * TPW * warp + g) * 128);
        // B fragments: lane l carries column n = l / 4 of the MMA (token n / 2 of its group,
        // limb n % 2); lanes of absent tokens hold zeros, so only the lanes with a token
        // load (at batch 1: 8 of 32 lanes, a quarter of the shared-memory wavefronts)
        auto load_frag = [&](int gcb, int tg, uint4& f0, uint4& f1) {
            f0 = f1 = make_uint4(0u, 0u, 0u, 0u);
            if (lane < 8 * (batch - 4 * tg)) {
                f0 = *frag_ptr<NTG>(frag, gcb, tg, 0, lane);
                f1 = *frag_ptr<NTG>(frag, gcb, tg, 1, lane);
            }
        };
        bool ok = true;
        for (int c = c_first; c < c_last; ++c) {
            if (!mbar_wait(smem_u32(&bar.full[slot]), ph, abort_flag, status)) {
                ok = false;
                break;
            }
            // plain loads (not volatile asm), so that the compiler can issue the next column
            // blocks' loads ahead of this one's MMAs; the stage's bytes are visible after the
            // mbarrier wait (a memory clobber)
            const uint32_t* st_row =
                reinterpret_cast<const uint32_t*>(gbase + (size_t)slot * kS2sStageBytes + row_off);
            const int cb_n = min(8, ncb - 8 * c);
            // one column block into accumulator set A (an explicit function of the block, so
            // that the two sets alternate without a run-time test)
            auto block = [&](int cb, int (&A)[TPW][NTG][4][4]) {
                // chunk cb of the row sits at chunk cb ^ (row & 7) = cb ^ g
                const uint32_t* a = st_row + ((cb ^ g) << 2) + tq;
                const int gcb = 8 * c + cb;
                if constexpr (TPW == 1) {
                    const uint32_t wa = a[0], wb = a[256];  // rows g and g + 8 (8 rows x 32 words apart)
                    const uint32_t x0 = wa >> 4, y0 = wb >> 4;
#pragma unroll
                    for (int tg = 0; tg < NTG; ++tg) {
                        uint4 f0, f1;
                        load_frag(gcb, tg, f0, f1);
                        const uint32_t bf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
                        for (int sft = 0; sft < 4; ++sft) {
                            const uint32_t M = 0x01010101u << sft;
                            mma_u8s8(A[0][tg][sft], wa & M, wb & M, x0 & M, y0 & M, bf[2 * sft], bf[2 * sft + 1]);
                        }
                    }
                } else {
                    const uint32_t wa0 = a[0], wb0 = a[256], wa1 = a[512], wb1 = a[768];
                    const uint32_t x0 = wa0 >> 4, y0 = wb0 >> 4, x1 = wa1 >> 4, y1 = wb1 >> 4;
#pragma unroll
                    for (int tg = 0; tg < NTG; ++tg) {
                        uint4 f0, f1;
                        load_frag(gcb, tg, f0, f1);
                        const uint32_t bf[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
                        for (int sft = 0; sft < 4; ++sft) {
                            const uint32_t M = 0x01010101u << sft;
                            mma_u8s8(A[0][tg][sft], wa0 & M, wb0 & M, x0 & M, y0 & M, bf[2 * sft], bf[2 * sft + 1]);
                            mma_u8s8(A[1][tg][sft], wa1 & M, wb1 & M, x1 & M, y1 & M, bf[2 * sft], bf[2 * sft + 1]);
                        }
                    }
                }
            };
            if (cb_n == 8) {
#pragma unroll
                for (int cb = 0; cb < 8; cb += 2) {
                    block(cb, acc);
                    block(cb + 1, acc2);
                }
            } else {
                int cb = 0;
                for (; cb + 1 < cb_n; cb += 2) {
                    block(cb, acc);
                    block(cb + 1, acc2);
                }
                if (cb < cb_n) block(cb, acc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar.empty[slot]));
            if (++slot == kS2sStages) {
                slot = 0;
                ph ^= 1u;
            }
        }
        if (!ok) break;
        // the warp's integer row sums: bq[tl][tg][0] for row g, [1] for row g + 8
        int bq[TPW][NTG][2];
#pragma unroll
        for (int tl = 0; tl < TPW; ++tl) {
#pragma unroll
            for (int tg = 0; tg < NTG; ++tg)
#pragma unroll
                for (int sft = 0; sft < 4; ++sft)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[tl][tg][sft][i] += acc2[tl][tg][sft][i];
#pragma unroll
            for (int tg = 0; tg < NTG; ++tg) combine<NTG>(acc[tl], tg, bq[tl][tg][0], bq[tl][tg][1]);
        }
        const int64_t m = L.m;
        const int64_t row_base = (int64_t)rb * kS2sRows + 16 * TPW * warp + g;  // + 16 tl (+ 8)
        auto store_y = [&](int tok, int64_t row, int64_t q) {  // q = 2 sum b q - sum q of (row, tok)
            if (row >= m) return;
            const float y = f16_to_f32(__ldg(L.s1 + row)) * ((float)q * pow2f(mi.e[tok] - kQBits));
            L.y[tok * m + row] = y;
            if (L.y_bf16) L.y_bf16[tok * m + row] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
        };
        const bool whole = c_first == 0 && c_last == nst;
        if (whole) {
#pragma unroll
            for (int tl = 0; tl < TPW; ++tl)
#pragma unroll
                for (int tg = 0; tg < NTG; ++tg) {
                    const int tok = 4 * tg + tq;
                    if (tok < batch) {
                        const int64_t qs = mi.qsum[tok];
                        store_y(tok, row_base + 16 * tl, 2 * (int64_t)bq[tl][tg][0] - qs);
                        store_y(tok, row_base + 16 * tl + 8, 2 * (int64_t)bq[tl][tg][1] - qs);
                    }
                }
        } else {
            // a unit shared with other CTAs: this CTA's integer sums into its own slot, then
            // the last to arrive adds the slots in CTA order and writes y.  Slot of the unit:
            // the index of the first CTA boundary inside it (unique per shared unit).
            const int ust = grp.st_start[k] + rb * nst;  // the unit's first stage
            const int c0 = cta_of_stage(ust);
            const int cnt_all = cta_of_stage(ust + nst - 1) - c0 + 1;
            const int slotu = c0 + 1, me = blockIdx.x - c0;
            int* mine = part + ((int64_t)slotu * kS2sMaxParts + me) * (kS2sRows * 8);
#pragma unroll
            for (int tl = 0; tl < TPW; ++tl)
#pragma unroll
                for (int tg = 0; tg < NTG; ++tg) {
                    const int tok = 4 * tg + tq;
                    if (tok < batch) {
                        const int rr = 16 * TPW * warp + 16 * tl + g;
                        mine[rr * 8 + tok] = bq[tl][tg][0];
                        mine[(rr + 8) * 8 + tok] = bq[tl][tg][1];
                    }
                }
            consumer_sync();
            if (threadIdx.x == 0) {
                __threadfence();
                bar.last = atomicAdd(part_cnt + slotu, 1) == cnt_all - 1;
                if (bar.last) __threadfence();
            }
            consumer_sync();
            if (bar.last) {
                const int* slots = part + (int64_t)slotu * kS2sMaxParts * (kS2sRows * 8);
                for (int i = threadIdx.x; i < kS2sRows * batch; i += NCT) {
                    const int rr = i / batch, tok = i % batch;
                    int64_t sum = 0;
                    for (int q = 0; q < cnt_all; ++q) sum += __ldcg(slots + q * (kS2sRows * 8) + rr * 8 + tok);
                    store_y(tok, (int64_t)rb * kS2sRows + rr, 2 * sum - mi.qsum[tok]);
                }
                if (threadIdx.x == 0) part_cnt[slotu] = 0;  // ready for the next call
            }
        }
        st += c_last - c_first;
    }
}

template <typename K>
static bool set_kernel_attributes(K kernel) {
    // the largest shared-memory carveout for every decode kernel, so that CTAs of the two
    // stages (and of consecutive calls) can share an SM
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) == cudaSuccess &&
           cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared) == cudaSuccess;
}

template <int NTG, bool CM>
int launch_stages(DecGroup& grp, cudaStream_t stream, int device, bool stage1_only, const S2sMaps* maps,
                  unsigned* status, int* s2s_part, int* s2s_cnt) {
    static unsigned long long init_mask = 0;  // devices whose kernel attributes are set
    const unsigned long long bit = 1ull << (device & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (!set_kernel_attributes(stage1_kernel<NTG, 2, CM>) || !set_kernel_attributes(stage2_kernel<NTG, CM>))
            return NQ_ERR_CUDA;
        if constexpr (NTG == 1)
            if (cudaFuncSetAttribute(stage2s_kernel<NTG, CM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)s2s_bytes(NTG)) != cudaSuccess)
                return NQ_ERR_CUDA;
        if constexpr (NTG == 1)
            if (!set_kernel_attributes(stage1_kernel<1, 1, CM>)) return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    const size_t smem1 = s1_bytes(grp.depth1, grp.batch, NTG);
    size_t smem2 = s2_bytes(grp.w2words, grp.rows2, grp.batch, grp.r2, NTG, grp.t_global != 0);
    // a one-wave stage-2 plan gives every SM the same work only if no SM takes more than
    // per_sm2 of its CTAs: ask for enough shared memory that one more does not fit
    if (grp.per_sm2 > 0) smem2 = std::max(smem2, kSmemPerSM / (grp.per_sm2 + 1) - kSmemReserve + 16);
    const unsigned grid1 = (unsigned)grp.s1_start[grp.count];
    // one tile per warp (one token group only) when the launch fits in one wave of four
    // 8-warp CTAs per SM
    cudaError_t err;
    if constexpr (NTG == 1) {
        if (grid1 <= 4u * (unsigned)sm_count())
            err = launch_pdl(stage1_kernel<1, 1, CM>, dim3(grid1), dim3(s1_threads<1>()), smem1, stream, grp);
        else
            err = launch_pdl(stage1_kernel<1, 2, CM>, dim3(grid1), dim3(s1_threads<2>()), smem1, stream, grp);
    } else {
        err = launch_pdl(stage1_kernel<NTG, 2, CM>, dim3(grid1), dim3(s1_threads<2>()), smem1, stream, grp);
    }
    if (err != cudaSuccess) return NQ_ERR_CUDA;
    if (stage1_only) return NQ_OK;
    if constexpr (NTG == 1) {
        if (grp.stream2) {
            const int stages = grp.st_start[grp.count];
        const int grid2 = std::min(stages, sm_count());  // every CTA has at least one stage
            return launch_pdl(stage2s_kernel<NTG, CM>, dim3((unsigned)grid2), dim3(s2s_threads(NTG)),
                              s2s_bytes(NTG), stream, grp, *maps, status, s2s_part, s2s_cnt) == cudaSuccess
                       ? NQ_OK
                       : NQ_ERR_CUDA;
        }
    }
    if (launch_pdl(stage2_kernel<NTG, CM>, dim3((unsigned)grp.s2_start[grp.count]), dim3(kThreads), smem2, stream,
                   grp) != cudaSuccess)
        return NQ_ERR_CUDA;
    return NQ_OK;
}

template <int NTG>
int launch_group(DecGroup& grp, cudaStream_t stream, int device, bool stage1_only, const S2sMaps* maps,
                 unsigned* status, int* s2s_part, int* s2s_cnt) {
    if constexpr (NTG == 1)
        if (grp.batch >= kColMajorMinBatch)
            return launch_stages<1, true>(grp, stream, device, stage1_only, maps, status, s2s_part, s2s_cnt);
    return launch_stages<NTG, false>(grp, stream, device, stage1_only, maps, status, s2s_part, s2s_cnt);
}

}  // namespace

// Stage-2 columns held on chip at a time: all of r when it fits (up to 4096 columns, less
// for larger batches since t takes batch x r2 x 4 bytes), else spans of a multiple of kChunk.
static int stage2_span(int64_t r_max, int64_t batch) {
    int64_t span = 8192 / batch;
    span = span / kChunk * kChunk;
    if (span > 4096) span = 4096;
    if (span < kChunk) span = kChunk;
    const int64_t need = (r_max + kCB - 1) / kCB * kCB;
    return (int)(need < span ? need : span);
}

// Stage-2 CTAs per layer (ctas[i]), the largest weight buffer (words) and the most rows
// of one CTA.  A launch that fits in one wave gets k CTAs per SM in all, the smallest
// k = 2 .. kMaxK2 for which k of them fit on an SM (shared memory): layer i gets CTAs in
// proportion to its work, tiles_i x column blocks_i (largest remainders, at least one and at
// most one per tile), and each CTA an even share of the layer's tiles, so that all CTAs
// carry about the same work.  A larger launch takes CTAs of kWaveTiles2 tiles (several waves).
static void stage2_plan(const DecodeCall* calls, int count, int64_t batch, int* ctas, int* w2words, int* rows2,
                        int* per_sm) {
    int64_t work = 0, tiles_all = 0, r_max = 0;
    for (int i = 0; i < count; ++i) {
        work += (calls[i].m / 16) * (calls[i].r / kCB);
        tiles_all += calls[i].m / 16;
        r_max = calls[i].r > r_max ? calls[i].r : r_max;
    }
    const int r2 = stage2_span(r_max, batch);
    const int ntg = batch <= 4 ? 1 : 2;
    const int sms = sm_count();
    auto measure = [&]() {  // buffer sizes of the current ctas[]
        int64_t words = 0, rows = 0;
        for (int i = 0; i < count; ++i) {
            const int64_t tl = (calls[i].m / 16 + ctas[i] - 1) / ctas[i];
            words = std::max(words, 16 * tl * s2_stride((int)calls[i].r, r2));
            rows = std::max(rows, 16 * tl);
        }
        *w2words = (int)words;
        *rows2 = (int)rows;
        return s2_bytes(*w2words, *rows2, (int)batch, r2, ntg) + kSmemReserve;
    };
    for (int k = 2; k <= kMaxK2; ++k) {
        const int64_t total = std::min<int64_t>((int64_t)k * sms, tiles_all);
        int64_t given = 0;
        double frac[kMaxGroup];
        for (int i = 0; i < count; ++i) {
            const int64_t ti = calls[i].m / 16;
            const double share = (double)total * (double)(ti * (calls[i].r / kCB)) / (double)work;
            const int64_t c = std::max<int64_t>(1, std::min<int64_t>((int64_t)share, ti));
            ctas[i] = (int)c;
            frac[i] = share - (double)c;
            given += c;
        }
        while (given < total) {  // largest remainders first, never past one CTA per tile
            int best = -1;
            for (int i = 0; i < count; ++i)
                if (ctas[i] < calls[i].m / 16 && (best < 0 || frac[i] > frac[best])) best = i;
            if (best < 0) break;
            ++ctas[best];
            frac[best] -= 1.0;
            ++given;
        }
        const size_t need = measure();
        if (total == tiles_all) {  // one tile per CTA: no smaller CTAs exist, and no cap is needed
            *per_sm = 0;
            return;
        }
        if ((size_t)k * need <= kSmemPerSM) {
            *per_sm = k;
            return;
        }
    }
    for (int i = 0; i < count; ++i) ctas[i] = (int)((calls[i].m / 16 + kWaveTiles2 - 1) / kWaveTiles2);
    *per_sm = 0;
    measure();
}

// A several-wave stage-2 plan at batch 1 without the staged copy of t (its 19 KB at r = 3840
// go to weight rows instead): the fewest tiles per CTA (from kWaveTiles2) for which the CTAs
// fill at most two waves of two CTAs per SM.  false (nothing changed) if there is none.
// Measured on a B200, the Llama-2-70B-shaped block at batch 1: 656 CTAs of 8 tiles (2.22
// waves) -> 587 CTAs of 9 tiles (1.98 waves), 36.9 -> 36.1 us per step.
static bool stage2_plan_t_global(const DecodeCall* calls, int count, int r2, int* ctas, int* w2words, int* rows2) {
    const int sms = sm_count();
    for (int tpc = kWaveTiles2; tpc <= 2 * kWaveTiles2; ++tpc) {
        int64_t total = 0, words = 0, rows = 0;
        for (int i = 0; i < count; ++i) {
            const int64_t ti = calls[i].m / 16, c = (ti + tpc - 1) / tpc;
            total += c;
            const int64_t tl = (ti + c - 1) / c;
            words = std::max(words, 16 * tl * s2_stride((int)calls[i].r, r2));
            rows = std::max(rows, 16 * tl);
        }
        if (total > 4 * (int64_t)sms) continue;  // two waves of two CTAs per SM
        if (2 * (s2_bytes((int)words, (int)rows, 1, r2, 1, true) + kSmemReserve) > kSmemPerSM) return false;
        for (int i = 0; i < count; ++i) ctas[i] = (int)((calls[i].m / 16 + tpc - 1) / tpc);
        *w2words = (int)words;
        *rows2 = (int)rows;
        return true;
    }
    return false;
}

// Column blocks per stage-1 split: about two CTAs per SM over the whole launch, at least
// 4 and (while the split count stays <= max_splits) at most kChunkCB column blocks per CTA,
// so that every CTA does one chunk.
static int stage1_cps(const DecodeCall* calls, int count, int max_splits) {
    int64_t units = 0, max_ncb = 0;
    for (int i = 0; i < count; ++i) {
        units += (calls[i].r / kRowsS1) * (calls[i].n / kCB);
        max_ncb = calls[i].n / kCB > max_ncb ? calls[i].n / kCB : max_ncb;
    }
    const int64_t target = 2 * (int64_t)sm_count();
    int64_t cps = (units + target - 1) / target;
    if (cps < 4) cps = 4;
    if (cps > kChunkCB) cps = kChunkCB;
    if ((max_ncb + cps - 1) / cps > max_splits) cps = (max_ncb + max_splits - 1) / max_splits;
    return (int)cps;
}

// Scratch of the streaming stage 2's shared units: per CTA boundary, kS2sMaxParts slots of
// 256 rows x 8 tokens of integer sums, and one arrival counter.
static int64_t s2s_part_ints() { return (int64_t)(sm_count() + 1) * kS2sMaxParts * kS2sRows * 8; }
static int64_t s2s_counter_ints() { return sm_count() + 1; }

// Whether the layers' shapes take the streaming stage 2: all of r fits its fragment buffer,
// no layer asks for the normalised output, and the classic plan finds no one-wave layout.
static bool s2s_shapes(const DecodeCall* calls, int count, int per_sm2) {
    int64_t r_max = 0;
    bool any_norm = false;
    for (int i = 0; i < count; ++i) {
        r_max = calls[i].r > r_max ? calls[i].r : r_max;
        any_norm = any_norm || calls[i].y_norm != nullptr;
    }
    return !any_norm && r_max <= kS2sMaxRank && per_sm2 == 0;
}

void decode_workspace_need(const DecodeCall* calls, int count, int64_t batch, int max_splits, int64_t* t_floats,
                           int64_t* tgmax_floats, int64_t* partial_floats, int64_t* counter_ints) {
    const int cps = stage1_cps(calls, count, max_splits);
    int ctas[kMaxGroup], w2words = 0, rows2 = 0, per_sm = 0;
    stage2_plan(calls, count, batch, ctas, &w2words, &rows2, &per_sm);
    const bool s2s = s2s_shapes(calls, count, per_sm);
    int64_t t = 0, gm = 0, pf = 0, ci = 0;
    for (int i = 0; i < count; ++i) {
        const int64_t ncb = calls[i].n / kCB, nsplit = (ncb + cps - 1) / cps;
        t += batch * calls[i].r;
        gm += batch * (calls[i].r / kRowsS1);
        if (nsplit > 1) pf += nsplit * batch * calls[i].r;
        ci += calls[i].r / kRowsS1;
        if (calls[i].y_norm) {  // per-CTA sums of y^2 and one arrival counter
            pf += batch * ctas[i];
            ci += 1;
        }
    }
    *t_floats = t;
    *tgmax_floats = gm;
    // the streaming stage 2's scratch comes last (decode_forward_group uses the stage only
    // when the workspace holds it)
    *partial_floats = pf + (s2s ? s2s_part_ints() : 0);
    *counter_ints = ci + (s2s ? s2s_counter_ints() : 0);
}

int decode_forward_group(const DecodeCall* calls, int count, int64_t batch, Workspace* ws, cudaStream_t stream,
                         int max_splits, bool stage1_only) {
    if (count < 1 || count > kMaxGroup) return NQ_ERR_SHAPE;
    int64_t need_t, need_g, need_p, need_c;
    decode_workspace_need(calls, count, batch, max_splits, &need_t, &need_g, &need_p, &need_c);
    // the streaming stage 2 is optional: without room for its scratch the classic one runs
    bool s2s_room = (size_t)need_p <= ws->partial_cap && (size_t)need_c <= ws->counter_cap;
    {
        int ctas0[kMaxGroup], w0 = 0, r0 = 0, ps0 = 0;
        stage2_plan(calls, count, batch, ctas0, &w0, &r0, &ps0);
        if (s2s_shapes(calls, count, ps0)) {
            need_p -= s2s_part_ints();
            need_c -= s2s_counter_ints();
        } else {
            s2s_room = false;
        }
    }
    if ((size_t)need_t > ws->t_cap || (size_t)need_g > ws->tgmax_cap || (size_t)need_p > ws->partial_cap ||
        (size_t)need_c > ws->counter_cap)
        return NQ_ERR_NOMEM;
    DecGroup grp;
    grp.count = count;
    grp.batch = (int)batch;
    int64_t r_max = 0;
    for (int i = 0; i < count; ++i) r_max = calls[i].r > r_max ? calls[i].r : r_max;
    int ctas[kMaxGroup];
    stage2_plan(calls, count, batch, ctas, &grp.w2words, &grp.rows2, &grp.per_sm2);
    const int cps = stage1_cps(calls, count, max_splits);
    grp.r2 = stage2_span(r_max, batch);
    // Stage 2 adds up the layers' split partials itself (no hand-off between the stage-1 CTAs
    // of a row block) when all of t fits one span and no layer has many splits: each stage-2
    // CTA then reads nsplit x r values per token instead of r, and stage 1 ends no earlier
    // unless every layer drops its hand-off (the layer of most splits has the longest).
    // Measured on a B200: the seven Llama-2-7B-shaped layers at batch 1 (4 and 11 splits)
    // 14.7 -> 13.6 us; the 70B-shaped block (8 and 28 splits) is slower with it for any
    // subset of its layers (36.5 -> 37.0-38.8 us), so it keeps the hand-off.
    int max_nsplit = 0;
    for (int i = 0; i < count; ++i) max_nsplit = std::max(max_nsplit, (int)((calls[i].n / kCB + cps - 1) / cps));
    // Streaming stage 2 (stage2s_kernel) where the layers' U does not fit on chip in one wave
    // of the classic plan (no per-SM cap found), all of r fits its fragment buffer and the
    // workspace holds its scratch.  (It records a timed-out wait in the workspace's status
    // word, so it needs one.)
    // Measured on a B200, the Llama-2-70B-shaped block: 2 tokens 53.3 -> 43.4 us, 4 tokens
    // 62.8 -> 54.8 us per step with it; 1 token 37.1 -> 38.8 us and 8 tokens (two token groups,
    // two 16-row tiles per warp) 106 -> 112 us, so those keep the classic kernel.
    const bool stream2 = !stage1_only && s2s_room && ws->status != nullptr && batch >= 2 && batch <= 4;
    grp.stream2 = stream2 ? 1 : 0;
    const bool s2sum = !stream2 && !stage1_only && r_max <= grp.r2 && r_max <= 4 * kSumSlots * kThreads &&
                       max_nsplit <= kS2SumMaxSplits;
    // One token, a several-wave stage-2 plan, one span, t from stage 1's hand-off: stage 2
    // builds its fragments from t in global memory, and the shared memory of the staged copy
    // goes to CTAs of more rows that fill two waves instead of two and a fraction.
    grp.t_global = 0;
    if (batch == 1 && !stage1_only && !stream2 && !s2sum && grp.per_sm2 == 0 && r_max <= grp.r2 &&
        stage2_plan_t_global(calls, count, grp.r2, ctas, &grp.w2words, &grp.rows2))
        grp.t_global = 1;
    grp.depth1 = cps > kChunkCB ? 2 : 1;
    size_t toff = 0, goff = 0, poff = 0, coff = 0;
    grp.s1_start[0] = grp.s2_start[0] = 0;
    // the normalisation's sums and counters go after every layer's stage-1 scratch
    size_t npoff = 0, ncoff = 0;
    for (int i = 0; i < count; ++i) {
        const int64_t nsplit = (calls[i].n / kCB + cps - 1) / cps;
        if (nsplit > 1) npoff += (size_t)nsplit * batch * calls[i].r;
        ncoff += (size_t)(calls[i].r / kRowsS1);
    }
    for (int i = 0; i < count; ++i) {
        const DecodeCall& c = calls[i];
        DecLayer& L = grp.L[i];
        L.x = c.x;
        L.Upk = c.Upk;
        L.Vpk = c.Vpk;
        L.s1 = c.s1;
        L.s2 = c.s2;
        L.y = c.y;
        L.y_bf16 = c.y_bf16;
        L.y_norm = c.y_norm;
        L.norm_partials = nullptr;
        L.norm_counter = nullptr;
        if (c.y_norm) {
            L.norm_partials = ws->partials + npoff;
            L.norm_counter = ws->counters + ncoff;
            npoff += (size_t)batch * ctas[i];
            ncoff += 1;
        }
        L.m = (int)c.m;
        L.n = (int)c.n;
        L.r = (int)c.r;
        L.s2_ctas = ctas[i];
        L.s2sum = s2sum ? 1 : 0;
        L.cps = cps;
        L.nsplit = (int)((c.n / kCB + cps - 1) / cps);
        L.t = ws->t + toff;
        L.tgmax = ws->tgmax + goff;
        L.partials = ws->partials + poff;
        L.counters = ws->counters + coff;
        toff += (size_t)batch * c.r;
        goff += (size_t)batch * (c.r / kRowsS1);
        if (L.nsplit > 1) poff += (size_t)L.nsplit * batch * c.r;
        coff += (size_t)(c.r / kRowsS1);
    }
    // Launch order of the layers' CTA ranges: the layers with the longest path through a
    // stage go first, so that their CTAs are the first resident and the first scheduled
    // (stage 1: most column splits, i.e. the longest hand-off; stage 2: largest rank, i.e.
    // the most fragments to build per CTA).  Ties keep the caller's order.
    int o1[kMaxGroup], o2[kMaxGroup];
    for (int i = 0; i < count; ++i) o1[i] = o2[i] = i;
    std::stable_sort(o1, o1 + count, [&](int a, int b) { return grp.L[a].nsplit > grp.L[b].nsplit; });
    std::stable_sort(o2, o2 + count, [&](int a, int b) { return grp.L[a].r > grp.L[b].r; });
    for (int k = 0; k < count; ++k) {
        const DecLayer& L1 = grp.L[o1[k]];
        const DecLayer& L2 = grp.L[o2[k]];
        grp.s1_layer[k] = (unsigned char)o1[k];
        grp.s2_layer[k] = (unsigned char)o2[k];
        grp.s1_start[k + 1] = grp.s1_start[k] + (L1.r / kRowsS1) * L1.nsplit;
        grp.s2_start[k + 1] = grp.s2_start[k] + L2.s2_ctas;
    }
    S2sMaps maps;
    int* s2s_part = reinterpret_cast<int*>(ws->partials + npoff);
    int* s2s_cnt = ws->counters + ncoff;
    if (stream2) {
        grp.u_start[0] = grp.st_start[0] = 0;
        for (int i = 0; i < count; ++i) {
            const DecLayer& L = grp.L[i];
            const int units = (L.m + kS2sRows - 1) / kS2sRows;  // a last unit of 128 rows reads zeros past m
            grp.u_start[i + 1] = grp.u_start[i] + units;
            grp.st_start[i + 1] = grp.st_start[i] + units * ((L.r + 1023) / 1024);
            if (!encode_map_u32_sw128(&maps.map[i], L.Upk, L.m, L.r / 32, kS2sBoxWords, kS2sRows)) return NQ_ERR_CUDA;
        }
    }
    unsigned* status = ws->status ? ws->status + 1 : nullptr;
    if (batch <= 4) return launch_group<1>(grp, stream, ws->device, stage1_only, &maps, status, s2s_part, s2s_cnt);
    return launch_group<2>(grp, stream, ws->device, stage1_only, &maps, status, s2s_part, s2s_cnt);
}

int decode_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                   const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                   Workspace* ws, cudaStream_t stream) {
    DecodeCall c{x, Upk, Vpk, s1, s2, y, m, n, r};
    return decode_forward_group(&c, 1, batch, ws, stream, kDecodeMaxSplits);
}

int decode_rank_vector(const uint16_t* x, const uint32_t* Vpk, const uint16_t* s2, int64_t n, int64_t r,
                       int64_t batch, float* t, Workspace* ws, cudaStream_t stream) {
    for (int64_t b0 = 0; b0 < batch; b0 += NQ_DECODE_MAX_BATCH) {
        const int64_t bc = batch - b0 < NQ_DECODE_MAX_BATCH ? batch - b0 : NQ_DECODE_MAX_BATCH;
        // stage 1 alone writes t of the only layer at the start of the workspace's t
        const DecodeCall c{x + b0 * n, nullptr, Vpk, nullptr, s2, nullptr, kRowsS1, n, r};
        int st = decode_forward_group(&c, 1, bc, ws, stream, kDecodeMaxSplits, true);
        if (st != NQ_OK) return st;
        if (cudaMemcpyAsync(t + b0 * r, ws->t, sizeof(float) * (size_t)(bc * r), cudaMemcpyDeviceToDevice, stream) !=
            cudaSuccess)
            return NQ_ERR_CUDA;
    }
    return NQ_OK;
}

}  // namespace nq

// ---------------------------------------------------------------------------------------
// Allocation-free decode entry point.
//
// Some callers cannot allocate device memory at the moment they run a layer: an inference
// engine that sized and froze its memory pool at start-up (any later cudaMalloc competes
// with the pool for the same HBM and may fail mid-request), or a process whose allocator is
// owned by another framework (a side allocation bypasses its accounting).  For them nq_lowrank_linear_fwd_noalloc keeps the decode path's scratch
// (t, the per-block maxima of |t|, the stage-1 split partials and arrival counters) in one
// fixed array of device memory that is part of this library's module, so a call allocates
// nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// it until the process exits.  Host code may not use its name as an address (on the host
// the name is a stand-in, not device memory), so the first call on each device resolves
// the device address with cudaGetSymbolAddress, with that device current, and caches it.
// All calls share the one array: calls whose kernels overlap on the GPU (different
// streams, or different host threads on one device) race and must be serialised by the
// caller.  The arrival counters must start at zero; each call clears them on its stream
// before its kernels run.
namespace nq {
namespace {

constexpr int64_t kNoAllocMaxRank = 4096;   // largest r
constexpr int kNoAllocMaxSplits = 8;        // stage-1 column splits
constexpr size_t kNoAllocT = (size_t)NQ_DECODE_MAX_BATCH * kNoAllocMaxRank;
constexpr size_t kNoAllocG = (size_t)NQ_DECODE_MAX_BATCH * (kNoAllocMaxRank / kRowsS1);
constexpr size_t kNoAllocP = (size_t)kNoAllocMaxSplits * NQ_DECODE_MAX_BATCH * kNoAllocMaxRank;
constexpr size_t kNoAllocC = kNoAllocMaxRank / kRowsS1;
constexpr size_t kNoAllocBytes = 4 * (kNoAllocT + kNoAllocG + kNoAllocP + kNoAllocC);
static_assert(kNoAllocBytes == 1180800, "the scratch size stated in nq.h");

}  // namespace
}  // namespace nq

static __device__ __align__(256) unsigned char g_noalloc_scratch[nq::kNoAllocBytes];

namespace nq {
namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[64];  // device address of g_noalloc_scratch, per device

int noalloc_scratch(int dev, void** out) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return NQ_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return NQ_OK;
}

// Memory the kernels launched on device `dev` may read: device memory of `dev` itself, or
// managed memory.  Device memory of another GPU is refused (without peer access a kernel
// given it faults), as is host memory.
bool is_device_memory(const void* p, int dev) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (attr.type == cudaMemoryTypeManaged) return true;
    return attr.type == cudaMemoryTypeDevice && attr.device == dev;
}

}  // namespace
}  // namespace nq

extern "C" int nq_lowrank_linear_fwd_noalloc(const void* x, const uint32_t* Upk, const uint32_t* Vpk, const void* s1,
                                             const void* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                                             void* stream) {
    using namespace nq;
    if (batch < 0) return NQ_ERR_BATCH;
    if (m <= 0 || n <= 0 || r <= 0 || m % 128 || n % 128 || r % 128 || m > (int64_t(1) << 20) ||
        n > (int64_t(1) << 20))
        return NQ_ERR_SHAPE;
    if (r > kNoAllocMaxRank || batch > NQ_DECODE_MAX_BATCH) return NQ_ERR_NOALLOC_LIMIT;
    if (batch == 0) return NQ_OK;
    if (!x || !Upk || !Vpk || !s1 || !s2 || !y) return NQ_ERR_NULL;
    const uintptr_t a = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(Upk) |
                        reinterpret_cast<uintptr_t>(Vpk) | reinterpret_cast<uintptr_t>(s1) |
                        reinterpret_cast<uintptr_t>(s2) | reinterpret_cast<uintptr_t>(y);
    if (a & 15u) return NQ_ERR_ALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return NQ_ERR_CUDA;
    }
    if (!is_device_memory(x, dev) || !is_device_memory(Upk, dev) || !is_device_memory(Vpk, dev) ||
        !is_device_memory(s1, dev) || !is_device_memory(s2, dev) || !is_device_memory(y, dev))
        return NQ_ERR_PTRKIND;
    void* scratch = nullptr;
    int st = noalloc_scratch(dev, &scratch);
    if (st != NQ_OK) return st;

    // a workspace view over the fixed array (nothing here is allocated)
    Workspace ws;
    ws.device = dev;
    ws.t = static_cast<float*>(scratch);
    ws.tgmax = ws.t + kNoAllocT;
    ws.partials = ws.tgmax + kNoAllocG;
    ws.counters = reinterpret_cast<int*>(ws.partials + kNoAllocP);
    ws.t_cap = kNoAllocT;
    ws.tgmax_cap = kNoAllocG;
    ws.partial_cap = kNoAllocP;
    ws.counter_cap = kNoAllocC;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws.counters, 0, sizeof(int) * kNoAllocC, s) != cudaSuccess) return NQ_ERR_CUDA;
    DecodeCall c{static_cast<const uint16_t*>(x), Upk, Vpk, static_cast<const uint16_t*>(s1),
                 static_cast<const uint16_t*>(s2), y, m, n, r};
    return decode_forward_group(&c, 1, batch, &ws, s, kNoAllocMaxSplits);
}
