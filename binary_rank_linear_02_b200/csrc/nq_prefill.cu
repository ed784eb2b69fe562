// nq_prefill.cu -- prefill path (batch > 8): the factorised linear as two dense
// tensor-core GEMMs on tcgen05 (hardwired.dev section "Cisla": binary GEMM kernels).
//
//   prescale : x'[b][.] = fp16(2^-e_b s2 (.) x[b])             (per token row, K-permuted)
//   GEMM 1   : T[b][k]  = sum_j V^T[k][j] x'[b][j]             M = r, N = batch, K = n
//   GEMM 2   : y[b][i]  = 2^e_b s1_i * sum_k U[i][k] T[b][k]   M = m, N = batch, K = r
//
// 2^-e_b is a power of two per token that keeps x' and T inside fp16's normal range
// (below 2^15 in magnitude) whatever the token's scale; it is undone exactly in GEMM 2's
// epilogue.
//
// Weights are the MMA's A operand (M = 128 rows per CTA), tokens its B operand (N = BN
// per CTA).  A is never stored expanded in memory: four "expander" warps read the packed
// sign words of their row, turn them into fp16 +1/-1 in registers and write the 128B-
// swizzled K-major tile the UMMA descriptor expects; B (x' or T, fp16) arrives by TMA.
// One thread issues tcgen05.mma (kind::f16, fp32 accumulators in tensor memory); the
// accumulators are read back (tcgen05.ld) for the epilogue, which writes T as fp16
// (GEMM 1) or y = s1 * acc as fp32 (GEMM 2).  Two GEMM kernels: a persistent one that
// splits K for small batches (at most 64 tokens), and one CTA per output tile above that.
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
#include "nq_sm100.cuh"

namespace nq {
namespace {

constexpr int kBM = 128;          // rows of A per CTA (tcgen05 M)
constexpr int kBK = 64;           // K elements per stage: one 128-byte swizzle atom of fp16
constexpr int kUmmaK = 16;        // K per tcgen05.mma (kind::f16)

// kind::f16 instruction descriptor: fp16 A and B, K-major both, fp32 D, M = 128, N = bn.
__host__ __device__ constexpr uint32_t idesc_f16(int bn) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
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

// ---------------------------------------------------------------------------- small batches
//
// Used up to 64 tokens, where a layer has fewer output tiles than the GPU has SMs.
// Persistent and warp-specialised: one CTA per SM walks a list of work items.  An item is
// a 128-row block of A (weights) times a tile of up to 256 tokens of B, over all of K or
// over one contiguous share of K (a "split").  Two schedules:
//  - units: the tokens of every row block are cut into 64-token units and each CTA takes
//    an equal run of consecutive units (to within one), cut into tiles of at most 4 units
//    inside a row block, so no SM idles while others finish a last wave;
//  - splits (few row blocks, at most 256 tokens): each row block's whole token range is
//    one tile and K is split so that every SM has work.  A split writes its fp32 partial
//    tile to the workspace; the CTA that completes a tile's last split (arrival counter)
//    adds the partials in split order (deterministic) and writes the output.
// The host picks the schedule with the smaller estimated time.
//
// Warp roles: warp 0 issues the TMA loads of B, warp 1 allocates tensor memory and issues
// tcgen05.mma, warps 2-5 expand the packed signs of A into shared memory, warps 6-9 read
// the accumulators back and write the output.  Tensor memory holds two 256-column fp32
// accumulators, so the read-out of one item overlaps the MMAs of the next.
constexpr int kMaxN = 256;                   // tokens per tile (tcgen05 N)
constexpr int kBox = 64;                     // rows of B per TMA box
constexpr int kMaxStages = 8;
constexpr int kABytes = kBM * kBK * 2;       // 16 KB of A per stage
constexpr int kBoxBytes = kBox * kBK * 2;    // 8 KB per 64 tokens of B per stage
constexpr int kGemmThreads = 320;
constexpr int kTmemCols = 2 * kMaxN;
// The A/B ring stays at 192 KB so that about 60 KB of the SM's unified L1 is left to cache
// the packed sign words the expanders read (measured: a 227 KB footprint slows every size).
constexpr int kRingBudget = 192 * 1024;
constexpr int kGemmSmemMax = kRingBudget + 1024 /*barriers*/ + 1024 /*alignment slack*/;
constexpr int kMaxSplits = 16;
constexpr int64_t kPersistentMaxBatch = 64;  // larger batches: the one-tile-per-CTA kernel below
constexpr size_t kPartialTileFloats = (size_t)kMaxN * kBM;  // [column][row] of one split item

struct Barriers {
    unsigned long long full_a[kMaxStages], full_b[kMaxStages], empty[kMaxStages];
    unsigned long long tmem_full[2], tmem_empty[2], drain;
    uint32_t tmem_base;
    int abort_flag;
    int last;    // epilogue: this CTA completes a split tile
    int epi_ok[2];  // epilogue: the accumulator of item i is ready (slot i & 1)
};

struct GemmArgs {
    const uint32_t* Wpk;  // M rows of K/32 words
    uint16_t* T_out;      // EPI 0: T[b][perm(k)] fp16
    float* y_out;         // EPI 1: y[b][i] fp32
    const uint16_t* s1;   // EPI 1
    const float* yscale;  // EPI 1: 2^e_b per token (the prescale's power of two, undone here)
    float* partials;      // split items: [row block][split][row][256 columns] fp32
    int* counters;        // split items: arrivals per row block, zero between calls
    unsigned* status;
    int64_t mdim, batch;
    int nkb;              // K / 64
    int nu;               // 64-token units per row block
    int64_t units;        // row blocks x nu
    int ks;               // 0: unit schedule; >= 1: split schedule with ks splits per row block
    int nrb;              // row blocks
    int stages;           // depth of the A/B ring
    int b_stage_bytes;    // B bytes per stage: widest tile of the launch x 128 B
};

struct Item {
    int64_t row0;  // first A row
    int col0;      // first token
    int ncols;     // valid tokens
    int n;         // MMA N: ncols rounded up to 16
    int nbox;      // TMA boxes of 64 tokens
    int kb0, kb1;  // k-blocks
    int split;     // split index
    int tt;        // split schedule with ks > 1: the row block (partials, counter); else -1
};

// Walks this CTA's items in order; every warp role runs its own copy.
struct ItemIter {
    int64_t u, u_end;  // unit schedule: next unit, end of this CTA's run
    int j;             // split schedule: next item index
};

__device__ __forceinline__ ItemIter item_begin(const GemmArgs& a) {
    ItemIter st;
    const int64_t P = gridDim.x, c = blockIdx.x;
    st.u = c * a.units / P;
    st.u_end = (c + 1) * a.units / P;
    st.j = (int)c;
    return st;
}

__device__ __forceinline__ bool item_next(const GemmArgs& a, ItemIter& st, Item& it) {
    if (a.ks == 0) {
        if (st.u >= st.u_end) return false;
        const int64_t rb = st.u / a.nu;
        const int cu = (int)(st.u % a.nu);
        int w = a.nu - cu;
        if (w > 4) w = 4;
        if ((int64_t)w > st.u_end - st.u) w = (int)(st.u_end - st.u);
        st.u += w;
        it.row0 = rb * kBM;
        it.col0 = cu * kBox;
        const int64_t left = a.batch - it.col0;
        it.ncols = (int)(left < (int64_t)w * kBox ? left : (int64_t)w * kBox);
        it.kb0 = 0;
        it.kb1 = a.nkb;
        it.split = 0;
        it.tt = -1;
    } else {
        if (st.j >= a.nrb * a.ks) return false;
        const int rb = st.j / a.ks;
        it.split = st.j % a.ks;
        st.j += (int)gridDim.x;
        it.row0 = (int64_t)rb * kBM;
        it.col0 = 0;
        it.ncols = (int)a.batch;
        it.kb0 = (int)((int64_t)it.split * a.nkb / a.ks);
        it.kb1 = (int)((int64_t)(it.split + 1) * a.nkb / a.ks);
        it.tt = a.ks > 1 ? rb : -1;
    }
    it.n = (it.ncols + 15) & ~15;
    it.nbox = (it.ncols + kBox - 1) / kBox;
    return true;
}

// Slot and phase of the A/B ring, advanced without a division.
struct Ring {
    int s = 0;
    uint32_t ph = 0;
    __device__ __forceinline__ void step(int S) {
        if (++s == S) {
            s = 0;
            ph ^= 1u;
        }
    }
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// ysc: the token's 2^e_b (EPI 1), passed in by the caller (one load per lane, broadcast
// by a shuffle, instead of a load per element).
template <int EPI>
__device__ __forceinline__ void store_out(const GemmArgs& a, int64_t b, int64_t grow, int64_t tcol, float s1v,
                                          float d, float ysc) {
    if (EPI == 0)
        a.T_out[b * a.mdim + tcol] = __half_as_ushort(__float2half_rn(d));
    else
        a.y_out[b * a.mdim + grow] = s1v * d * ysc;
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap bmap, const __grid_constant__ GemmArgs a) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const int S = a.stages, BSB = a.b_stage_bytes;
    // smem: S x A (16 KB) | S x B | barriers
    const uint32_t a_smem = base;
    const uint32_t b_smem = base + S * kABytes;
    Barriers& bar = *reinterpret_cast<Barriers*>(gbase + S * (kABytes + BSB));
    volatile int* abort_flag = &bar.abort_flag;
    unsigned* status = a.status;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t wpr = (int64_t)a.nkb * 2;  // words per A row

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&bar.full_a[s]), 128);
            mbar_init(smem_u32(&bar.full_b[s]), 1);
            mbar_init(smem_u32(&bar.empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bar.tmem_full[b]), 1);
            mbar_init(smem_u32(&bar.tmem_empty[b]), 128);
        }
        mbar_init(smem_u32(&bar.drain), 1);
        bar.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&bmap)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&bar.tmem_base)), "r"((uint32_t)kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    pdl_trigger();  // the next kernel may stage its own weights while this one runs

    if (warp == 0) {
        // ---------------- TMA producer of the B tiles (activations)
        if (lane == 0) {
            pdl_wait();  // B comes from the previous kernel (prescale or GEMM 1)
            int g = 0;
            Ring ring;
            bool ok = true;
            Item it;
            ItemIter st = item_begin(a);
            while (ok && item_next(a, st, it)) {
                for (int kb = it.kb0; kb < it.kb1; ++kb, ++g, ring.step(S)) {
                    const int s = ring.s;
                    const uint32_t ph = ring.ph;
                    if (!mbar_wait(smem_u32(&bar.empty[s]), ph ^ 1u, abort_flag, status)) { ok = false; break; }
                    mbar_expect_tx(smem_u32(&bar.full_b[s]), (uint32_t)(it.nbox * kBoxBytes));
                    for (int bx = 0; bx < it.nbox; ++bx)
                        tma_load_2d(b_smem + s * BSB + bx * kBoxBytes, &bmap, kb * kBK, it.col0 + bx * kBox,
                                    smem_u32(&bar.full_b[s]));
                }
            }
            if (!ok) {
                // let the loads already issued land before the CTA's shared memory goes away
                for (int q = g - S < 0 ? 0 : g - S; q < g; ++q)
                    mbar_drain(smem_u32(&bar.full_b[q % S]), (uint32_t)(q / S) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            int g = 0;
            Ring ring;
            bool ok = true;
            Item it;
            ItemIter st = item_begin(a);
            for (int i = 0; ok && item_next(a, st, it); ++i) {
                const int buf = i & 1;
                const uint32_t use = (uint32_t)(i >> 1) & 1u;
                if (!mbar_wait(smem_u32(&bar.tmem_empty[buf]), use ^ 1u, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * kMaxN);
                const uint32_t idesc = idesc_f16(it.n);
                for (int kb = it.kb0; kb < it.kb1; ++kb, ++g, ring.step(S)) {
                    const int s = ring.s;
                    const uint32_t ph = ring.ph;
                    if (!mbar_wait(smem_u32(&bar.full_a[s]), ph, abort_flag, status) ||
                        !mbar_wait(smem_u32(&bar.full_b[s]), ph, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(a_smem + s * kABytes);
                    const uint64_t bd = sw128_desc(b_smem + s * BSB);
#pragma unroll
                    for (int k = 0; k < kBK / kUmmaK; ++k)
                        umma_f16(d, ad + (uint64_t)(k * kUmmaK * 2 / 16), bd + (uint64_t)(k * kUmmaK * 2 / 16), idesc,
                                 (kb > it.kb0 || k > 0) ? 1u : 0u);
                    umma_commit(smem_u32(&bar.empty[s]));
                }
                if (ok) umma_commit(smem_u32(&bar.tmem_full[buf]));
            }
            if (!ok) {
                // aborted: make sure the MMAs already issued are finished before teardown
                umma_commit(smem_u32(&bar.drain));
                mbar_drain(smem_u32(&bar.drain), 0);
            }
        }
    } else if (warp < 6) {
        // ---------------- expanders: one thread per A row
        const int row = threadIdx.x - 64;  // 0..127
        const uint32_t a_row_off = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
        int g = 0;
        Ring ring;
        bool ok = true;
        Item it;
        ItemIter st = item_begin(a);
        while (ok && item_next(a, st, it)) {
            const uint2* wrow = reinterpret_cast<const uint2*>(a.Wpk + (it.row0 + row) * wpr);  // one uint2 per k-block
            uint2 w0 = __ldg(wrow + it.kb0);
            uint2 w1 = it.kb0 + 1 < it.kb1 ? __ldg(wrow + it.kb0 + 1) : make_uint2(0, 0);
            for (int kb = it.kb0; kb < it.kb1; ++kb, ++g, ring.step(S)) {
                const int s = ring.s;
                const uint32_t ph = ring.ph;
                const uint2 cur = w0;
                w0 = w1;
                if (kb + 2 < it.kb1) w1 = __ldg(wrow + kb + 2);
                if (!mbar_wait(smem_u32(&bar.empty[s]), ph ^ 1u, abort_flag, status)) { ok = false; break; }
                uint32_t h0[16], h1[16];
                expand_word(cur.x, h0);
                expand_word(cur.y, h1);
                const uint32_t dst = a_smem + s * kABytes + a_row_off;
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
            }
        }
    } else {
        // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = rows of the tile
        const int quad = warp & 3;
        const int r_in_tile = quad * 32 + lane;
        const int et = threadIdx.x - 192;  // 0..127
        Item it;
        ItemIter st = item_begin(a);
        for (int i = 0; item_next(a, st, it); ++i) {
            const int buf = i & 1;
            const uint32_t use = (uint32_t)(i >> 1) & 1u;
            // one thread waits and tells the others, so that all 128 leave together on an abort
            // (two slots: the waiting thread may reach the next item before a slow one has read this)
            if (et == 0) bar.epi_ok[buf] = mbar_wait(smem_u32(&bar.tmem_full[buf]), use, abort_flag, status);
            epi_bar();
            if (!bar.epi_ok[buf]) break;
            tc_fence_after();
            const int64_t grow = it.row0 + r_in_tile;
            const float s1v = EPI == 1 ? __half2float(__ushort_as_half(a.s1[grow])) : 1.f;
            const int64_t tcol = EPI == 0 ? (grow & ~31ll) + kperm((int)(grow & 31)) : 0;
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * kMaxN);
            // split partial: [row][256 columns] fp32, this thread's row contiguous
            float* part = it.tt >= 0
                              ? a.partials + (size_t)(it.tt * a.ks + it.split) * kPartialTileFloats + (size_t)r_in_tile * kMaxN
                              : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < it.n; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + (uint32_t)c0, v);
                if (it.tt < 0) {
                    const float ysc_l = (EPI == 1 && c0 + lane < it.ncols) ? __ldg(a.yscale + it.col0 + c0 + lane) : 1.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float ysc = __shfl_sync(__activemask(), ysc_l, j);
                        if (c0 + j < it.ncols)
                            store_out<EPI>(a, it.col0 + c0 + j, grow, tcol, s1v, __uint_as_float(v[j]), ysc);
                    }
                } else {
                    float4* q = reinterpret_cast<float4*>(part + c0);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        q[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                           __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&bar.tmem_empty[buf]));  // the MMA warp may reuse this accumulator
            if (it.tt >= 0) {
                epi_bar();
                if (et == 0) {
                    __threadfence();
                    bar.last = atomicAdd(a.counters + it.tt, 1) == a.ks - 1;
                }
                epi_bar();
                if (bar.last) {
                    __threadfence();
                    const float* p0 = a.partials + (size_t)it.tt * a.ks * kPartialTileFloats + (size_t)r_in_tile * kMaxN;
                    for (int c0 = 0; c0 < it.ncols; c0 += 16) {
                        float4 acc[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
                        for (int sp = 0; sp < a.ks; ++sp) {
                            const float4* q4 = reinterpret_cast<const float4*>(p0 + (size_t)sp * kPartialTileFloats + c0);
                            float4 v4[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) v4[q] = __ldcg(q4 + q);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                acc[q].x += v4[q].x;
                                acc[q].y += v4[q].y;
                                acc[q].z += v4[q].z;
                                acc[q].w += v4[q].w;
                            }
                        }
                        const float* accf = reinterpret_cast<const float*>(acc);
                        const float ysc_l =
                            (EPI == 1 && c0 + (lane & 15) < it.ncols) ? __ldg(a.yscale + it.col0 + c0 + (lane & 15)) : 1.f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float ysc = __shfl_sync(__activemask(), ysc_l, j);
                            if (c0 + j < it.ncols) store_out<EPI>(a, it.col0 + c0 + j, grow, tcol, s1v, accf[j], ysc);
                        }
                    }
                    if (et == 0) a.counters[it.tt] = 0;  // ready for the next call
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTmemCols));
    }
}

constexpr int kTileThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 expand + epilogue
// Two CTAs per SM (up to 104 KB each: 4 stages at BN = 64, 3 at 128 and 144, 2 at 176 and
// 256), so that one CTA's epilogue runs while the other's MMAs do.  Measured against one
// CTA per SM with twice the stages: 103 vs 129 us at 1024 tokens, 49 vs 57 us at 256.
constexpr int kTileSmemBudget = 112 * 1024;

template <int BN>
struct Geometry {
    static constexpr int kABytes = kBM * kBK * 2;          // 16 KB per stage
    static constexpr int kBBytes = BN * kBK * 2;           // BN rows x 128 B
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = (kTileSmemBudget - 2048) / kStageBytes > 8 ? 8 : (kTileSmemBudget - 2048) / kStageBytes;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*barriers*/ + 1024 /*alignment slack*/;
    static constexpr int kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;  // a power of 2
};

struct TileBarriers {
    unsigned long long full_a[8], full_b[8], empty[8];
    unsigned long long tmem_full, drain;
    uint32_t tmem_base;
    int abort_flag;
};

// ---------------------------------------------------------------------------- large batches
//
// One CTA per 128 x BN output tile (grid = row blocks x token tiles, about two waves or
// more): D = A . B^T with A = expanded signs (rows m0..m0+127 of `Wpk`, K = kdim) and B =
// TMA tiles of `bmap` (rows n0..n0+BN-1).  Warp 0 loads B, warp 1 issues the MMAs, warps
// 2-5 expand A and then read the accumulator back.  EPI 0: T[b][perm(k)] = fp16(D)
// (GEMM 1);  EPI 1: y[b][i] = s1_i * D (GEMM 2).  Measured on a B200 on the 11008 x 4096,
// r = 2432 layer: faster than the persistent kernel above from 128 tokens up (41.8 vs
// 55.7 us at 128, 273 vs 306 us at 4096), level at 64, slower below (39.5 vs 32.2 us at
// 16).  Its epilogue does not overlap the next tile's MMAs, but neither does it compete
// with them: with the persistent kernel's overlapped epilogue the global stores slowed the
// main loop (27 us of 306 at 4096 tokens).
//
// Hand-off from GEMM 1 to GEMM 2 by token tile (`handoff`, for a GEMM 1 of more tiles than
// one wave holds): a GEMM 1 CTA releases its dependants as soon as its own dependency wait
// is over and, once its tile of T is stored, adds one to the counter of its token tile
// (sync[tile]); a GEMM 2 CTA waits only for the counters of the GEMM 1 token tiles its own
// tokens fall in (every row block of GEMM 1 done), so GEMM 2 fills the SMs that GEMM 1's
// last wave leaves idle.  The GEMM 2 CTAs that depend on a token tile count themselves past
// the wait in sync[ntt1 + tile]; the last one clears both counters for the next call.  The
// waits are bounded (NQ_ERR_TIMEOUT in the status word).  Without it GEMM 1 releases GEMM 2
// from its epilogue and GEMM 2 waits for all of GEMM 1.  Measured on the 11008 x 4096,
// r = 2432 layer: 4096 tokens (GEMM 1: 304 tiles for 296 slots) 268 -> 256 us with it;
// below, where GEMM 1 fits one wave, GEMM 2's early CTAs only crowd GEMM 1's SMs (1024
// tokens 101.6 us without, 103.8 us with).
template <int BN, int EPI>
__global__ void __launch_bounds__(kTileThreads, 2)
tile_gemm_kernel(const __grid_constant__ CUtensorMap bmap, const uint32_t* __restrict__ Wpk, int64_t kdim,
            int64_t mdim, int64_t batch, uint16_t* __restrict__ T_out, float* __restrict__ y_out,
            const uint16_t* __restrict__ s1, const float* __restrict__ yscale, unsigned* __restrict__ status,
            int* __restrict__ sync, int bn1, int ntt1, int nrb1, int handoff) {
    using G = Geometry<BN>;
    constexpr int S = G::kStages;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    TileBarriers& bar = *reinterpret_cast<TileBarriers*>(gbase + S * G::kStageBytes);
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
            if (EPI == 0 || !handoff) {
                pdl_wait();  // B comes from the previous kernel (prescale or GEMM 1)
                if (handoff) pdl_trigger();  // GEMM 2 may launch: it waits on the token-tile counters
            } else {
                // B = T: the GEMM 1 token tiles that hold tokens n0 .. n0 + BN - 1
                const int tt0 = (int)(n0 / bn1);
                const int tt1 = (int)(((n0 + BN < batch ? n0 + BN : batch) - 1) / bn1);
                bool ok = true;
                for (int tt = tt0; tt <= tt1 && ok; ++tt) ok = wait_count(sync + tt, nrb1, status);
                if (ok) {
                    fence_proxy_async_global();
                    for (int tt = tt0; tt <= tt1; ++tt) {
                        // GEMM 2 CTAs that read token tile tt: all row blocks x the GEMM 2
                        // token tiles overlapping it
                        const int64_t e1 = ((int64_t)(tt + 1) * bn1 < batch ? (int64_t)(tt + 1) * bn1 : batch) - 1;
                        const int users = (int)gridDim.x * (int)(e1 / BN - (int64_t)tt * bn1 / BN + 1);
                        if (atomicAdd(sync + ntt1 + tt, 1) == users - 1) {
                            sync[tt] = 0;
                            sync[ntt1 + tt] = 0;
                        }
                    }
                } else {
                    *abort_flag = 1;
                }
            }
            int issued = 0;
            const int nkb_go = *abort_flag ? 0 : nkb;  // none after a failed wait
            for (int kb = 0; kb < nkb_go; ++kb) {
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
                const int64_t bl = n0 + c0 + lane;
                const float ysc_l = (EPI == 1 && c0 + lane < BN && bl < batch) ? __ldg(yscale + bl) : 1.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int64_t b = n0 + c0 + j;
                    const float ysc = __shfl_sync(__activemask(), ysc_l, j);
                    if (c0 + j < BN && b < batch) {  // BN need not be a multiple of 32
                        const float d = __uint_as_float(v[j]);
                        if (EPI == 0)
                            T_out[b * mdim + tcol] = __half_as_ushort(__float2half_rn(d));
                        else
                            y_out[b * mdim + grow] = s1v * d * ysc;
                    }
                }
            }
        }
        if (EPI == 0 && handoff) {  // the tile of T is stored: count it for its token tile
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (threadIdx.x == 64 && !*abort_flag) {
                __threadfence();
                atomicAdd(sync + blockIdx.y, 1);
            }
        }
    }

    // GEMM 2 completes only after GEMM 1 has, so that the next kernel's dependency wait covers both
    if (EPI == 1 && threadIdx.x == 0) pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)G::kTmemCols));
    }
}

// Self-test of the failure path: the GEMMs' bounded mbarrier wait on a barrier that
// nothing arrives on, with a short limit; it gives up, records NQ_ERR_TIMEOUT in the
// status word exactly as a GEMM would, and the kernel exits.
__global__ void wait_selftest_kernel(unsigned long long limit_ns, unsigned* status) {
    __shared__ unsigned long long bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
}

// x'[b][perm(j)] = fp16(2^-e_b * bf16 x[b][j] * fp16 s2[j]) and xscale[b] = 2^e_b.  The power of two is chosen per token from the row's sum
// L_b = sum_j |s2_j x[b][j]| (fp32) so that 2^-e_b L_b < 2^15: every |x'| and every entry
// of T = V^T x' (each a signed sum of the x') then stays below 2^15 < 65504, so neither
// overflows fp16, and every token uses fp16's normal range down to 2^-29 L_b whatever its
// magnitude (without it a token of small activations falls into fp16's subnormals and a
// token of large ones overflows T).  GEMM 2's epilogue multiplies by 2^e_b, which is exact,
// so the result is that of the unscaled operands up to their rounding.
constexpr int kPrescaleThreads = 256;

__device__ __forceinline__ float prescale_pow2(int k) { return __int_as_float((k + 127) << 23); }  // |k| <= 126

// TPR threads per token row (32 .. 256, a power of two: about one 32-column group each),
// kPrescaleThreads / TPR rows per CTA at a time; the row's sum is reduced by a warp
// shuffle and, across the row's warps, through shared memory in warp order.
template <int TPR>
__global__ void __launch_bounds__(kPrescaleThreads)
prescale_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ s2, int64_t n, int64_t batch,
                uint16_t* __restrict__ xp, float* __restrict__ xscale) {
    constexpr int kRows = kPrescaleThreads / TPR, kWarpsPerRow = TPR / 32;
    __shared__ float red[kPrescaleThreads / 32];
    const int64_t groups = n / 32;
    const int sub = threadIdx.x / TPR, tid = threadIdx.x % TPR, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    // every CTA runs the same number of iterations (the barrier below is CTA-wide)
    const int64_t iters = (batch + (int64_t)gridDim.x * kRows - 1) / ((int64_t)gridDim.x * kRows);
    for (int64_t it = 0; it < iters; ++it) {
        const int64_t b = (it * gridDim.x + blockIdx.x) * kRows + sub;
        const bool live = b < batch;
        const uint16_t* xrow = x + (live ? b : 0) * n;
        // column c of a group sits in half (c & 1) of word c / 2
        auto load = [&](int64_t g, uint32_t (&xv)[16], uint32_t (&sv)[16]) {
            const uint4* xs = reinterpret_cast<const uint4*>(xrow + g * 32);
            const uint4* ss = reinterpret_cast<const uint4*>(s2 + g * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 a = __ldg(xs + i), c = __ldg(ss + i);
                xv[4 * i] = a.x; xv[4 * i + 1] = a.y; xv[4 * i + 2] = a.z; xv[4 * i + 3] = a.w;
                sv[4 * i] = c.x; sv[4 * i + 1] = c.y; sv[4 * i + 2] = c.z; sv[4 * i + 3] = c.w;
            }
        };
        auto value = [](const uint32_t (&xv)[16], const uint32_t (&sv)[16], int c) {
            const uint16_t xb = (uint16_t)(xv[c >> 1] >> (16 * (c & 1)));
            const uint16_t sb = (uint16_t)(sv[c >> 1] >> (16 * (c & 1)));
            return __uint_as_float((uint32_t)xb << 16) * __half2float(__ushort_as_half(sb));  // exact in fp32
        };
        float l1 = 0.f;
        if (live)
            for (int64_t g = tid; g < groups; g += TPR) {
                uint32_t xv[16], sv[16];
                load(g, xv, sv);
#pragma unroll
                for (int c = 0; c < 32; ++c) l1 += fabsf(value(xv, sv, c));
            }
        for (int o = 16; o > 0; o >>= 1) l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        if (kWarpsPerRow > 1) {
            if (lane == 0) red[warp] = l1;
            __syncthreads();
            l1 = 0.f;
#pragma unroll
            for (int w = 0; w < kWarpsPerRow; ++w) l1 += red[sub * kWarpsPerRow + w];
            __syncthreads();  // red is rewritten in the next iteration
        }
        if (!live) continue;
        int e = 0;
        frexpf(l1, &e);  // l1 < 2^e (e = 0 for a zero row)
        e = min(max(e - 15, -110), 112);
        const float down = prescale_pow2(-e);
        if (tid == 0) xscale[b] = prescale_pow2(e);
        for (int64_t g = tid; g < groups; g += TPR) {
            uint32_t xv[16], sv[16], out[16];
            load(g, xv, sv);
            // output pair q = (column q, column q+16)
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                uint32_t pair = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    pair |= (uint32_t)__half_as_ushort(__float2half_rn(value(xv, sv, q + 16 * h) * down)) << (16 * h);
                out[q] = pair;
            }
            uint4* o = reinterpret_cast<uint4*>(xp + b * n + g * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
        }
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

// 2D tensor [rows][cols] (row-major) of 2- or 4-byte elements, box = box_cols x box_rows.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int box_cols, int box_rows, bool f32,
              bool swizzle) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int esz = f32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * esz)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                    const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Work plan of one GEMM (M rows of A, K, `batch` tokens) on `sms` SMs.
struct Plan {
    int nkb, nu, nrb, ks, grid;  // ks == 0: unit schedule, else split schedule
    int64_t units;
};

// Relative cost of one k-block step of a tile of n tokens: the MMAs (4 x 128 x n x 16 at
// 8192 flop per clock: 2 clocks per token) or the sign expansion (~160 clocks).  (Scaling
// the floor to the ~1000 clocks a step measures at 16 tokens made the plan choose more
// splits, which measured slower: the split items' partials and reduction cost more than
// the model's estimate, so the low floor stands in for both.)
double step_clk(int64_t n) {
    const double mma = 2.0 * (double)((n + 15) & ~15ll);
    return mma > 160.0 ? mma : 160.0;
}

// The busiest CTA of the unit schedule, in clocks.
double unit_cost(int64_t nrb, int nu, int64_t batch, int nkb, int P) {
    const int64_t units = nrb * nu;
    double worst = 0.0;
    for (int c = 0; c < P; ++c) {
        int64_t u = (int64_t)c * units / P;
        const int64_t ue = (int64_t)(c + 1) * units / P;
        double cost = 0.0;
        while (u < ue) {
            const int cu = (int)(u % nu);
            int64_t w = nu - cu;
            if (w > 4) w = 4;
            if (w > ue - u) w = ue - u;
            const int64_t left = batch - (int64_t)cu * kBox;
            cost += nkb * step_clk(left < w * kBox ? left : w * kBox);
            u += w;
        }
        worst = cost > worst ? cost : worst;
    }
    return worst;
}

Plan plan_gemm(int64_t M, int64_t K, int64_t batch, int sms) {
    Plan p;
    p.nkb = (int)(K / kBK);
    p.nu = (int)((batch + kBox - 1) / kBox);
    p.nrb = (int)(M / kBM);
    p.units = (int64_t)p.nrb * p.nu;
    p.ks = 0;
    const int units_grid = (int)(p.units < sms ? p.units : sms);
    double best = unit_cost(p.nrb, p.nu, batch, p.nkb, units_grid);
    if (p.nu <= 4) {
        // split schedule: one tile per row block, K in ks shares; a split also writes its
        // partial tile, and the last one reads ks of them back (a 16-column group of 4
        // splits per L2 round trip of ~800 clocks).  Partials are capped at 64 MB.
        for (int ks = 1; ks <= kMaxSplits && ks <= p.nkb; ++ks) {
            if (ks > 1 && (double)p.nrb * ks * kPartialTileFloats * 4 > 64.0 * (1 << 20)) break;
            const int64_t items = (int64_t)p.nrb * ks;
            double cost = (double)((items + sms - 1) / sms) * (double)((p.nkb + ks - 1) / ks) * step_clk(batch);
            if (ks > 1) cost += 1500.0 + 800.0 * (double)((batch + 15) / 16) * (double)((ks + 3) / 4);
            if (cost < best) {
                best = cost;
                p.ks = ks;
            }
        }
    }
    if (p.ks == 0) {
        p.grid = units_grid;
    } else {
        const int64_t items = (int64_t)p.nrb * p.ks;
        p.grid = (int)(items < sms ? items : sms);
    }
    return p;
}

template <int EPI>
int launch_gemm(const CUtensorMap& map, const uint32_t* Wpk, int64_t M, int64_t K, int64_t batch, uint16_t* T_out,
                float* y_out, const uint16_t* s1, Workspace* ws, cudaStream_t stream) {
    const Plan p = plan_gemm(M, K, batch, sm_count());
    GemmArgs a;
    a.Wpk = Wpk;
    a.T_out = T_out;
    a.y_out = y_out;
    a.s1 = s1;
    a.yscale = ws->xscale;
    a.partials = ws->partials;
    a.counters = ws->counters;
    a.status = ws->status + 1;
    a.mdim = M;
    a.batch = batch;
    a.nkb = p.nkb;
    a.nu = p.nu;
    a.units = p.units;
    a.ks = p.ks;
    a.nrb = p.nrb;
    // ring: B sized for the widest tile of the launch, as many stages as fit (at most 8)
    const int wide = p.nu < 4 ? p.nu : 4;
    a.b_stage_bytes = wide * kBoxBytes;
    a.stages = kRingBudget / (kABytes + a.b_stage_bytes);
    if (a.stages > kMaxStages) a.stages = kMaxStages;
    const size_t smem = 1024 + (size_t)a.stages * (kABytes + a.b_stage_bytes) + 1024;
    if (p.ks > 1 &&
        ((size_t)p.nrb * p.ks * kPartialTileFloats > ws->partial_cap || (size_t)p.nrb > ws->counter_cap))
        return NQ_ERR_NOMEM;
    return launch_pdl(gemm_kernel<EPI>, dim3((unsigned)p.grid), dim3(kGemmThreads), smem, stream, map, a) ==
                   cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}

cudaError_t launch_prescale(const uint16_t* x, const uint16_t* s2, int64_t n, int64_t batch, Workspace* ws,
                            cudaStream_t stream) {
    // threads per row: the row's 32-column groups rounded up to a power of two, 32 .. 256
    const int64_t groups = n / 32;
    int tpr = 32;
    while (tpr < 256 && tpr < groups) tpr *= 2;
    const int64_t rows_per_cta = kPrescaleThreads / tpr;
    const int64_t want = (batch + rows_per_cta - 1) / rows_per_cta, cap = 8 * (int64_t)sm_count();
    const dim3 grid((unsigned)(want < cap ? want : cap)), block(kPrescaleThreads);
    switch (tpr) {
        case 32: return launch_pdl(prescale_kernel<32>, grid, block, 0, stream, x, s2, n, batch, ws->xprime, ws->xscale);
        case 64: return launch_pdl(prescale_kernel<64>, grid, block, 0, stream, x, s2, n, batch, ws->xprime, ws->xscale);
        case 128: return launch_pdl(prescale_kernel<128>, grid, block, 0, stream, x, s2, n, batch, ws->xprime, ws->xscale);
        default: return launch_pdl(prescale_kernel<256>, grid, block, 0, stream, x, s2, n, batch, ws->xprime, ws->xscale);
    }
}

template <int BN, int EPI>
int launch_tile_gemm(const void* bsrc, int64_t K, const uint32_t* Wpk, int64_t M, int64_t batch, uint16_t* T_out,
                     float* y_out, const uint16_t* s1, Workspace* ws, cudaStream_t stream, int bn1, int nrb1) {
    using G = Geometry<BN>;
    static unsigned long long init_mask = 0;
    const unsigned long long bit = 1ull << (ws->device & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (cudaFuncSetAttribute(tile_gemm_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 G::kSmemBytes) != cudaSuccess)
            return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    CUtensorMap map;
    if (!make_map(&map, bsrc, batch, K, kBK, BN, false, true)) return NQ_ERR_CUDA;
    const unsigned ntiles = (unsigned)((batch + BN - 1) / BN);
    const int ntt1 = (int)((batch + bn1 - 1) / bn1);  // GEMM 1 token tiles
    // the hand-off when GEMM 1's tiles exceed one wave (two CTAs per SM)
    const int handoff = (int64_t)nrb1 * ntt1 > 2 * (int64_t)sm_count() ? 1 : 0;
    return launch_pdl(tile_gemm_kernel<BN, EPI>, dim3((unsigned)(M / kBM), ntiles), dim3(kTileThreads),
                      (size_t)G::kSmemBytes, stream, map, Wpk, K, M, batch, T_out, y_out, s1,
                      (const float*)ws->xscale, ws->status + 1, ws->counters, bn1, ntt1, nrb1, handoff) == cudaSuccess
               ? NQ_OK
               : NQ_ERR_CUDA;
}

// Token-tile width of one GEMM (M rows of A, `batch` tokens): the candidate with the least
// estimated time, (tiles per SM, rounded up) x (BN + 200), the 200 standing for the
// per-k-block cost that does not shrink with the tile (sign expansion, ring hand-offs).
// Fitted to a sweep of all width pairs on the 11008 x 4096, r = 2432 layer on a B200
// (within 3 % of the best pair from 128 to 4096 tokens); e.g. 517 tokens: GEMM 2 at 176
// wide, 59 us against 71 us at 128; 2048 tokens: GEMM 1 at 144, 144 us against 151 us.
int choose_bn(int64_t M, int64_t batch, int sms) {
    if (batch <= 256) return 128;  // measured best for both GEMMs up to 256 tokens
    static const int cand[] = {64, 128, 144, 176, 256};
    int best = 256;
    double best_t = 1e300;
    for (int bn : cand) {
        const int64_t tiles = (M / kBM) * ((batch + bn - 1) / bn);
        const double t = (double)((tiles + sms - 1) / sms) * (bn + 200);
        if (t < best_t - 1e-9) {
            best_t = t;
            best = bn;
        }
    }
    return best;
}

// bn1, nrb1: GEMM 1's token-tile width and row blocks (the token-tile counters' layout)
template <int EPI>
int launch_tile_gemm_bn(int bn, const void* bsrc, int64_t K, const uint32_t* Wpk, int64_t M, int64_t batch,
                        uint16_t* T_out, float* y_out, const uint16_t* s1, Workspace* ws, cudaStream_t stream,
                        int bn1, int nrb1) {
    switch (bn) {
        case 64: return launch_tile_gemm<64, EPI>(bsrc, K, Wpk, M, batch, T_out, y_out, s1, ws, stream, bn1, nrb1);
        case 128: return launch_tile_gemm<128, EPI>(bsrc, K, Wpk, M, batch, T_out, y_out, s1, ws, stream, bn1, nrb1);
        case 144: return launch_tile_gemm<144, EPI>(bsrc, K, Wpk, M, batch, T_out, y_out, s1, ws, stream, bn1, nrb1);
        case 176: return launch_tile_gemm<176, EPI>(bsrc, K, Wpk, M, batch, T_out, y_out, s1, ws, stream, bn1, nrb1);
        default: return launch_tile_gemm<256, EPI>(bsrc, K, Wpk, M, batch, T_out, y_out, s1, ws, stream, bn1, nrb1);
    }
}

int run_tile_gemms(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                   const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y, Workspace* ws,
                   cudaStream_t stream) {
    if (launch_prescale(x, s2, n, batch, ws, stream) != cudaSuccess) return NQ_ERR_CUDA;
    const int sms = sm_count();
    const int bn1 = choose_bn(r, batch, sms), nrb1 = (int)(r / kBM);
    int st = launch_tile_gemm_bn<0>(bn1, ws->xprime, n, Vpk, r, batch, ws->T, nullptr, nullptr, ws, stream, bn1, nrb1);
    if (st != NQ_OK) return st;
    return launch_tile_gemm_bn<1>(choose_bn(m, batch, sms), ws->T, r, Upk, m, batch, nullptr, y, s1, ws, stream, bn1,
                                  nrb1);
}

}  // namespace

bool encode_map_u32_sw128(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int box_cols, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 4)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int selftest_wait_timeout(int64_t limit_ns, Workspace* ws, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_ns, ws->status + 1);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

void prefill_workspace_need(int64_t m, int64_t n, int64_t r, int64_t batch, int64_t* partial_floats,
                            int64_t* counter_ints) {
    const int sms = sm_count();
    int64_t pf = 0, ci = 0;
    if (batch > kPersistentMaxBatch) {  // the token-tile counters of the GEMM 1 -> GEMM 2 hand-off
        *partial_floats = 0;
        *counter_ints = 2 * ((batch + 63) / 64);
        return;
    }
    const Plan p1 = plan_gemm(r, n, batch, sms), p2 = plan_gemm(m, r, batch, sms);
    for (const Plan& p : {p1, p2}) {
        if (p.ks > 1) {
            const int64_t f = (int64_t)p.nrb * p.ks * (int64_t)kPartialTileFloats;
            pf = f > pf ? f : pf;
            ci = p.nrb > ci ? p.nrb : ci;
        }
    }
    *partial_floats = pf;
    *counter_ints = ci;
}

// t = V^T (s2 (.) x) in fp32 (batch x r, row-major) for more than NQ_DECODE_MAX_BATCH
// tokens: the prescale and GEMM 1 with the y epilogue (fp32, times the token's 2^e) and unit
// scales (`ones`, r fp16 1.0) in place of s1.
int prefill_rank_vector(const uint16_t* x, const uint32_t* Vpk, const uint16_t* s2, int64_t n, int64_t r,
                        int64_t batch, float* t, const uint16_t* ones, Workspace* ws, cudaStream_t stream) {
    if (batch > kPersistentMaxBatch) {
        if (launch_prescale(x, s2, n, batch, ws, stream) != cudaSuccess) return NQ_ERR_CUDA;
        const int bn = choose_bn(r, batch, sm_count());
        // bn1 = bn, nrb1 = 1: no token-tile hand-off (there is no GEMM 1 to wait for)
        return launch_tile_gemm_bn<1>(bn, ws->xprime, n, Vpk, r, batch, nullptr, t, ones, ws, stream, bn, 1);
    }
    static unsigned long long init_mask = 0;
    const unsigned long long bit = 1ull << (ws->device & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (cudaFuncSetAttribute(gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemMax) !=
            cudaSuccess)
            return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    CUtensorMap map_x;
    if (!make_map(&map_x, ws->xprime, batch, n, kBK, kBox, false, true)) return NQ_ERR_CUDA;
    if (launch_prescale(x, s2, n, batch, ws, stream) != cudaSuccess) return NQ_ERR_CUDA;
    return launch_gemm<1>(map_x, Vpk, r, n, batch, nullptr, t, ones, ws, stream);
}

int prefill_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                    const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                    Workspace* ws, cudaStream_t stream) {
    if (batch > kPersistentMaxBatch) return run_tile_gemms(x, Upk, Vpk, s1, s2, m, n, r, batch, y, ws, stream);
    static unsigned long long init_mask = 0;
    const unsigned long long bit = 1ull << (ws->device & 63);
    if (!(__atomic_load_n(&init_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (cudaFuncSetAttribute(gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemMax) !=
                cudaSuccess ||
            cudaFuncSetAttribute(gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemMax) !=
                cudaSuccess)
            return NQ_ERR_CUDA;
        __atomic_fetch_or(&init_mask, bit, __ATOMIC_RELEASE);
    }
    CUtensorMap map_x, map_t;
    if (!make_map(&map_x, ws->xprime, batch, n, kBK, kBox, false, true) ||
        !make_map(&map_t, ws->T, batch, r, kBK, kBox, false, true))
        return NQ_ERR_CUDA;
    if (launch_prescale(x, s2, n, batch, ws, stream) != cudaSuccess) return NQ_ERR_CUDA;
    int st = launch_gemm<0>(map_x, Vpk, r, n, batch, ws->T, nullptr, nullptr, ws, stream);
    if (st != NQ_OK) return st;
    return launch_gemm<1>(map_t, Upk, m, r, batch, nullptr, y, s1, ws, stream);
}

}  // namespace nq
