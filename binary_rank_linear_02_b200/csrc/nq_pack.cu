// nq_pack.cu -- one-bit storage of sign matrices on the device: packing, unpacking and
// the transpose of a packed matrix (the backward pass reads U and V along the other axis).
//
// The stored form (one bit per +1/-1 entry, hardwired.dev section "Jak NanoQuant
// funguje"; bit 1 = +1, least significant bit = lowest column, sign(0) = +1) is the
// contract of nq.h.  One thread builds one 32-bit word from 32 consecutive int8 entries
// of a row, read as two 16-byte vectors when the row slice is aligned.
#include "nq_internal.cuh"

namespace nq {
namespace {

__global__ void pack_kernel(const int8_t* __restrict__ signs, int64_t rows, int64_t cols, int64_t wpr,
                            uint32_t* __restrict__ out, unsigned* __restrict__ flag) {
    const int64_t total = rows * wpr;
    const bool vec_ok = (cols % 32) == 0 && (reinterpret_cast<uintptr_t>(signs) % 16) == 0;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = idx / wpr, w = idx % wpr;
        const int8_t* src = signs + row * cols + 32 * w;
        uint32_t word = 0;
        bool bad = false;
        if (vec_ok) {
            const int4* v = reinterpret_cast<const int4*>(src);
            int4 lo = v[0], hi = v[1];
            const int32_t parts[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int p = 0; p < 8; ++p) {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    int8_t s = (int8_t)((parts[p] >> (8 * b)) & 0xFF);
                    bad |= (s < -1) | (s > 1);
                    word |= (s >= 0 ? 1u : 0u) << (4 * p + b);
                }
            }
        } else {
            for (int b = 0; b < 32; ++b) {
                int64_t col = 32 * w + b;
                if (col < cols) {
                    int8_t s = src[b];
                    bad |= (s < -1) | (s > 1);
                    word |= (s >= 0 ? 1u : 0u) << b;
                }
            }
        }
        if (bad) atomicOr(flag, 1u);
        out[idx] = word;
    }
}

__global__ void unpack_kernel(const uint32_t* __restrict__ packed, int64_t rows, int64_t cols, int64_t wpr,
                              int8_t* __restrict__ out) {
    const int64_t total = rows * cols;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = idx / cols, col = idx % cols;
        uint32_t word = packed[row * wpr + col / 32];
        out[idx] = ((word >> (col % 32)) & 1u) ? (int8_t)1 : (int8_t)-1;
    }
}

// Transpose of a packed sign matrix, one warp per 32 x 32 tile: lane l holds the word of
// input row 32*tr + l for column block tc; ballot c collects bit c of the 32 words, i.e. the
// word of output row 32*tc + c for row block tr, and lane c keeps it.  Rows beyond the
// matrix read as zero words, so the unused high bits of the output stay zero.
__global__ void transpose_kernel(const uint32_t* __restrict__ in, int64_t rows, int64_t cols, int64_t wpr_in,
                                 int64_t wpr_out, uint32_t* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t tiles_c = wpr_in, tiles = ((rows + 31) / 32) * tiles_c;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t tile = blockIdx.x * (int64_t)(blockDim.x / 32) + (threadIdx.x >> 5); tile < tiles; tile += warps) {
        const int64_t tr = tile / tiles_c, tc = tile % tiles_c;
        const int64_t row = 32 * tr + lane;
        const uint32_t w = row < rows ? in[row * wpr_in + tc] : 0u;
        uint32_t mine = 0;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const uint32_t b = __ballot_sync(0xffffffffu, (w >> c) & 1u);
            if (lane == c) mine = b;
        }
        const int64_t col = 32 * tc + lane;
        if (col < cols) out[col * wpr_out + tr] = mine;
    }
}

int grid_for(int64_t items, int threads) {
    int64_t blocks = (items + threads - 1) / threads;
    int64_t cap = (int64_t)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

int pack_device(const int8_t* signs, int64_t rows, int64_t cols, uint32_t* out, unsigned* flag,
                cudaStream_t stream) {
    const int64_t wpr = (cols + 31) / 32;
    const int threads = 256;
    pack_kernel<<<grid_for(rows * wpr, threads), threads, 0, stream>>>(signs, rows, cols, wpr, out, flag);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

int unpack_device(const uint32_t* packed, int64_t rows, int64_t cols, int8_t* out, cudaStream_t stream) {
    const int64_t wpr = (cols + 31) / 32;
    const int threads = 256;
    unpack_kernel<<<grid_for(rows * cols, threads), threads, 0, stream>>>(packed, rows, cols, wpr, out);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

int transpose_device(const uint32_t* packed, int64_t rows, int64_t cols, uint32_t* out, cudaStream_t stream) {
    const int64_t wpr_in = (cols + 31) / 32, wpr_out = (rows + 31) / 32;
    const int threads = 256;
    const int64_t tiles = ((rows + 31) / 32) * wpr_in;
    transpose_kernel<<<grid_for(tiles * 32, threads), threads, 0, stream>>>(packed, rows, cols, wpr_in, wpr_out, out);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_CUDA;
}

}  // namespace nq
